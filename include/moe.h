/*
 * moe.h -- C ABI of the single-GPU Mixture-of-Experts feed-forward layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer is the moe_ffn pseudocode of "Decoding Trillion-Parameter MoE
 * LLMs: Sparse Architecture and Agentic Intelligence", section "Routing:
 * Top-K Experts Plus a Shared Expert":
 *
 *   logits = x Wr^T                                   router GEMM     [T, E]
 *   idx, w = top-k of the scores, renormalised        moe_route       [T, k]
 *   rows of x grouped by expert (dispatch on 1 GPU)   moe_permute     [T*k, d]
 *   h = silu(x W1^T) * (x W3^T);  y = h W2^T          moe_grouped_ffn per expert
 *   out[t] = sum_j w[t,j] y[row(t,j)] + shared(x[t])   moe_combine     [T, d]
 *
 * moe_layer_forward runs all of it on one stream.
 *
 * Conventions (all entry points):
 *  - Every pointer argument is caller-owned DEVICE memory unless stated.  The
 *    library allocates nothing and keeps no state between calls; a caller-
 *    provided workspace holds every intermediate.
 *  - Every call is asynchronous on `stream` (stream-ordered), except
 *    moe_workspace_size, moe_status_string and moe_read_device_status.
 *  - Host-side checks run before any launch; a failed check launches nothing
 *    and returns MOE_ERR_INVALID_ARG (null pointer, non-positive size),
 *    MOE_ERR_UNSUPPORTED (k > E, k > 16, E > 1024, d % 128, I % 128, d > 16384,
 *    I > 16384, T*k >= 2^31, n_shared > 8, unsupported dtype combination) or
 *    MOE_ERR_WORKSPACE (workspace too small).  A launch error returns
 *    MOE_ERR_CUDA.
 *  - Faults the device detects (an expert index outside [0, E) fed to
 *    moe_permute; an FP8 block scale that is not a positive normal power of
 *    two; a bounded wait inside a kernel that ran out) are written to
 *    a status word in the first bytes of the workspace, never trapped; read
 *    it with moe_read_device_status.  The workspace must start zeroed once
 *    (moe_reset_device_status) before its first use.
 *  - Matrices are row-major.  Weight matrices are K-major ("nn.Linear"
 *    layout [out_features, in_features]).
 *  - dtypes: activations MOE_BF16, MOE_E4M3 (with fp32 1x128 scales) or
 *    MOE_F32; weights the same family (bf16 weights with bf16 activations,
 *    e4m3 weights + fp32 128x128 block scales with e4m3 activations, f32 with
 *    f32), or MOE_E2M1 (MXFP4) weights with MOE_E4M3 activations; or MOE_BF16
 *    activations with MOE_E4M3 or MOE_E2M1 weights, quantised to e4m3 in the
 *    permutation (see moe_permute).  f32 inputs are rounded to bf16 (nearest
 *    even) on entry; the tensor cores compute in bf16 (or e4m3 / e2m1 x e4m3)
 *    with fp32 accumulation.  The router weights are bf16 for the bf16, e4m3 and
 *    e2m1 families, f32 for f32; the router takes x as given (bf16, or e4m3
 *    dequantised exactly).
 *    FP8 block scales must be positive normal powers of two (exactly what the
 *    tensor cores' UE8M0 scale factors represent); any other scale sets the
 *    device status MOE_ERR_DEVICE_VALUE.  MXFP4 scale bytes are used as given
 *    (code 0xFF, NaN in E8M0, gives undefined results).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_DEVICE_INDEX = 5,   /* device status: an expert index outside [0, E) */
  MOE_ERR_TIMEOUT = 6,        /* device status: a bounded in-kernel wait ran out */
  MOE_ERR_DEVICE_VALUE = 7    /* device status: an FP8 block scale that is not a positive,
                                 normal power of two (the tensor cores take the scale's
                                 exponent only); the results of that call are not valid */
} moe_status;

/* Router score function.
 * SOFTMAX: select the k largest logits; gate_j = exp(l_j - max) / sum over the
 *   selected (the "topk_softmax" of the pseudocode).
 * SIGMOID_BIAS: s = sigmoid(l); select the k largest s + sel_bias[e]; gate_j =
 *   s_j / sum over the selected s (the bias steers selection only) -- the
 *   "auxiliary-loss-free bias routing" named by "Chapter 7: Serving Mega MoE
 *   at scale", roadmap item "Architectural Foundations of Trillion-Parameter
 *   Sparse MoE Models".
 * Both: the k slots of a token are ordered by selection key descending,
 * equal keys by lower expert index. */
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID_BIAS = 1 } moe_score_fn;

/* MOE_E2M1: FP4 weights in the OCP MXFP4 format -- E2M1 codes packed two per byte (element
 * 2j in the low nibble of byte j), one E8M0 scale byte (2^(code - 127)) per 32 consecutive
 * elements along K -- taken with e4m3 activations ("FP8/FP4 grouped GEMM", GC-MoE title).
 * The scale bytes of a [rows, K] weight matrix are stored as 512-byte atoms, one per 128
 * rows x 128 K-elements, [rows/128][K/128][512]: inside an atom the scale of row r (0..127)
 * and 32-element run q (0..3) sits at byte (r % 32) * 16 + (r / 32) * 4 + q -- the layout
 * the tensor cores' scale-factor copy takes, so the kernels copy atoms without reshuffling. */
/* MOE_E4M3_FP32_SCALE: e4m3 values whose fp32 block scales (1x128 for activations, 128x128
 * for weights, as for MOE_E4M3) may be any positive finite value, not only powers of two.
 * The expert GEMMs then multiply without block scaling and fold each 128-K block's
 * s_weight * s_activation into fp32 accumulators (exact up to fp32 rounding), on 32-token
 * tiles for decode-sized batches and 64-token tiles above: slower than MOE_E4M3, whose
 * power-of-two scales the tensor cores apply directly.
 * Activations and weights both take this dtype.  The router takes x = code x scale as a
 * bf16 part plus its bf16 remainder (two router GEMMs, summed with the split-K partials):
 * x to ~2^-17 relative, where a single bf16 rounding would move the logits by ~2^-9. */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_E4M3 = 2, MOE_E2M1 = 3, MOE_E4M3_FP32_SCALE = 4 } moe_dtype;

/* The layer's sizes: T tokens x d_model activations, E routed experts, top_k,
 * expert intermediate size d_ff (I), n_shared always-on shared experts of
 * intermediate d_ff_shared (must equal d_ff).  `out` is MOE_BF16 or MOE_F32. */
typedef struct {
  int32_t T, d_model, E, top_k, d_ff, n_shared, d_ff_shared;
  moe_score_fn score;
  moe_dtype act, weight, out;
} moe_config;

/* Weights of one layer (device pointers).
 *   wr     [E, d]          router weights (bf16; f32 for the f32 family)
 *   sel_bias [E] fp32      selection bias (SIGMOID_BIAS only; may be NULL = 0)
 *   w13    [E, 2I, d]      per expert: W1 (gate, rows 0..I-1) over W3 (up, rows I..2I-1)
 *   w2     [E, d, I]       per expert down projection
 *   w13_s, w2_s            block scales of the weights:
 *                          e4m3: fp32 [E, 2I/128, d/128] and [E, d/128, I/128];
 *                          e2m1: uint8 E8M0 codes in scale atoms (see MOE_E2M1),
 *                          [E, 2I/128, d/128, 512] and [E, d/128, I/128, 512],
 *                          16-byte aligned (w13 is then [E, 2I, d/2] bytes, w2
 *                          [E, d, I/2], both 32-byte aligned); unused (NULL) otherwise
 *   ws13 [S, 2I, d], ws2 [S, d, I] (+ ws13_s, ws2_s): shared experts (NULL when S = 0) */
typedef struct {
  const void *wr;
  const float *sel_bias;
  const void *w13, *w2;
  const void *w13_s, *w2_s;
  const void *ws13, *ws2;
  const void *ws13_s, *ws2_s;
} moe_weights;

/* Bytes of workspace moe_layer_forward / moe_permute / moe_grouped_ffn need
 * for `cfg` (the largest of the three).  Host only; no CUDA call. */
MOE_API moe_status moe_workspace_size(const moe_config *cfg, size_t *bytes);

/* Router top-k and gates ("topk_softmax" step).
 *   logits   [T, E] fp32   router logits (input)
 *   sel_bias [E] fp32 or NULL (SIGMOID_BIAS only)
 *   topk_idx [T, k] int32  selected experts, slot order as above (output)
 *   topk_w   [T, k] fp32   renormalised gates (output)
 * One warp per token; no workspace. */
MOE_API moe_status moe_route(const moe_config *cfg, const float *logits, const float *sel_bias,
                     int32_t *topk_idx, float *topk_w, cudaStream_t stream);

/* Dispatch on one GPU: a stable permutation of the T*k (token, slot) pairs into
 * per-expert contiguous groups, expert-major, ascending token inside a group
 * (the pseudocode's `dispatch(experts, idx)` without the all-to-all).
 *   topk_idx      [T, k] int32 (input); an entry outside [0, E) sets the device
 *                 status MOE_ERR_DEVICE_INDEX and that pair is dropped
 *   x             [T, d] activations (cfg->act); x_scale [T, d/128] fp32 (e4m3) or NULL
 *   x_perm        [T*k, d] permuted rows (output, same dtype as x);
 *                 x_perm_scale [T*k, d/128] (e4m3) or NULL
 *   perm_token    [T*k] int32  token of each permuted row (output)
 *   inv_perm      [T, k] int32 permuted row of (token, slot) (output)
 *   group_offsets [E+1] int32  exclusive prefix of group sizes (output)
 *   ws, ws_bytes  workspace (>= moe_workspace_size)
 * Quantise-in-permute: with bf16 activations and e4m3 or FP4 expert weights
 * (cfg->act MOE_BF16, cfg->weight MOE_E4M3 / MOE_E2M1) the rows are quantised to
 * e4m3 in the same pass, as the expert GEMMs take them: each token's 128-value
 * block gets the scale 2^e, e the smallest integer with amax <= 448 * 2^e (e = 0
 * for an all-zero block), and each value x becomes e4m3(x / 2^e), round to nearest
 * even.  x_perm [T*k, d] then receives e4m3 codes and x_perm_scale [T*k, d/128]
 * (required) the fp32 scales 2^e; x_scale is unused. */
MOE_API moe_status moe_permute(const moe_config *cfg, const int32_t *topk_idx, const void *x,
                       const float *x_scale, void *x_perm, float *x_perm_scale,
                       int32_t *perm_token, int32_t *inv_perm, int32_t *group_offsets,
                       void *ws, size_t ws_bytes, cudaStream_t stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory to give the library -- for instance a plugin whose host application
 * owns every device allocation through its own pool, or code on a latency path
 * where cudaMalloc (which may synchronise the device) is not allowed.  The pages
 * have no counterpart: it is the same permutation with the same arguments and
 * results as moe_permute, minus ws / ws_bytes.
 * bf16 rows for e4m3 or FP4 experts (the quantising permutation) are not taken
 * here: MOE_ERR_UNSUPPORTED.
 * Its scratch is a fixed array inside the library (about 1 MiB per GPU that
 * loads the library, held until the process exits), so it accepts only
 * ceil(T / 256) * E <= 262144 (for example T <= 65536 with E <= 1024); larger
 * shapes return MOE_ERR_UNSUPPORTED.  It calls no allocator.
 *  - The first call on a device looks up the array's device address (with that
 *    device current); make that first call before any stream capture.
 *  - Every call shares the one array, which keeps the previous call's contents;
 *    the call clears what must start at zero itself.  Calls whose kernels
 *    overlap on the GPU (several streams, or several host threads) race on it:
 *    serialise them.
 *  - Every dtype moe_permute takes: f32, bf16, and e4m3 rows, whose fp32
 *    1x128 scales x_scale [T, d/128] are permuted into x_perm_scale
 *    [T*k, d/128] (both required, non-NULL, when act is e4m3 and T > 0).
 *  - No device status is recorded.  Pairs with an expert index outside [0, E)
 *    are dropped (inv_perm = -1, not counted in group_offsets).  An expert
 *    listed twice in one token's row is not detected: both slots get the same
 *    permuted row, the group counts it once, and a combine over this result
 *    adds that expert's output twice.  moe_permute reports both faults as
 *    MOE_ERR_DEVICE_INDEX; call it where the indices are untrusted. */
MOE_API moe_status moe_permute_noalloc(const moe_config *cfg, const int32_t *topk_idx,
                                       const void *x, const float *x_scale, void *x_perm,
                                       float *x_perm_scale, int32_t *perm_token,
                                       int32_t *inv_perm, int32_t *group_offsets,
                                       cudaStream_t stream);

/* Grouped SwiGLU expert FFN over ragged groups (one expert per group):
 *   y[r] = (silu(a[r] W1_g^T) * (a[r] W3_g^T)) W2_g^T  for rows r of group g.
 *   n_groups        G (<= E + n_shared of cfg, which sizes the workspace); group g
 *                   uses weights w13[g], w2[g]
 *   group_offsets   [G+1] int32 DEVICE array of row offsets into a / y
 *                   (non-decreasing; read on the device, never copied to the host).
 *                   Offsets that decrease or pass n_rows set the device status
 *                   MOE_ERR_DEVICE_INDEX and the layer computes nothing.
 *   n_rows          rows allocated in a and y (>= offsets[G], <= T*k + n_shared*T,
 *                   the most the workspace holds); nothing past row n_rows is
 *                   read or written
 *   a               [offsets[G], d] rows in the token dtype of the expert GEMMs:
 *                   cfg->act, except e4m3 whenever the weights are e4m3 or FP4
 *                   (as moe_permute returns them); a_scale [rows, d/128] fp32 for
 *                   e4m3 rows, else NULL.  For the f32 family a, w13 and w2 are
 *                   rounded to bf16 into the workspace first.
 *   w13, w2         [G, 2I, d], [G, d, I] (+ block scales for e4m3 and e2m1 weights,
 *                   laid out as in moe_weights)
 *   y               [offsets[G], d] bf16 output
 * The shared expert is this call with n_groups = 1, offsets {0, T}, a = x.
 * The intermediate h lives in the workspace.  A persistent tcgen05/TMA kernel
 * walks the groups with a device-side tile scheduler (no host sync). */
MOE_API moe_status moe_grouped_ffn(const moe_config *cfg, int32_t n_groups, const int32_t *group_offsets,
                           int32_t n_rows, const void *a, const float *a_scale, const void *w13,
                           const void *w13_s, const void *w2, const void *w2_s, void *y,
                           void *ws, size_t ws_bytes, cudaStream_t stream);

/* Weighted un-permute (the pseudocode's `out += weights[..., k] * e(x)` and
 * `out += s(x)`): out[t] = sum_j topk_w[t,j] * y_perm[inv_perm[t,j]]
 * + sum_s y_shared[s, t], summed in slot order, then shared expert order, in
 * fp32 registers (no atomics), rounded once and written as cfg->out.
 *   y_perm [T*k, d] bf16; inv_perm [T, k] int32 (entries outside [0, T*k) add 0);
 *   topk_w [T, k] fp32;
 *   y_shared [cfg->n_shared, T, d] bf16: the shared experts' outputs stacked, or
 *            NULL (nothing added; also when cfg->n_shared = 0 any pointer is ignored);
 *   y [T, d] (output). */
MOE_API moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *inv_perm,
                       const float *topk_w, const void *y_shared, void *y, cudaStream_t stream);

/* The whole layer: router GEMM, route, permute, grouped routed + shared expert
 * FFN, combine.  x [T, d] (+ x_scale for e4m3); y [T, d] (cfg->out).
 * topk_idx_out [T, k] / topk_w_out [T, k] receive the routing when non-NULL. */
MOE_API moe_status moe_layer_forward(const moe_config *cfg, const moe_weights *weights, const void *x,
                             const float *x_scale, void *y, int32_t *topk_idx_out,
                             float *topk_w_out, void *ws, size_t ws_bytes, cudaStream_t stream);

/* moe_layer_forward that also records stage_events[0..7] (host array of 8
 * caller-created CUDA events) on `stream`: before the router GEMM and after
 * each of router GEMM, route, permute, tile plan, FFN1 (gate/up GEMM +
 * SwiGLU), FFN2 (down GEMM), combine -- so a caller can time every kernel of
 * the layer in place with cudaEventElapsedTime.  Same results as
 * moe_layer_forward; any null event -> MOE_ERR_INVALID_ARG. */
MOE_API moe_status moe_layer_forward_staged(const moe_config *cfg, const moe_weights *weights,
                                            const void *x, const float *x_scale, void *y,
                                            int32_t *topk_idx_out, float *topk_w_out, void *ws,
                                            size_t ws_bytes, cudaStream_t stream,
                                            cudaEvent_t *stage_events);

/* The whole layer recorded once into a CUDA graph and replayed: every kernel of
 * moe_layer_forward (8 to 14 launches) goes to the GPU as one graph launch, which
 * removes the per-launch host cost and the gaps between the layer's kernels on a
 * decode step ("Fused single-kernel decode layer ... or a CUDA-graph capture"; the
 * 3-node CUDA graph of the GC-MoE key changes).
 *  moe_layer_graph_create  checks its arguments as moe_layer_forward does, then
 *      records the layer for exactly these pointers and sizes on an internal stream
 *      (no kernel runs) and instantiates the graph into *graph_out.  The graph reads x
 *      (and x_scale) and writes y, the routing outputs and ws at the addresses given
 *      here: to run the layer on new activations, write them into x and launch again.
 *      It allocates host memory for the handle and the graph; no device memory.
 *  moe_layer_graph_launch  enqueues one layer call on `stream` (stream-ordered, like
 *      moe_layer_forward).  Launches of one graph must not overlap on the GPU: they
 *      share the workspace.
 *  moe_layer_graph_destroy frees the handle (after its launches have completed). */
typedef struct moe_layer_graph_t *moe_layer_graph;
MOE_API moe_status moe_layer_graph_create(const moe_config *cfg, const moe_weights *weights,
                                          const void *x, const float *x_scale, void *y,
                                          int32_t *topk_idx_out, float *topk_w_out, void *ws,
                                          size_t ws_bytes, moe_layer_graph *graph_out);
MOE_API moe_status moe_layer_graph_launch(moe_layer_graph graph, cudaStream_t stream);
MOE_API moe_status moe_layer_graph_destroy(moe_layer_graph graph);

/* Self-test of the device-side failure path (no counterpart on the pages): a
 * tiny kernel waits on a barrier that nothing completes, gives up after
 * `budget_cycles` SM clock cycles (1 .. 2^33), writes MOE_ERR_TIMEOUT into the
 * status word of workspace `ws` and returns -- the bounded-wait path every
 * tcgen05 kernel of the library takes instead of hanging.  Asynchronous; read
 * the result with moe_read_device_status. */
MOE_API moe_status moe_selftest_bounded_wait(void *ws, long long budget_cycles, cudaStream_t stream);

/* Synchronises `stream`, then reads the device status word of workspace `ws`
 * into *out (MOE_OK when no device fault was recorded).  Does not clear it. */
MOE_API moe_status moe_read_device_status(const void *ws, cudaStream_t stream, moe_status *out);

/* Zeroes the device status word (and the workspace header) of `ws`, on `stream`. */
MOE_API moe_status moe_reset_device_status(void *ws, cudaStream_t stream);

/* Static text for a status code. */
MOE_API const char *moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
