// internal.h -- declarations shared by the library's translation units (host side).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime_api.h>

#include "../../include/moe.h"

namespace moe {

// Host-side configuration checks shared by every entry point (MOE_OK or the error code).
moe_status validate_config(const moe_config* c);

// One group chunk of at most kChunkRows token rows, as produced by the tile
// planner and consumed by the grouped GEMM kernels.
//   seg    0 = routed groups (rows of the permuted activations),
//          1 = shared experts (rows of the unpermuted activations)
//   group  group (expert) index inside the segment: selects the weights
//   b_row  first row of the token operand (x_perm / x / h) the chunk reads
//   o_row  first row of the output (h / y) the chunk writes
//   nrows  rows in the chunk (1..kChunkRows)
struct Chunk {
  int32_t seg, group, b_row, o_row, nrows, pad0, pad1, pad2;
};

constexpr int kChunkRows = 128;     // tokens per GEMM tile, bf16 (UMMA N <= 128)
constexpr int kChunkRowsFP8 = 112;  // tokens per GEMM tile, FP8 (TMEM also holds scale factors)
constexpr int kChunkRowsWide = 256; // rows per chunk, bf16, once groups can exceed 128 rows
                                    // (tiles take half a chunk)
constexpr int kChunkRowsNarrow = 32; // tokens per GEMM tile, bf16 decode-sized batches
constexpr int kMaxGroups = 1024 + 8;

// Upper bound on the chunks of `rows` rows spread over `groups` groups.
inline int64_t max_chunks(int64_t rows, int64_t groups, int chunk_rows = kChunkRowsNarrow) {
  return rows / chunk_rows + groups + 1;
}

// ---------------------------------------------------------------- kernels
// logits: n_partials partial [T, E] arrays `partial_stride` floats apart, summed in
// order before scoring (1 = plain logits).
cudaError_t launch_route(const float* logits, int n_partials, long long partial_stride,
                         const float* sel_bias, int T, int E, int k, int score, int32_t* topk_idx,
                         float* topk_w, cudaStream_t s);

// K splits of the router GEMM for T tokens, E experts and d_model: about 48 CTAs
// when the (token chunk, expert block) tiles alone are fewer -- enough to stream
// Wr quickly, few enough that summing the partial logits stays cheap (at most 32, the
// route kernel's limit); every split non-empty.  Host only.
inline int router_splits(int64_t T, int64_t E, int64_t d, int64_t max_splits = 32) {
  const int64_t tiles = ((T + 127) / 128) * ((E + 127) / 128);
  const int64_t kb = d / 64;
  if (tiles == 0) return 1;                 // empty batch: nothing to split
  int64_t s = tiles >= 48 ? 1 : 48 / tiles;
  if (s > max_splits) s = max_splits;
  if (s > kb) s = kb;
  if (s < 1) s = 1;
  const int64_t per = (kb + s - 1) / s;
  return static_cast<int>((kb + per - 1) / per);
}

// Permutation.  `chunk_counts` holds ceil(T / 256) * E ints; `done` one zeroed
// counter (left zero on exit).
cudaError_t launch_permute(const int32_t* topk_idx, int T, int E, int k, const void* x,
                           int row_bytes, const float* x_scale, int scale_cols, void* x_perm,
                           float* x_perm_scale, int32_t* perm_token, int32_t* inv_perm,
                           int32_t* offsets, int32_t* chunk_counts, unsigned* done, int* status,
                           cudaStream_t s);
inline int permute_chunks(int T) { return (T + 255) / 256; }

// The routing tables of the permutation alone (group offsets, perm_token, inv_perm): the
// count (+ rank) kernels, no row copy.
cudaError_t launch_permute_index(const int32_t* topk_idx, int T, int E, int k, int32_t* perm_token,
                                 int32_t* inv_perm, int32_t* offsets, int32_t* chunk_counts,
                                 unsigned* done, int* status, cudaStream_t s);

// The permutation of bf16 rows [T, d] into e4m3 rows for e4m3 expert GEMMs, quantised in
// the copy (one power-of-two scale per token per 128 values, round to nearest even).  Block
// scales go to x_perm_scale ([T k][d/128] fp32) when it is non-null, else to x_perm_w as
// UE8M0 words ([d/128][T k]); x_q / x_q_w (both or neither): every token's own quantised
// row [T, d] and scale words [d/128][T].  x_perm null: only x_q / x_q_w are written.
cudaError_t launch_permute_quant(const int32_t* topk_idx, int T, int E, int k, const void* x_bf16,
                                 int d, void* x_perm, float* x_perm_scale, uint32_t* x_perm_w,
                                 void* x_q, uint32_t* x_q_w, int32_t* perm_token, int32_t* inv_perm,
                                 int32_t* offsets, int32_t* chunk_counts, unsigned* done,
                                 int* status, cudaStream_t s);

// Tile planner: routed groups (device offsets [G+1], rows <= n_rows) followed
// by n_shared groups of T rows each (token rows 0..T-1 of the unpermuted
// activations, output rows shared_o_row + s*T).  Heavy groups first.
// Also writes the chunk prefix of the groups in plan order (grp_cp [n_grp + 1]), then
// their prefix in half chunks (grp_cp[n_grp + 1 ..], n_grp + 1 entries), and the number
// of groups (n_grp); the GEMM kernels use them to order their tiles.
cudaError_t launch_plan(const int32_t* offsets, int G, int n_rows, int n_shared, int T,
                        int shared_o_row, int chunk_rows, Chunk* chunks, int32_t* n_chunks,
                        int32_t* grp_cp, int32_t* n_grp, int* status, cudaStream_t s);

// kFFN2M256 / kFFN2M512: FFN2 (bf16) with 256 / 512 weight rows per tile, as two / four
// 128-row blocks (M512: decode-sized token tiles only).  kFFN1F4 / kFFN2F4: the FP8 GEMMs
// with FP4 (MXFP4) weights.  kFFN2F8M256 / kFFN2F4M256: FP8 / FP4 FFN2 with two 128-row
// weight blocks per tile (decode-sized token tiles).  kFFN1X / kFFN2X: e4m3 GEMMs with
// arbitrary fp32 block scales (per-K-block partial sums rescaled in fp32).
enum GemmMode { kRouter = 0, kFFN1 = 1, kFFN2 = 2, kFFN1F8 = 3, kFFN2F8 = 4, kFFN2M256 = 5,
                kFFN2M512 = 6, kFFN1F4 = 7, kFFN2F4 = 8, kFFN2F8M256 = 9, kFFN2F4M256 = 10,
                kFFN1X = 11, kFFN2X = 12, kFFN2XM256 = 13 };

struct GemmLaunch {
  int mode;
  int tile_tokens;           // bf16 expert GEMMs: token-tile width (32, 128 or 256)
  bool halves;               // chunks are twice the tile width: one tile per half chunk
  // weight (A) maps per segment (boxes of 128 rows); token (B) maps per segment with
  // boxes of 128, 64, 32 and 16 rows
  CUtensorMap wmap[2];
  CUtensorMap tmap[2][4];
  const Chunk* chunks;       // device (FFN modes)
  const int32_t* n_chunks;   // device (FFN modes)
  const int32_t* grp_cp;     // device (FFN modes): plan-order group chunk prefix
  const int32_t* n_grp;      // device (FFN modes)
  int router_T;              // router mode: tokens
  int n_mblk;                // weight-row tiles per group (128 rows; 256 for kFFN2M256)
  int k_blocks;              // K / 64 (bf16) or K / 128 (e4m3)
  int k_splits;              // router: K split across CTAs (1 = none); every split non-empty
  long long split_stride;    // router: elements between consecutive partial outputs
  int w_rows_per_group;      // weight rows per group (FFN1: 2I, FFN2: d)
  int up_offset;             // FFN1: I
  int m_valid;               // router: E
  void* out;
  int ld_out;
  int* status;
  int num_sms;
  // FP8 modes: weight block scales (UE8M0 replicated x16, [groups][row blocks][k blocks])
  // and token scales (UE8M0 replicated x4, [k blocks][rows]) per segment; FFN1 writes
  // the scales of its requantised output to out_sf ([I / 128][ld_out_sf]).
  const uint4* wsf[2];
  int wsf_rb_per_group;
  // gather-on-load (first GEMM, wide token tiles): token row n of a chunk is row
  // gidx[seg][b_row + n] (gidx null: b_row + n) of gsrc[seg], g_ld bytes apart
  bool gather;
  const void* gsrc[2];
  const int32_t* gidx[2];
  int g_ld;
  // fp32-scale modes: token scales fp32 [rows][fs_a_ld] (first GEMM) and weight block
  // scales fp32 [groups][row blocks][k blocks], per segment
  const float* fs_a[2];
  int fs_a_ld;
  const float* fs_w[2];
  // FP4 modes: E8M0 weight scale codes per segment in 512-byte atoms
  // [groups][rows / 128][K / 128][32 x 16 bytes] (row r, K run q at (r % 32) * 16 + (r / 32) * 4 + q)
  const uint4* wsc[2];
  const uint32_t* tsf[2];
  int tsf_ld[2];
  int tsf_rows[2];
  uint32_t* out_sf;
  int ld_out_sf;
};
cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t s);

// Tensor map of a row-major [rows, cols] matrix of 2-byte elements, box
// {64 columns, box_rows rows}, 128-byte swizzle.  Returns false on failure.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
// Same for 1-byte (e4m3) elements, box {128 columns, box_rows rows}.
bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows);
// Packed FP4 (two E2M1 codes per byte, `cols` elements per row), box {128 elements,
// box_rows rows}, loaded into shared memory unpacked to one 16-byte slot per 16 elements
// (8 data bytes, 8 bytes of gap): the e4m3 tile layout the block-scaled MMA reads FP4
// operands from.  Needs a 32-byte aligned base and cols a multiple of 128.
bool make_tmap_fp4(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows);

// FP8 preparation kernels.
// x e4m3 [T, d] + x_scale fp32 [T, d/128] -> x_bf16 [T, d] (exact) and x_sf [d/128][T]
// (UE8M0 replicated x4).  Either output may be null.  Scales that are not positive normal
// powers of two record MOE_ERR_DEVICE_VALUE in *status (both functions).
// x_lo (optional): the bf16 remainder v - bf16(v) of each value v = code x scale.
cudaError_t launch_act_prep_fp8(const uint8_t* x, const float* x_scale, int T, int d, void* x_bf16,
                                uint32_t* x_sf, int* status, cudaStream_t s, void* x_lo = nullptr);
// fp32 power-of-two block scales [n] -> UE8M0 replicated x16 [n] (uint4).
cudaError_t launch_weight_sf(const float* scales, size_t n, uint4* out, int* status, cudaStream_t s);
// x_perm_sf[kb][r] = x_sf[kb][perm_token[r]] for r < offsets_total (device).
cudaError_t launch_gather_sf(const uint32_t* x_sf, int T, int kbs, const int32_t* perm_token,
                             const int32_t* total, int R, uint32_t* x_perm_sf, cudaStream_t s);

cudaError_t launch_combine(const void* y_perm, const int32_t* inv_perm, const float* topk_w,
                           const void* y_shared, int n_shared, int T, int d, int k, int R,
                           bool out_f32, void* y, cudaStream_t s);

cudaError_t launch_f32_to_bf16(const float* src, void* dst, size_t n, cudaStream_t s);

}  // namespace moe
