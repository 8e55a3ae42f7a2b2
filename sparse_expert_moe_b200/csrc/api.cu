// api.cu -- the C ABI declared in include/moe.h: host-side validation,
// workspace carving, TMA descriptor encoding and the launch sequence.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;
// header words
constexpr int kHdrStatus = 0;
constexpr int kHdrPermuteDone = 1;
constexpr int kHdrNChunks = 2;
constexpr int kHdrNGroups = 3;

inline size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

// The expert GEMMs take e4m3 token rows: e4m3 activations, or bf16 activations quantised
// in the permutation because the expert weights are e4m3 or FP4.
inline bool tok_e4m3(const moe_config& c) {
  return c.act == MOE_E4M3 || c.weight == MOE_E4M3 || c.weight == MOE_E2M1 ||
         c.act == MOE_E4M3_FP32_SCALE;
}
// e4m3 operands with arbitrary fp32 block scales (exact per-K-block rescale)
inline bool fp32_scaled(const moe_config& c) { return c.weight == MOE_E4M3_FP32_SCALE; }

// K splits of the router GEMM, and the partial logit arrays the route kernel sums: with
// fp32-scaled activations the router runs on x's bf16 part and on its bf16 remainder (two
// sets of splits, at most 32 partials in all).
inline int router_k_splits(const moe_config& c) {
  return router_splits(c.T, c.E, c.d_model, fp32_scaled(c) ? 16 : 32);
}
inline int router_parts(const moe_config& c) { return (fp32_scaled(c) ? 2 : 1) * router_k_splits(c); }
inline bool quant_in_permute(const moe_config& c) { return c.act == MOE_BF16 && tok_e4m3(c); }

// Byte offsets of every workspace region for one configuration.
struct Layout {
  size_t logits, topk_idx, topk_w, offsets, chunk_counts, perm_token, inv_perm, x_perm, chunks,
      grp_cp, h,
      y_rows, x_bf16, x_lo, wr_bf16, w13_bf16, w2_bf16, a_bf16, x_sf, x_perm_sf, h_sf, a_sf, wsf13, wsf2,
      total;
  int64_t R, rows_all, n_chunk_max;

  explicit Layout(const moe_config& c) {
    const int64_t T = c.T, d = c.d_model, E = c.E, k = c.top_k, I = c.d_ff, S = c.n_shared;
    R = T * k;
    rows_all = R + S * T;
    n_chunk_max = max_chunks(rows_all, E + S);
    const bool f32 = c.act == MOE_F32;
    const bool fp8 = tok_e4m3(c);                  // e4m3 token operand (e4m3 or FP4 weights)
    const bool q8 = fp8 && c.act == MOE_BF16;      // bf16 activations quantised in the permute
    const bool w8 = c.weight == MOE_E4M3;          // fp32 block scales re-encoded per call
    size_t o = kHeaderBytes;
    auto take = [&](size_t bytes) {
      const size_t at = o;
      o = align_up(o + bytes);
      return at;
    };
    logits = take(sizeof(float) * router_parts(c) * T * E);
    topk_idx = take(sizeof(int32_t) * R);
    topk_w = take(sizeof(float) * R);
    offsets = take(sizeof(int32_t) * (E + 1));
    chunk_counts = take(sizeof(int32_t) * permute_chunks(static_cast<int>(T)) * E);
    perm_token = take(sizeof(int32_t) * R);
    inv_perm = take(sizeof(int32_t) * R);
    x_perm = take(2 * R * d);
    chunks = take(sizeof(Chunk) * n_chunk_max);
    grp_cp = take(sizeof(int32_t) * 2 * (E + S + 1));
    h = take(2 * rows_all * I);
    y_rows = take(2 * rows_all * d);
    x_bf16 = take(f32 || fp8 ? 2 * T * d : 0);   // q8: the quantised x [T, d] e4m3
    x_lo = take(fp32_scaled(c) ? 2 * T * d : 0);  // bf16 remainder of fp32-scaled x
    (void)q8;
    wr_bf16 = take(f32 ? 2 * E * d : 0);
    w13_bf16 = take(f32 ? 2 * (E + S) * 2 * I * d : 0);
    w2_bf16 = take(f32 ? 2 * (E + S) * d * I : 0);
    a_bf16 = take(f32 ? 2 * rows_all * d : 0);
    // FP8: UE8M0 scale factors in the layouts the grouped GEMM's scale warp reads
    x_sf = take(fp8 ? 4 * (d / 128) * T : 0);
    x_perm_sf = take(fp8 ? 4 * (d / 128) * R : 0);
    h_sf = take(fp8 ? 4 * (I / 128) * rows_all : 0);
    a_sf = take(fp8 ? 4 * (d / 128) * rows_all : 0);
    wsf13 = take(w8 ? 16 * (E + S) * (2 * I / 128) * (d / 128) : 0);
    wsf2 = take(w8 ? 16 * (E + S) * (d / 128) * (I / 128) : 0);
    total = o;
  }
};

template <class T>
inline T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}
inline int* status_word(void* ws) { return at<int>(ws, kHdrStatus * sizeof(int)); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }


moe_status check_config(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d_model <= 0 || c->E <= 0 || c->top_k <= 0 || c->d_ff <= 0 ||
      c->n_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID_BIAS) return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->E || c->top_k > 16 || c->E > 1024) return MOE_ERR_UNSUPPORTED;
  if (c->d_model % 128 || c->d_ff % 128 || c->d_model > 16384 || c->d_ff > 16384)
    return MOE_ERR_UNSUPPORTED;
  if (c->n_shared > 8 || (c->n_shared > 0 && c->d_ff_shared != c->d_ff)) return MOE_ERR_UNSUPPORTED;
  const int64_t rows_all = static_cast<int64_t>(c->T) * (c->top_k + c->n_shared);
  if (rows_all >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  const bool fam_bf16 = c->act == MOE_BF16 && c->weight == MOE_BF16;
  const bool fam_f32 = c->act == MOE_F32 && c->weight == MOE_F32;
  const bool fam_fp8 = c->act == MOE_E4M3 && c->weight == MOE_E4M3;
  const bool fam_w4a8 = c->act == MOE_E4M3 && c->weight == MOE_E2M1;
  // bf16 activations into e4m3 or FP4 experts: quantised to e4m3 in the permutation
  const bool fam_q8 = c->act == MOE_BF16 && (c->weight == MOE_E4M3 || c->weight == MOE_E2M1);
  const bool fam_fs = c->act == MOE_E4M3_FP32_SCALE && c->weight == MOE_E4M3_FP32_SCALE;
  if (!(fam_bf16 || fam_f32 || fam_fp8 || fam_w4a8 || fam_q8 || fam_fs)) return MOE_ERR_UNSUPPORTED;
  if (c->out != MOE_BF16 && c->out != MOE_F32) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// bf16 chunk rows for groups of at most `max_group` rows: 32 for decode-sized batches
// (one token tile per chunk), else 256 (expert GEMM tiles of half a chunk).
int bf16_chunk_rows(int64_t max_group) {
  return max_group <= kChunkRows ? kChunkRowsNarrow : kChunkRowsWide;
}

// fp32-scale chunk rows: 32 for decode-sized batches, else 64 (the token tiles of the
// fp32-scale GEMMs, whose accumulators live in registers).
int fs_chunk_rows(int64_t max_group) {
  return max_group <= kChunkRows ? kChunkRowsNarrow : 2 * kChunkRowsNarrow;
}

// FP8 / FP4-weight chunk rows: 32 for decode-sized batches (groups of at most 128 rows:
// small token tiles leave shared memory to the weight stream), else 112, or 224 once
// groups can exceed 112 rows (FFN2 tiles of 224 tokens, FFN1 tiles of half a chunk).
int fp8_chunk_rows(int64_t max_group) {
  if (max_group <= kChunkRows) return kChunkRowsNarrow;
  return max_group <= kChunkRowsFP8 ? kChunkRowsFP8 : 2 * kChunkRowsFP8;
}

// ---------------------------------------------------------------- TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

moe_status validate_config(const moe_config* c) { return check_config(c); }

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols == 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_fp4(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols == 0 || cols % 128) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols / 2};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols == 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// Token-operand maps with boxes of 128, 64, 32 and 16 rows.
bool make_tok_maps(CUtensorMap (&m)[4], const void* base, uint64_t rows, uint64_t cols, bool u8) {
  for (int i = 0; i < 4; ++i) {
    const uint32_t box = 128u >> i;
    if (!(u8 ? make_tmap_u8(&m[i], base, rows, cols, box) : make_tmap_bf16(&m[i], base, rows, cols, box)))
      return false;
  }
  return true;
}
void copy_maps(CUtensorMap (&dst)[4], const CUtensorMap (&src)[4]) {
  for (int i = 0; i < 4; ++i) dst[i] = src[i];
}

// One segment of the FP8 block-scaled expert GEMMs: token rows `a` (e4m3) with their
// UE8M0 scale factors a_sf [d/128][a_rows], and `groups` experts' weights -- e4m3 with
// UE8M0 block scale factors wsf13 / wsf2 (re-encoded from the caller's fp32 128x128
// scales), or FP4 (packed E2M1) with the caller's E8M0 scale atoms wsc13 / wsc2.
struct Fp8Seg {
  const void* a;
  const uint32_t* a_sf;
  int64_t a_rows;
  const void* w13;
  const void* w2;
  const uint4* wsf13;
  const uint4* wsf2;
  const uint4* wsc13;
  const uint4* wsc2;
  int64_t groups;
  const int32_t* gidx;   // gather-on-load: token row n of a chunk is row gidx[b_row + n] of a
};

bool weight_map(CUtensorMap* m, const void* w, int64_t rows, int64_t cols, bool w4) {
  return w4 ? make_tmap_fp4(m, w, rows, cols, 128) : make_tmap_u8(m, w, rows, cols, 128);
}

// The FP8 block-scaled expert GEMMs over a chunk list already planned into the
// workspace: seg0 the routed rows, seg1 the shared experts (groups = 0: absent).  h
// (e4m3) and its scales live in the workspace; y has rows_all rows.
moe_status run_ffn_fp8(const moe_config& c, const Layout& L, void* ws, const Fp8Seg& s0,
                       const Fp8Seg& s1, int64_t rows_all, void* y, int chunk_rows, cudaStream_t s,
                       cudaEvent_t* ev = nullptr, bool gather = false) {
  const int64_t d = c.d_model, I = c.d_ff;
  const bool w4 = c.weight == MOE_E2M1;
  void* h = at<void>(ws, L.h);
  uint32_t* h_sf = at<uint32_t>(ws, L.h_sf);
  const Fp8Seg* seg[2] = {&s0, s1.groups > 0 ? &s1 : &s0};
  GemmLaunch g{};
  g.chunks = at<Chunk>(ws, L.chunks);
  g.n_chunks = at<int32_t>(ws, kHdrNChunks * sizeof(int));
  g.grp_cp = at<int32_t>(ws, L.grp_cp);
  g.n_grp = at<int32_t>(ws, kHdrNGroups * sizeof(int));
  g.status = status_word(ws);
  g.num_sms = num_sms();

  // FFN1 tiles hold 32 tokens on decode-sized chunks, else 112 (half a 224-row chunk when
  // chunks are 224 rows); FFN2 tiles are one chunk wide
  g.mode = w4 ? kFFN1F4 : kFFN1F8;
  g.halves = chunk_rows == 2 * kChunkRowsFP8;
  g.tile_tokens = chunk_rows == kChunkRowsNarrow ? kChunkRowsNarrow : kChunkRows;
  // gather-on-load: token rows straight from the (unpermuted) e4m3 activations
  g.gather = gather && chunk_rows != kChunkRowsNarrow;
  for (int i = 0; i < 2; ++i) {
    g.gsrc[i] = seg[i]->a;
    g.gidx[i] = seg[i]->gidx;
  }
  g.g_ld = static_cast<int>(d);
  for (int i = 0; i < 2; ++i) {
    const Fp8Seg& q = *seg[i];
    if (!weight_map(&g.wmap[i], q.w13, q.groups * 2 * I, d, w4) ||
        !make_tok_maps(g.tmap[i], q.a, q.a_rows, d, true))
      return MOE_ERR_CUDA;
    g.wsf[i] = q.wsf13;
    g.wsc[i] = q.wsc13;
    g.tsf[i] = q.a_sf;
    g.tsf_ld[i] = static_cast<int>(q.a_rows);
    g.tsf_rows[i] = static_cast<int>(q.a_rows);
  }
  g.n_mblk = static_cast<int>(I / 128);
  g.k_blocks = static_cast<int>(d / 128);
  g.w_rows_per_group = static_cast<int>(2 * I);
  g.wsf_rb_per_group = static_cast<int>(2 * I / 128);
  g.up_offset = static_cast<int>(I);
  g.m_valid = static_cast<int>(I);
  g.out = h;
  g.ld_out = static_cast<int>(I);
  g.out_sf = h_sf;
  g.ld_out_sf = static_cast<int>(rows_all);
  moe_status st = cuda_status(launch_gemm(g, s));
  if (st != MOE_OK) return st;
  if (ev && (st = cuda_status(cudaEventRecord(ev[0], s))) != MOE_OK) return st;

  // decode-sized token tiles: two 128-row weight blocks per tile (256 output columns), as
  // d_model allows
  const bool m256 = chunk_rows == kChunkRowsNarrow && d % 256 == 0;
  g.mode = m256 ? (w4 ? kFFN2F4M256 : kFFN2F8M256) : (w4 ? kFFN2F4 : kFFN2F8);
  g.halves = false;
  g.gather = false;
  g.tile_tokens = chunk_rows;
  if (!make_tok_maps(g.tmap[0], h, rows_all, I, true)) return MOE_ERR_CUDA;
  copy_maps(g.tmap[1], g.tmap[0]);
  for (int i = 0; i < 2; ++i) {
    const Fp8Seg& q = *seg[i];
    if (!weight_map(&g.wmap[i], q.w2, q.groups * d, I, w4)) return MOE_ERR_CUDA;
    g.wsf[i] = q.wsf2;
    g.wsc[i] = q.wsc2;
    g.tsf[i] = h_sf;
    g.tsf_ld[i] = static_cast<int>(rows_all);
    g.tsf_rows[i] = static_cast<int>(rows_all);
  }
  g.n_mblk = static_cast<int>(m256 ? d / 256 : d / 128);
  g.k_blocks = static_cast<int>(I / 128);
  g.w_rows_per_group = static_cast<int>(d);
  g.wsf_rb_per_group = static_cast<int>(d / 128);
  g.up_offset = 0;
  g.m_valid = static_cast<int>(d);
  g.out = y;
  g.ld_out = static_cast<int>(d);
  g.out_sf = nullptr;
  st = cuda_status(launch_gemm(g, s));
  if (st != MOE_OK) return st;
  if (ev) st = cuda_status(cudaEventRecord(ev[1], s));
  return st;
}

// The two expert GEMMs over a chunk list already planned into the workspace.
// seg 0: routed (a0 rows, w13_0 / w2_0 with G0 groups); seg 1: shared (a1 rows,
// w13_1 / w2_1 with S groups) or absent.  h and y have rows_all rows.
// The e4m3 expert GEMMs with arbitrary fp32 block scales over a chunk list of 32-row chunks
// planned into the workspace: seg0 the routed rows, seg1 the shared experts (groups = 0:
// absent).  a_scale: fp32 [a_rows][d/128]; w13_s / w2_s: fp32 128x128 block scales.  h
// (e4m3, power-of-two 1x128 scales as UE8M0 words) lives in the workspace.
struct FsSeg {
  const void* a;
  const float* a_scale;
  int64_t a_rows;
  const void* w13;
  const void* w2;
  const float* w13_s;
  const float* w2_s;
  int64_t groups;
};

moe_status run_ffn_fs(const moe_config& c, const Layout& L, void* ws, const FsSeg& s0,
                      const FsSeg& s1, int64_t rows_all, void* y, int chunk_rows, cudaStream_t s,
                      cudaEvent_t* ev = nullptr) {
  const int64_t d = c.d_model, I = c.d_ff;
  void* h = at<void>(ws, L.h);
  uint32_t* h_sf = at<uint32_t>(ws, L.h_sf);
  const FsSeg* seg[2] = {&s0, s1.groups > 0 ? &s1 : &s0};
  GemmLaunch g{};
  g.chunks = at<Chunk>(ws, L.chunks);
  g.n_chunks = at<int32_t>(ws, kHdrNChunks * sizeof(int));
  g.grp_cp = at<int32_t>(ws, L.grp_cp);
  g.n_grp = at<int32_t>(ws, kHdrNGroups * sizeof(int));
  g.status = status_word(ws);
  g.num_sms = num_sms();

  g.mode = kFFN1X;
  g.tile_tokens = chunk_rows;        // one chunk per tile: 32 or 64 tokens
  for (int i = 0; i < 2; ++i) {
    const FsSeg& q = *seg[i];
    if (!make_tmap_u8(&g.wmap[i], q.w13, q.groups * 2 * I, d, 128) ||
        !make_tok_maps(g.tmap[i], q.a, q.a_rows, d, true))
      return MOE_ERR_CUDA;
    g.fs_a[i] = q.a_scale;
    g.fs_w[i] = q.w13_s;
  }
  g.fs_a_ld = static_cast<int>(d / 128);
  g.n_mblk = static_cast<int>(I / 128);
  g.k_blocks = static_cast<int>(d / 128);
  g.w_rows_per_group = static_cast<int>(2 * I);
  g.wsf_rb_per_group = static_cast<int>(2 * I / 128);
  g.up_offset = static_cast<int>(I);
  g.m_valid = static_cast<int>(I);
  g.out = h;
  g.ld_out = static_cast<int>(I);
  g.out_sf = h_sf;
  g.ld_out_sf = static_cast<int>(rows_all);
  moe_status st = cuda_status(launch_gemm(g, s));
  if (st != MOE_OK) return st;
  if (ev && (st = cuda_status(cudaEventRecord(ev[0], s))) != MOE_OK) return st;

  // two 128-row weight blocks (256 output columns) per tile, as d_model allows
  const bool m256 = d % 256 == 0;
  g.mode = m256 ? kFFN2XM256 : kFFN2X;
  if (!make_tok_maps(g.tmap[0], h, rows_all, I, true)) return MOE_ERR_CUDA;
  copy_maps(g.tmap[1], g.tmap[0]);
  for (int i = 0; i < 2; ++i) {
    const FsSeg& q = *seg[i];
    if (!make_tmap_u8(&g.wmap[i], q.w2, q.groups * d, I, 128)) return MOE_ERR_CUDA;
    g.fs_w[i] = q.w2_s;
    g.tsf[i] = h_sf;
    g.tsf_ld[i] = static_cast<int>(rows_all);
    g.tsf_rows[i] = static_cast<int>(rows_all);
  }
  g.n_mblk = static_cast<int>(m256 ? d / 256 : d / 128);
  g.k_blocks = static_cast<int>(I / 128);
  g.w_rows_per_group = static_cast<int>(d);
  g.wsf_rb_per_group = static_cast<int>(d / 128);
  g.up_offset = 0;
  g.m_valid = static_cast<int>(d);
  g.out = y;
  g.ld_out = static_cast<int>(d);
  g.out_sf = nullptr;
  st = cuda_status(launch_gemm(g, s));
  if (st != MOE_OK) return st;
  if (ev) st = cuda_status(cudaEventRecord(ev[1], s));
  return st;
}

moe_status run_ffn(const moe_config& c, const Layout& L, void* ws, const void* a0, int64_t a0_rows,
                   const void* w13_0, const void* w2_0, int64_t G0, const void* a1, int64_t a1_rows,
                   const void* w13_1, const void* w2_1, int64_t S, int64_t rows_all, void* y,
                   int chunk_rows, cudaStream_t s, cudaEvent_t* ev = nullptr) {
  const int64_t d = c.d_model, I = c.d_ff;
  void* h = at<void>(ws, L.h);
  GemmLaunch g{};
  g.chunks = at<Chunk>(ws, L.chunks);
  g.n_chunks = at<int32_t>(ws, kHdrNChunks * sizeof(int));
  g.grp_cp = at<int32_t>(ws, L.grp_cp);
  g.n_grp = at<int32_t>(ws, kHdrNGroups * sizeof(int));
  g.status = status_word(ws);
  g.num_sms = num_sms();

  // FFN1 keeps single-CTA 128-token tiles (two accumulator buffers overlap its SwiGLU
  // epilogue with the next tile's MMAs); on 256-row chunks each tile takes half a chunk.
  // FFN2 stages several 128-row weight blocks per K block (its tiles span 256 output
  // columns, 512 on decode-sized token tiles), as d_model allows; with d_model not a
  // multiple of 256, one 128-row block on whole chunks.
  g.mode = kFFN1;
  g.tile_tokens = chunk_rows == kChunkRowsWide ? kChunkRows : chunk_rows;
  g.halves = chunk_rows == kChunkRowsWide;
  if (!make_tmap_bf16(&g.wmap[0], w13_0, G0 * 2 * I, d, 128) ||
      !make_tok_maps(g.tmap[0], a0, a0_rows, d, false))
    return MOE_ERR_CUDA;
  if (S > 0) {
    if (!make_tmap_bf16(&g.wmap[1], w13_1, S * 2 * I, d, 128) ||
        !make_tok_maps(g.tmap[1], a1, a1_rows, d, false))
      return MOE_ERR_CUDA;
  } else {
    g.wmap[1] = g.wmap[0];
    copy_maps(g.tmap[1], g.tmap[0]);
  }
  g.n_mblk = static_cast<int>(I / 128);
  g.k_blocks = static_cast<int>(d / 64);
  g.w_rows_per_group = static_cast<int>(2 * I);
  g.up_offset = static_cast<int>(I);
  g.m_valid = static_cast<int>(I);
  g.out = h;
  g.ld_out = static_cast<int>(I);
  moe_status st = cuda_status(launch_gemm(g, s));
  if (st != MOE_OK) return st;
  if (ev && (st = cuda_status(cudaEventRecord(ev[0], s))) != MOE_OK) return st;

  g.gather = false;
  const bool m512 = d % 512 == 0 && chunk_rows == kChunkRowsNarrow;
  const bool m256 = d % 256 == 0 && !m512;
  g.mode = m512 ? kFFN2M512 : (m256 ? kFFN2M256 : kFFN2);
  g.halves = m256 && chunk_rows == kChunkRowsWide;
  g.tile_tokens = g.halves ? kChunkRows : chunk_rows;
  if (!make_tmap_bf16(&g.wmap[0], w2_0, G0 * d, I, 128) ||
      !make_tok_maps(g.tmap[0], h, rows_all, I, false))
    return MOE_ERR_CUDA;
  if (S > 0) {
    if (!make_tmap_bf16(&g.wmap[1], w2_1, S * d, I, 128)) return MOE_ERR_CUDA;
  } else {
    g.wmap[1] = g.wmap[0];
  }
  copy_maps(g.tmap[1], g.tmap[0]);
  g.n_mblk = static_cast<int>(m512 ? d / 512 : (m256 ? d / 256 : d / 128));
  g.k_blocks = static_cast<int>(I / 64);
  g.w_rows_per_group = static_cast<int>(d);
  g.up_offset = 0;
  g.m_valid = static_cast<int>(d);
  g.out = y;
  g.ld_out = static_cast<int>(d);
  st = cuda_status(launch_gemm(g, s));
  if (st != MOE_OK) return st;
  if (ev) st = cuda_status(cudaEventRecord(ev[1], s));
  return st;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_workspace_size(const moe_config* cfg, size_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  *bytes = Layout(*cfg).total;
  return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const float* logits, const float* sel_bias,
                     int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  const float* bias = cfg->score == MOE_SCORE_SIGMOID_BIAS ? sel_bias : nullptr;
  return cuda_status(launch_route(logits, 1, 0, bias, cfg->T, cfg->E, cfg->top_k, cfg->score,
                                  topk_idx, topk_w, stream));
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                       const float* x_scale, void* x_perm, float* x_perm_scale,
                       int32_t* perm_token, int32_t* inv_perm, int32_t* group_offsets, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!group_offsets || !ws) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_idx || !x || !x_perm || !perm_token || !inv_perm))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  const Layout L(*cfg);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (quant_in_permute(*cfg)) {   // bf16 rows -> e4m3 rows + fp32 power-of-two scales
    if (cfg->T > 0 && !x_perm_scale) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_permute_quant(
        topk_idx, cfg->T, cfg->E, cfg->top_k, x, cfg->d_model, x_perm, x_perm_scale, nullptr,
        nullptr, nullptr, perm_token, inv_perm, group_offsets, at<int32_t>(ws, L.chunk_counts),
        at<unsigned>(ws, kHdrPermuteDone * sizeof(int)), status_word(ws), stream));
  }
  const bool fp8 = cfg->act == MOE_E4M3 || cfg->act == MOE_E4M3_FP32_SCALE;
  if (fp8 && cfg->T > 0 && (!x_scale || !x_perm_scale)) return MOE_ERR_INVALID_ARG;
  const int elem = cfg->act == MOE_F32 ? 4 : (fp8 ? 1 : 2);
  return cuda_status(launch_permute(topk_idx, cfg->T, cfg->E, cfg->top_k, x, cfg->d_model * elem,
                                    fp8 ? x_scale : nullptr, fp8 ? cfg->d_model / 128 : 0, x_perm,
                                    fp8 ? x_perm_scale : nullptr, perm_token, inv_perm,
                                    group_offsets, at<int32_t>(ws, L.chunk_counts),
                                    at<unsigned>(ws, kHdrPermuteDone * sizeof(int)),
                                    status_word(ws), stream));
}

moe_status moe_grouped_ffn(const moe_config* cfg, int32_t n_groups, const int32_t* group_offsets,
                           int32_t n_rows, const void* a, const float* a_scale, const void* w13,
                           const void* w13_s, const void* w2, const void* w2_s, void* y,
                           void* ws, size_t ws_bytes, cudaStream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (n_groups <= 0 || n_groups > 1024 || n_rows < 0) return MOE_ERR_INVALID_ARG;
  if (!group_offsets || !a || !w13 || !w2 || !y || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w13) || !aligned16(w2) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  // packed FP4 weights are loaded by TMA from 32-byte aligned bases, their scale atoms in
  // 16-byte copies
  if (cfg->weight == MOE_E2M1 && (!aligned32(w13) || !aligned32(w2) || !aligned16(w13_s) ||
                                  !aligned16(w2_s)))
    return MOE_ERR_INVALID_ARG;
  const Layout L(*cfg);
  if (n_rows > L.rows_all) return MOE_ERR_UNSUPPORTED;
  // the workspace's chunk list and group tables are sized for E + n_shared groups
  if (n_groups > cfg->E + cfg->n_shared) return MOE_ERR_UNSUPPORTED;
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (n_rows == 0) return MOE_OK;
  const int64_t d = cfg->d_model, I = cfg->d_ff;
  const void* a_b = a;
  const void* w13_b = w13;
  const void* w2_b = w2;
  if (cfg->act == MOE_F32) {
    st = cuda_status(launch_f32_to_bf16(static_cast<const float*>(a), at<void>(ws, L.a_bf16),
                                        static_cast<size_t>(n_rows) * d, stream));
    if (st == MOE_OK)
      st = cuda_status(launch_f32_to_bf16(static_cast<const float*>(w13), at<void>(ws, L.w13_bf16),
                                          static_cast<size_t>(n_groups) * 2 * I * d, stream));
    if (st == MOE_OK)
      st = cuda_status(launch_f32_to_bf16(static_cast<const float*>(w2), at<void>(ws, L.w2_bf16),
                                          static_cast<size_t>(n_groups) * d * I, stream));
    if (st != MOE_OK) return st;
    a_b = at<void>(ws, L.a_bf16);
    w13_b = at<void>(ws, L.w13_bf16);
    w2_b = at<void>(ws, L.w2_bf16);
  }
  if (fp32_scaled(*cfg)) {   // e4m3 rows and weights with arbitrary fp32 block scales
    if (!a_scale || !w13_s || !w2_s) return MOE_ERR_INVALID_ARG;
    const int chunk_rows = fs_chunk_rows(n_rows);
    st = cuda_status(launch_plan(group_offsets, n_groups, n_rows, 0, cfg->T, 0, chunk_rows,
                                 at<Chunk>(ws, L.chunks), at<int32_t>(ws, kHdrNChunks * sizeof(int)),
                                 at<int32_t>(ws, L.grp_cp), at<int32_t>(ws, kHdrNGroups * sizeof(int)),
                                 status_word(ws), stream));
    if (st != MOE_OK) return st;
    const FsSeg s0{a, a_scale, n_rows, w13, w2, static_cast<const float*>(w13_s),
                   static_cast<const float*>(w2_s), n_groups};
    return run_ffn_fs(*cfg, L, ws, s0, FsSeg{}, n_rows, y, chunk_rows, stream);
  }
  if (tok_e4m3(*cfg)) {   // e4m3 token rows (as moe_permute gives them for e4m3 / FP4 experts)
    if (!a_scale || !w13_s || !w2_s) return MOE_ERR_INVALID_ARG;
    const bool w4 = cfg->weight == MOE_E2M1;
    uint32_t* a_sf = at<uint32_t>(ws, L.a_sf);
    Fp8Seg s0{a, a_sf, n_rows, w13, w2, nullptr, nullptr, nullptr, nullptr, n_groups, nullptr};
    st = cuda_status(launch_act_prep_fp8(static_cast<const uint8_t*>(a), a_scale, n_rows,
                                         static_cast<int>(d), nullptr, a_sf, status_word(ws), stream));
    if (w4) {
      s0.wsc13 = static_cast<const uint4*>(w13_s);
      s0.wsc2 = static_cast<const uint4*>(w2_s);
    } else {
      s0.wsf13 = at<uint4>(ws, L.wsf13);
      s0.wsf2 = at<uint4>(ws, L.wsf2);
      if (st == MOE_OK)
        st = cuda_status(launch_weight_sf(static_cast<const float*>(w13_s),
                                          static_cast<size_t>(n_groups) * (2 * I / 128) * (d / 128),
                                          at<uint4>(ws, L.wsf13), status_word(ws), stream));
      if (st == MOE_OK)
        st = cuda_status(launch_weight_sf(static_cast<const float*>(w2_s),
                                          static_cast<size_t>(n_groups) * (d / 128) * (I / 128),
                                          at<uint4>(ws, L.wsf2), status_word(ws), stream));
    }
    const int chunk_rows = fp8_chunk_rows(n_rows);
    if (st == MOE_OK)
      st = cuda_status(launch_plan(group_offsets, n_groups, n_rows, 0, cfg->T, 0, chunk_rows,
                                   at<Chunk>(ws, L.chunks), at<int32_t>(ws, kHdrNChunks * sizeof(int)),
                                   at<int32_t>(ws, L.grp_cp), at<int32_t>(ws, kHdrNGroups * sizeof(int)),
                                   status_word(ws), stream));
    if (st != MOE_OK) return st;
    const Fp8Seg none{};
    return run_ffn_fp8(*cfg, L, ws, s0, none, n_rows, y, chunk_rows, stream);
  }
  const int chunk_rows = bf16_chunk_rows(n_rows);
  st = cuda_status(launch_plan(group_offsets, n_groups, n_rows, 0, cfg->T, 0, chunk_rows,
                               at<Chunk>(ws, L.chunks), at<int32_t>(ws, kHdrNChunks * sizeof(int)),
                               at<int32_t>(ws, L.grp_cp), at<int32_t>(ws, kHdrNGroups * sizeof(int)),
                               status_word(ws), stream));
  if (st != MOE_OK) return st;
  return run_ffn(*cfg, L, ws, a_b, n_rows, w13_b, w2_b, n_groups, nullptr, 0, nullptr, nullptr, 0,
                 n_rows, y, chunk_rows, stream);
}

moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* inv_perm,
                       const float* topk_w, const void* y_shared, void* y, cudaStream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!y_perm || !inv_perm || !topk_w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(y) || !aligned16(y_shared)) return MOE_ERR_INVALID_ARG;
  const int R = cfg->T * cfg->top_k;
  // y_shared holds the n_shared shared experts' outputs stacked [n_shared, T, d]
  return cuda_status(launch_combine(y_perm, inv_perm, topk_w, y_shared, y_shared ? cfg->n_shared : 0, cfg->T,
                                    cfg->d_model, cfg->top_k, R, cfg->out == MOE_F32, y, stream));
}

}  // extern "C"

namespace moe {
namespace {

// The whole layer.  When `ev` is non-null, ev[0..7] are recorded on the stream
// before the router GEMM and after each of: router GEMM, route, permute, plan,
// FFN1, FFN2, combine.
moe_status layer_forward_impl(const moe_config* cfg, const moe_weights* wts, const void* x,
                              const float* x_scale, void* y, int32_t* topk_idx_out,
                              float* topk_w_out, void* ws, size_t ws_bytes, cudaStream_t stream,
                              cudaEvent_t* ev) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!wts || !ws) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *cfg;
  if (c.T == 0) return MOE_OK;
  if (!x || !y || !wts->wr || !wts->w13 || !wts->w2) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && (!wts->ws13 || !wts->ws2)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(wts->wr) || !aligned16(wts->w13) ||
      !aligned16(wts->w2) || !aligned16(wts->ws13) || !aligned16(wts->ws2))
    return MOE_ERR_INVALID_ARG;
  const bool fp8 = tok_e4m3(c);            // e4m3 token operand of the expert GEMMs
  const bool q8 = quant_in_permute(c);     // ... quantised from bf16 x in the permutation
  const bool fs = fp32_scaled(c);          // ... with arbitrary fp32 block scales
  const bool w4 = c.weight == MOE_E2M1;
  if (fp8 && ((!q8 && !x_scale) || !wts->w13_s || !wts->w2_s ||
              (c.n_shared > 0 && (!wts->ws13_s || !wts->ws2_s))))
    return MOE_ERR_INVALID_ARG;
  // packed FP4 weights are loaded by TMA from 32-byte aligned bases, their scale atoms in
  // 16-byte copies
  if (w4 && (!aligned32(wts->w13) || !aligned32(wts->w2) || !aligned32(wts->ws13) ||
             !aligned32(wts->ws2) || !aligned16(wts->w13_s) || !aligned16(wts->w2_s) ||
             !aligned16(wts->ws13_s) || !aligned16(wts->ws2_s)))
    return MOE_ERR_INVALID_ARG;
  const Layout L(c);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  const int64_t T = c.T, d = c.d_model, E = c.E, I = c.d_ff, S = c.n_shared;
  const int64_t R = L.R;
  cudaStream_t s = stream;
  int* status = status_word(ws);
  auto mark = [&](int i) {
    return ev ? cuda_status(cudaEventRecord(ev[i], s)) : MOE_OK;
  };

  // f32 family: round every input to bf16 once, into the workspace
  const void* x_b = x;
  const void* wr_b = wts->wr;
  const void* w13_b = wts->w13;
  const void* w2_b = wts->w2;
  const void* ws13_b = wts->ws13;
  const void* ws2_b = wts->ws2;
  if (c.act == MOE_F32) {
    auto conv = [&](const void* src, size_t off, size_t n) {
      return cuda_status(launch_f32_to_bf16(static_cast<const float*>(src), at<void>(ws, off), n, s));
    };
    st = conv(x, L.x_bf16, T * d);
    if (st == MOE_OK) st = conv(wts->wr, L.wr_bf16, E * d);
    if (st == MOE_OK) st = conv(wts->w13, L.w13_bf16, E * 2 * I * d);
    if (st == MOE_OK) st = conv(wts->w2, L.w2_bf16, E * d * I);
    if (st == MOE_OK && S > 0) st = conv(wts->ws13, L.w13_bf16 + 2 * E * 2 * I * d, S * 2 * I * d);
    if (st == MOE_OK && S > 0) st = conv(wts->ws2, L.w2_bf16 + 2 * E * d * I, S * d * I);
    if (st != MOE_OK) return st;
    x_b = at<void>(ws, L.x_bf16);
    wr_b = at<void>(ws, L.wr_bf16);
    w13_b = at<void>(ws, L.w13_bf16);
    w2_b = at<void>(ws, L.w2_bf16);
    ws13_b = at<char>(ws, L.w13_bf16) + 2 * E * 2 * I * d;
    ws2_b = at<char>(ws, L.w2_bf16) + 2 * E * d * I;
  }
  // FP8 family: bf16 copy of x for the router (exact) and UE8M0 scale factors
  const void* x_router = x_b;
  uint32_t* x_sf = at<uint32_t>(ws, L.x_sf);
  uint4* wsf13 = at<uint4>(ws, L.wsf13);
  uint4* wsf2 = at<uint4>(ws, L.wsf2);
  const size_t n13 = static_cast<size_t>(2 * I / 128) * (d / 128);
  const size_t n2 = static_cast<size_t>(d / 128) * (I / 128);
  if (fp8) {
    if (!q8)   // fp32-scaled rows: no UE8M0 factors (no power-of-two check), a bf16 remainder
      st = cuda_status(launch_act_prep_fp8(static_cast<const uint8_t*>(x), x_scale, c.T,
                                           static_cast<int>(d), at<void>(ws, L.x_bf16),
                                           fs ? nullptr : x_sf, status, s,
                                           fs ? at<void>(ws, L.x_lo) : nullptr));
    if (c.weight == MOE_E4M3) {   // power-of-two fp32 block scales -> UE8M0 scale factors
      auto wsf = [&](const void* src, size_t n, uint4* dst) {
        return cuda_status(launch_weight_sf(static_cast<const float*>(src), n, dst, status, s));
      };
      if (st == MOE_OK) st = wsf(wts->w13_s, E * n13, wsf13);
      if (st == MOE_OK) st = wsf(wts->w2_s, E * n2, wsf2);
      if (st == MOE_OK && S > 0) st = wsf(wts->ws13_s, S * n13, wsf13 + E * n13);
      if (st == MOE_OK && S > 0) st = wsf(wts->ws2_s, S * n2, wsf2 + E * n2);
    }
    if (st != MOE_OK) return st;
    if (!q8) x_router = at<void>(ws, L.x_bf16);    // e4m3 x dequantised for the router
  }

  // 1. router GEMM: logits[T, E] = x Wr^T (fp32)
  float* logits = at<float>(ws, L.logits);
  if ((st = mark(0)) != MOE_OK) return st;
  {
    GemmLaunch g{};
    g.mode = kRouter;
    if (!make_tmap_bf16(&g.wmap[0], wr_b, E, d, 128) || !make_tok_maps(g.tmap[0], x_router, T, d, false))
      return MOE_ERR_CUDA;
    g.wmap[1] = g.wmap[0];
    copy_maps(g.tmap[1], g.tmap[0]);
    g.router_T = static_cast<int>(T);
    g.n_mblk = static_cast<int>((E + 127) / 128);
    g.k_blocks = static_cast<int>(d / 64);
    g.k_splits = router_k_splits(c);
    g.split_stride = static_cast<long long>(T) * E;
    g.m_valid = static_cast<int>(E);
    g.out = logits;
    g.ld_out = static_cast<int>(E);
    g.status = status;
    g.num_sms = num_sms();
    st = cuda_status(launch_gemm(g, s));
    if (st != MOE_OK) return st;
    if (fs) {   // the bf16 remainder of x into the next set of partial logits
      if (!make_tok_maps(g.tmap[0], at<void>(ws, L.x_lo), T, d, false)) return MOE_ERR_CUDA;
      copy_maps(g.tmap[1], g.tmap[0]);
      g.out = logits + static_cast<size_t>(g.k_splits) * T * E;
      st = cuda_status(launch_gemm(g, s));
      if (st != MOE_OK) return st;
    }
  }
  if ((st = mark(1)) != MOE_OK) return st;

  // 2. route
  int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.topk_idx);
  float* gate = topk_w_out ? topk_w_out : at<float>(ws, L.topk_w);
  const float* bias = c.score == MOE_SCORE_SIGMOID_BIAS ? wts->sel_bias : nullptr;
  st = cuda_status(launch_route(logits, router_parts(c), static_cast<long long>(T) * E, bias,
                                c.T, c.E, c.top_k, c.score, idx, gate, s));
  if (st != MOE_OK) return st;
  if ((st = mark(2)) != MOE_OK) return st;

  // 3. permute.  Groups hold at most T rows, which picks the token-tile width of the expert
  // GEMMs.  With e4m3 token rows on wide tiles (more than 128 tokens) the first GEMM gathers
  // its token rows from x itself (gather-on-load), so only the routing tables are built
  // here; otherwise the rows are copied into x_perm (bf16 rows, or e4m3 rows + scale
  // factors).  bf16 rows keep the copy: measured on the R1 prefill layer, the first GEMM
  // fed by TMA from x_perm is faster than with gathered rows by more than the copy costs.
  const int chunk_rows = fs ? fs_chunk_rows(T) : (fp8 ? fp8_chunk_rows(T) : bf16_chunk_rows(T));
  // (the fp32-scale GEMMs read their token rows from x_perm at every width)
  const bool gather = fp8 && !fs && chunk_rows != kChunkRowsNarrow;
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm_token = at<int32_t>(ws, L.perm_token);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  void* x_perm = at<void>(ws, L.x_perm);
  uint32_t* x_perm_sf = at<uint32_t>(ws, L.x_perm_sf);
  int32_t* counts = at<int32_t>(ws, L.chunk_counts);
  unsigned* ticket = at<unsigned>(ws, kHdrPermuteDone * sizeof(int));
  const void* x_tok = x_b;     // the unpermuted token rows the expert GEMMs take
  if (q8) {
    // bf16 rows quantised to e4m3 in the copy: every token's own quantised row (the shared
    // experts' rows and, with gather-on-load, the routed ones) and, on decode-sized tiles,
    // x_perm with its UE8M0 scale words
    st = cuda_status(launch_permute_quant(idx, c.T, c.E, c.top_k, x_b, static_cast<int>(d),
                                          gather ? nullptr : x_perm, nullptr,
                                          gather ? nullptr : x_perm_sf, at<void>(ws, L.x_bf16), x_sf,
                                          perm_token, inv_perm, offsets, counts, ticket, status, s));
    x_tok = at<void>(ws, L.x_bf16);
  } else if (gather) {
    st = cuda_status(launch_permute_index(idx, c.T, c.E, c.top_k, perm_token, inv_perm, offsets,
                                          counts, ticket, status, s));
  } else if (fs) {   // e4m3 rows with their fp32 scales, [R][d/128]
    st = cuda_status(launch_permute(idx, c.T, c.E, c.top_k, x_b, static_cast<int>(d), x_scale,
                                    static_cast<int>(d / 128), x_perm,
                                    reinterpret_cast<float*>(x_perm_sf), perm_token, inv_perm,
                                    offsets, counts, ticket, status, s));
  } else {
    st = cuda_status(launch_permute(idx, c.T, c.E, c.top_k, x_b, static_cast<int>(fp8 ? d : d * 2),
                                    nullptr, 0, x_perm, nullptr, perm_token, inv_perm, offsets,
                                    counts, ticket, status, s));
    if (st == MOE_OK && fp8)
      st = cuda_status(launch_gather_sf(x_sf, c.T, static_cast<int>(d / 128), perm_token,
                                        offsets + E, static_cast<int>(R), x_perm_sf, s));
  }
  if (st != MOE_OK) return st;
  if ((st = mark(3)) != MOE_OK) return st;

  // 4. plan routed groups + shared experts, 5./6. the two grouped GEMMs.
  st = cuda_status(launch_plan(offsets, c.E, static_cast<int>(R), c.n_shared, c.T,
                               static_cast<int>(R), chunk_rows,
                               at<Chunk>(ws, L.chunks), at<int32_t>(ws, kHdrNChunks * sizeof(int)),
                               at<int32_t>(ws, L.grp_cp), at<int32_t>(ws, kHdrNGroups * sizeof(int)),
                               status, s));
  if (st != MOE_OK) return st;
  if ((st = mark(4)) != MOE_OK) return st;
  void* y_rows = at<void>(ws, L.y_rows);
  if (fs) {
    const FsSeg s0{x_perm, reinterpret_cast<const float*>(x_perm_sf), R, w13_b, w2_b,
                   static_cast<const float*>(wts->w13_s), static_cast<const float*>(wts->w2_s), E};
    const FsSeg s1{x_b, x_scale, T, ws13_b, ws2_b, static_cast<const float*>(wts->ws13_s),
                   static_cast<const float*>(wts->ws2_s), S};
    st = run_ffn_fs(c, L, ws, s0, s1, L.rows_all, y_rows, chunk_rows, s, ev ? ev + 5 : nullptr);
  } else if (fp8) {
    Fp8Seg s0{x_perm, x_perm_sf, R, w13_b, w2_b, nullptr, nullptr, nullptr, nullptr, E, nullptr};
    if (gather) s0 = Fp8Seg{x_tok, x_sf, T, w13_b, w2_b, nullptr, nullptr, nullptr, nullptr, E, perm_token};
    Fp8Seg s1{x_tok, x_sf, T, ws13_b, ws2_b, nullptr, nullptr, nullptr, nullptr, S, nullptr};
    if (w4) {
      s0.wsc13 = static_cast<const uint4*>(wts->w13_s);
      s0.wsc2 = static_cast<const uint4*>(wts->w2_s);
      s1.wsc13 = static_cast<const uint4*>(wts->ws13_s);
      s1.wsc2 = static_cast<const uint4*>(wts->ws2_s);
    } else {
      s0.wsf13 = wsf13;
      s0.wsf2 = wsf2;
      s1.wsf13 = wsf13 + E * n13;
      s1.wsf2 = wsf2 + E * n2;
    }
    st = run_ffn_fp8(c, L, ws, s0, s1, L.rows_all, y_rows, chunk_rows, s, ev ? ev + 5 : nullptr,
                     gather);
  } else {
    st = run_ffn(c, L, ws, x_perm, R, w13_b, w2_b, E, x_b, T, ws13_b, ws2_b, S, L.rows_all, y_rows,
                 chunk_rows, s, ev ? ev + 5 : nullptr);
  }
  if (st != MOE_OK) return st;

  // 7. combine
  const void* y_shared = S > 0 ? static_cast<const void*>(at<char>(ws, L.y_rows) + 2 * R * d) : nullptr;
  st = cuda_status(launch_combine(y_rows, inv_perm, gate, y_shared, c.n_shared, c.T, c.d_model,
                                  c.top_k, static_cast<int>(R), c.out == MOE_F32, y, s));
  if (st != MOE_OK) return st;
  return mark(7);
}

}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_layer_forward(const moe_config* cfg, const moe_weights* wts, const void* x,
                             const float* x_scale, void* y, int32_t* topk_idx_out,
                             float* topk_w_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return layer_forward_impl(cfg, wts, x, x_scale, y, topk_idx_out, topk_w_out, ws, ws_bytes, stream,
                            nullptr);
}

moe_status moe_layer_forward_staged(const moe_config* cfg, const moe_weights* wts, const void* x,
                                    const float* x_scale, void* y, int32_t* topk_idx_out,
                                    float* topk_w_out, void* ws, size_t ws_bytes,
                                    cudaStream_t stream, cudaEvent_t* stage_events) {
  if (!stage_events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 8; ++i)
    if (!stage_events[i]) return MOE_ERR_INVALID_ARG;
  return layer_forward_impl(cfg, wts, x, x_scale, y, topk_idx_out, topk_w_out, ws, ws_bytes, stream,
                            stage_events);
}

moe_status moe_read_device_status(const void* ws, cudaStream_t stream, moe_status* out) {
  if (!ws || !out) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  *out = static_cast<moe_status>(v);
  return MOE_OK;
}

}  // extern "C"

struct moe_layer_graph_t {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

extern "C" {

moe_status moe_layer_graph_create(const moe_config* cfg, const moe_weights* wts, const void* x,
                                  const float* x_scale, void* y, int32_t* topk_idx_out,
                                  float* topk_w_out, void* ws, size_t ws_bytes,
                                  moe_layer_graph* graph_out) {
  if (!graph_out) return MOE_ERR_INVALID_ARG;
  *graph_out = nullptr;
  // the host checks of the layer itself, before anything is recorded
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!wts || !ws) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < Layout(*cfg).total) return MOE_ERR_WORKSPACE;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
  moe_layer_graph_t* g = new moe_layer_graph_t();
  // relaxed mode: the launch helpers set kernel attributes while recording
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
    st = MOE_ERR_CUDA;
  } else {
    st = layer_forward_impl(cfg, wts, x, x_scale, y, topk_idx_out, topk_w_out, ws, ws_bytes, cs,
                            nullptr);
    const cudaError_t e = cudaStreamEndCapture(cs, &g->graph);
    if (st == MOE_OK && e != cudaSuccess) st = MOE_ERR_CUDA;
  }
  if (st == MOE_OK && cudaGraphInstantiate(&g->exec, g->graph, 0) != cudaSuccess) st = MOE_ERR_CUDA;
  cudaStreamDestroy(cs);
  if (st != MOE_OK) {
    moe_layer_graph_destroy(g);
    return st;
  }
  *graph_out = g;
  return MOE_OK;
}

moe_status moe_layer_graph_launch(moe_layer_graph graph, cudaStream_t stream) {
  if (!graph || !graph->exec) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaGraphLaunch(graph->exec, stream));
}

moe_status moe_layer_graph_destroy(moe_layer_graph graph) {
  if (!graph) return MOE_OK;
  moe_status st = MOE_OK;
  if (graph->exec && cudaGraphExecDestroy(graph->exec) != cudaSuccess) st = MOE_ERR_CUDA;
  if (graph->graph && cudaGraphDestroy(graph->graph) != cudaSuccess) st = MOE_ERR_CUDA;
  delete graph;
  return st;
}

moe_status moe_reset_device_status(void* ws, cudaStream_t stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, kHeaderBytes, stream));
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_INDEX: return "device: index or offset out of range";
    case MOE_ERR_TIMEOUT: return "device: bounded wait timed out";
    case MOE_ERR_DEVICE_VALUE: return "device: FP8 block scale not a positive normal power of two";
  }
  return "unknown status";
}

}  // extern "C"
