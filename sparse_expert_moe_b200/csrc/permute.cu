// permute.cu -- dispatch on one GPU: stable permutation of (token, slot) pairs
// into per-expert contiguous groups (the `dispatch(experts, idx)` step of the
// moe_ffn pseudocode in "Decoding Trillion-Parameter MoE LLMs", section
// "Routing: Top-K Experts Plus a Shared Expert", without the all-to-all).
//
// Order: expert-major, ascending token inside a group -- the order a sort of
// the keys (expert, token) gives.  No atomics decide any position:
//  1. count: one CTA per chunk of 256 tokens (8 warps x 32 lanes).  Each warp
//     builds, per expert, a 32-bit mask of the lanes (tokens) that selected it
//     (shared-memory atomicOr: order-free).  Per-chunk counts go to global
//     memory; the last CTA to finish (global ticket) scans them into the group
//     offsets and per-(chunk, expert) base rows.
//  2. rank: each CTA rebuilds its masks; the row of (token t, slot j) with
//     expert e is base(chunk, e) + earlier warps' counts + popc(mask & lanes
//     below t).  With a single chunk (T <= 256) the count CTA, which still holds
//     the masks after the scan, ranks the pairs itself (one launch less).
//  3. copy: x_perm[inv_perm[t, j]] = x[t] for every slot j of token t.  One warp per
//     (token, 4 KB piece of its row) reads the piece once and writes it to the token's
//     k permuted rows, so x is read exactly once (a copy in permuted-row order re-reads
//     each token's row k times, and x does not stay in L2 between those reads at
//     prefill sizes).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kChunkTokens = kWarps * 32;

// Builds the per-warp lane masks of this CTA's chunk: masks[w * E + e].
__device__ __forceinline__ void build_masks(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                                            uint32_t* masks, int* status, bool report) {
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) masks[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kChunkTokens + threadIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(topk_idx + static_cast<size_t>(t) * k + j);
      if (e >= 0 && e < E) {
        const uint32_t old = atomicOr(&masks[warp * E + e], 1u << lane);
        if (report && (old & (1u << lane))) record_status(status, kStatusDeviceIndex);  // duplicate
      } else if (report) {
        record_status(status, kStatusDeviceIndex);
      }
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256) permute_count_kernel(const int32_t* __restrict__ topk_idx,
                                                            int T, int E, int k,
                                                            int32_t* __restrict__ chunk_counts,
                                                            int32_t* __restrict__ offsets,
                                                            unsigned* done, int* status,
                                                            int32_t* __restrict__ perm_token,
                                                            int32_t* __restrict__ inv_perm) {
  extern __shared__ uint32_t masks[];   // [kWarps][E] (+ [kWarps][E] row bases, one chunk)
  __shared__ int32_t warp_tot[kWarps];
  __shared__ bool is_last;
  const int nch = gridDim.x;
  build_masks(topk_idx, T, E, k, masks, status, true);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) c += __popc(masks[w * E + e]);
    chunk_counts[static_cast<size_t>(blockIdx.x) * E + e] = c;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1u) == static_cast<unsigned>(nch - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // Last CTA: totals per expert, exclusive scan over experts, then per-chunk bases.  Thread
  // i owns experts i, i + 256, ... (E <= 1024): each chunk row is read coalesced, 8 chunk
  // counts in flight at a time; the experts' blocks of 256 are scanned in order.
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int run = 0;                                   // groups of the expert blocks before this one
  for (int q = 0; q * 256 < E; ++q) {            // uniform over the CTA
    const int e = q * 256 + tid;
    int tot = 0;
    if (e < E) {
      for (int c0 = 0; c0 < nch; c0 += 8) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          v[u] = c0 + u < nch ? __ldcg(chunk_counts + static_cast<size_t>(c0 + u) * E + e) : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) tot += v[u];
      }
    }
    int incl = tot;                              // block exclusive scan of `tot`
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int warp_base = 0, block_tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      warp_base += w < warp ? warp_tot[w] : 0;
      block_tot += warp_tot[w];
    }
    if (e < E) {
      int base = run + warp_base + incl - tot;
      offsets[e] = base;
      for (int c0 = 0; c0 < nch; c0 += 8) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          v[u] = c0 + u < nch ? __ldcg(chunk_counts + static_cast<size_t>(c0 + u) * E + e) : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (c0 + u < nch) {
            chunk_counts[static_cast<size_t>(c0 + u) * E + e] = base;
            base += v[u];
          }
        }
      }
    }
    run += block_tot;
    __syncthreads();                             // warp_tot is reused by the next block
  }
  if (tid == 0) offsets[E] = run;
  if (tid == 0) *done = 0u;   // ready for the next call on this workspace
  if (nch == 1 && perm_token) {
    // one chunk (T <= 256): this CTA still holds the lane masks, so it ranks the pairs
    // itself instead of a second launch; chunk bases are the group offsets
    __syncthreads();
    int32_t* wbase = reinterpret_cast<int32_t*>(masks + kWarps * E);
    for (int e = tid; e < E; e += blockDim.x) {
      int r = __ldcg(offsets + e);
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        wbase[w * E + e] = r;
        r += __popc(masks[w * E + e]);
      }
    }
    __syncthreads();
    const int t = threadIdx.x;
    const uint32_t below = (1u << lane) - 1u;
    if (t < T) {
      for (int j = 0; j < k; ++j) {
        const int e = __ldg(topk_idx + static_cast<size_t>(t) * k + j);
        int row = -1;
        if (e >= 0 && e < E) {
          row = wbase[warp * E + e] + __popc(masks[warp * E + e] & below);
          perm_token[row] = t;
        }
        inv_perm[static_cast<size_t>(t) * k + j] = row;
      }
    }
  }
}

__global__ void __launch_bounds__(256) permute_rank_kernel(const int32_t* __restrict__ topk_idx,
                                                           int T, int E, int k,
                                                           const int32_t* __restrict__ chunk_base,
                                                           int32_t* __restrict__ perm_token,
                                                           int32_t* __restrict__ inv_perm) {
  extern __shared__ uint32_t smem[];
  uint32_t* masks = smem;                                         // [kWarps][E]
  int32_t* wbase = reinterpret_cast<int32_t*>(smem + kWarps * E); // [kWarps][E]
  build_masks(topk_idx, T, E, k, masks, nullptr, false);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = chunk_base[static_cast<size_t>(blockIdx.x) * E + e];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      wbase[w * E + e] = run;
      run += __popc(masks[w * E + e]);
    }
  }
  __syncthreads();
  const int t = blockIdx.x * kChunkTokens + threadIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t >= T) return;
  const uint32_t below = (1u << lane) - 1u;
  for (int j = 0; j < k; ++j) {
    const int e = __ldg(topk_idx + static_cast<size_t>(t) * k + j);
    int row = -1;
    if (e >= 0 && e < E) {
      row = wbase[warp * E + e] + __popc(masks[warp * E + e] & below);
      perm_token[row] = t;
    }
    inv_perm[static_cast<size_t>(t) * k + j] = row;
  }
}

// One warp per (token t, piece c of its row): the piece's 16-byte vectors (up to 8 per
// lane in flight) are read once and stored to the k rows inv_perm[t, 0..k-1]; entries
// outside [0, R) (dropped pairs) are skipped.  Streaming (evict-first) stores: x_perm is
// not read again by this kernel.  The piece-0 warp also copies the row's e4m3 scales.
constexpr int kPieceVecs = 256;   // 16-byte vectors per piece (4 KB)

__global__ void __launch_bounds__(256) scatter_rows_kernel(const uint4* __restrict__ x, int vec_per_row,
                                                           const float* __restrict__ x_scale,
                                                           int scale_cols, uint4* __restrict__ x_perm,
                                                           float* __restrict__ x_perm_scale,
                                                           const int32_t* __restrict__ inv_perm,
                                                           int T, int k, int R) {
  const int lane = threadIdx.x & 31;
  const int pieces = (vec_per_row + kPieceVecs - 1) / kPieceVecs;
  const long long items = static_cast<long long>(T) * pieces;
  const long long warps_total = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long it = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       it < items; it += warps_total) {
    const int t = static_cast<int>(it / pieces);
    const int c = static_cast<int>(it - static_cast<long long>(t) * pieces);
    int dst = -1;                                  // lane j < k: permuted row of slot j
    if (lane < k) {
      const int r = __ldg(inv_perm + static_cast<size_t>(t) * k + lane);
      dst = (r >= 0 && r < R) ? r : -1;
    }
    const int v0 = c * kPieceVecs;
    const uint4* src = x + static_cast<size_t>(t) * vec_per_row;
    uint4 buf[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vec_per_row) buf[u] = __ldg(src + v);
    }
    for (int j = 0; j < k; ++j) {
      const int r = __shfl_sync(0xffffffffu, dst, j);
      if (r < 0) continue;                         // warp-uniform
      uint4* o = x_perm + static_cast<size_t>(r) * vec_per_row;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vec_per_row) __stcs(o + v, buf[u]);
      }
    }
    if (x_scale && c == 0) {
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, dst, j);
        if (r < 0) continue;
        for (int q = lane; q < scale_cols; q += 32)
          x_perm_scale[static_cast<size_t>(r) * scale_cols + q] =
              __ldg(x_scale + static_cast<size_t>(t) * scale_cols + q);
      }
    }
  }
}

// The same copy for bf16 rows that feed e4m3 expert GEMMs, quantising on the way (the
// fused quantisation of the FP8 path): each 128-value block of a token's row gets the
// power-of-two scale 2^e with e the smallest exponent that brings the block's amax to 448
// or below, and every value x goes to e4m3(x / 2^e), round to nearest even, saturating.
// One warp per (token, piece of 2048 values = 16 blocks); in each step lanes 0-15 and
// 16-31 hold the 16 vectors of one block each, so a block's amax is a half-warp max.
// Outputs per destination row r: 8 bytes per lane-vector into x_perm (e4m3, d bytes per
// row) and the block scales -- fp32 values into scale_f32 [rows][d/128] (the ABI's scale
// format), or UE8M0 words (4 copies of e + 127) into scale_w [d/128][ld_w] (the layout the
// grouped GEMM's scale warp reads).  x_q / x_q_w (optional): the token's own quantised
// row and scale words (row t), the token operand of the shared experts.
__global__ void __launch_bounds__(256) scatter_quant_rows_kernel(
    const uint4* __restrict__ x, int vec_per_row, uint2* __restrict__ x_perm,
    float* __restrict__ scale_f32, uint32_t* __restrict__ scale_w, int ld_w,
    uint2* __restrict__ x_q, uint32_t* __restrict__ x_q_w, const int32_t* __restrict__ inv_perm,
    int T, int k, int R) {
  const int lane = threadIdx.x & 31;
  const int blocks_per_row = vec_per_row / 16;          // 128 bf16 values = 16 vectors
  const int pieces = (vec_per_row + kPieceVecs - 1) / kPieceVecs;
  const long long items = static_cast<long long>(T) * pieces;
  const long long warps_total = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const uint32_t half_mask = lane < 16 ? 0x0000FFFFu : 0xFFFF0000u;
  for (long long it = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       it < items; it += warps_total) {
    const int t = static_cast<int>(it / pieces);
    const int c = static_cast<int>(it - static_cast<long long>(t) * pieces);
    int dst = -1;
    if (lane < k) {
      const int r = __ldg(inv_perm + static_cast<size_t>(t) * k + lane);
      dst = (r >= 0 && r < R) ? r : -1;
    }
    const uint4* src = x + static_cast<size_t>(t) * vec_per_row;
    uint4 buf[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = c * kPieceVecs + u * 32 + lane;
      if (v < vec_per_row) buf[u] = __ldg(src + v);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = c * kPieceVecs + u * 32 + lane;
      if (c * kPieceVecs + u * 32 >= vec_per_row) break;   // warp-uniform
      // rows hold whole 16-vector blocks, so each half-warp is entirely valid or not
      const bool valid = v < vec_per_row;
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&buf[u]);
      float f[8];
      uint32_t amax = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 p2 = __bfloat1622float2(h[i]);
        f[2 * i] = p2.x;
        f[2 * i + 1] = p2.y;
        amax = max(amax, max(__float_as_uint(fabsf(p2.x)), __float_as_uint(fabsf(p2.y))));
      }
      amax = __reduce_max_sync(half_mask, amax);
      const int e = e4m3_scale_exponent(amax);
      uint2 q;
      uint16_t* qh = reinterpret_cast<uint16_t*>(&q);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        qh[i] = __nv_cvt_float2_to_fp8x2(make_float2(scalbnf(f[2 * i], -e), scalbnf(f[2 * i + 1], -e)),
                                         __NV_SATFINITE, __NV_E4M3);
      const int blk = v / 16;                             // 128-value block of the row
      const bool head = valid && (lane & 15) == 0;        // writes the block's scale
      for (int j = 0; j < k && x_perm; ++j) {
        const int r = __shfl_sync(0xffffffffu, dst, j);
        if (r < 0) continue;                               // warp-uniform
        if (valid) __stcs(x_perm + static_cast<size_t>(r) * vec_per_row + v, q);
        if (head) {
          if (scale_f32) scale_f32[static_cast<size_t>(r) * blocks_per_row + blk] = ldexpf(1.0f, e);
          else scale_w[static_cast<size_t>(blk) * ld_w + r] = 0x01010101u * static_cast<uint32_t>(e + 127);
        }
      }
      if (x_q && valid) {
        x_q[static_cast<size_t>(t) * vec_per_row + v] = q;
        if (head) x_q_w[static_cast<size_t>(blk) * T + t] = 0x01010101u * static_cast<uint32_t>(e + 127);
      }
    }
  }
}

}  // namespace

// count (+ rank) kernels of the permutation: group offsets, perm_token and inv_perm
cudaError_t launch_permute_index(const int32_t* topk_idx, int T, int E, int k, int32_t* perm_token,
                                 int32_t* inv_perm, int32_t* offsets, int32_t* chunk_counts,
                                 unsigned* done, int* status, cudaStream_t s) {
  const int nch = permute_chunks(T);
  const size_t smem_count = sizeof(uint32_t) * kWarps * E;
  const size_t smem_rank = 2 * smem_count;
  cudaError_t err;
  if (smem_count > 48 * 1024) {
    err = cudaFuncSetAttribute(permute_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_count));
    if (err != cudaSuccess) return err;
  }
  if (smem_rank > 48 * 1024) {
    err = cudaFuncSetAttribute(permute_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_rank));
    if (err != cudaSuccess) return err;
  }
  if (nch == 1) {
    // one chunk: the count kernel ranks too
    if (smem_rank > 48 * 1024) {
      err = cudaFuncSetAttribute(permute_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem_rank));
      if (err != cudaSuccess) return err;
    }
    permute_count_kernel<<<1, kChunkTokens, smem_rank, s>>>(topk_idx, T, E, k, chunk_counts,
                                                            offsets, done, status, perm_token,
                                                            inv_perm);
  } else {
    permute_count_kernel<<<nch, kChunkTokens, smem_count, s>>>(topk_idx, T, E, k, chunk_counts,
                                                               offsets, done, status, nullptr,
                                                               nullptr);
    permute_rank_kernel<<<nch, kChunkTokens, smem_rank, s>>>(topk_idx, T, E, k, chunk_counts,
                                                             perm_token, inv_perm);
  }
  return cudaGetLastError();
}

static unsigned copy_blocks(int T, int vec) {
  const long long items = static_cast<long long>(T) * ((vec + kPieceVecs - 1) / kPieceVecs);
  long long blocks = (items + 7) / 8;
  if (blocks > 148 * 8) blocks = 148 * 8;            // 8 resident CTAs of 256 threads per SM
  return static_cast<unsigned>(blocks);
}

cudaError_t launch_permute_quant(const int32_t* topk_idx, int T, int E, int k, const void* x_bf16,
                                 int d, void* x_perm, float* x_perm_scale, uint32_t* x_perm_w,
                                 void* x_q, uint32_t* x_q_w, int32_t* perm_token, int32_t* inv_perm,
                                 int32_t* offsets, int32_t* chunk_counts, unsigned* done,
                                 int* status, cudaStream_t s) {
  if (T == 0) return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
  cudaError_t err = launch_permute_index(topk_idx, T, E, k, perm_token, inv_perm, offsets,
                                         chunk_counts, done, status, s);
  if (err != cudaSuccess) return err;
  const int vec = d / 8;                                 // bf16 vectors per row
  scatter_quant_rows_kernel<<<copy_blocks(T, vec), 256, 0, s>>>(
      static_cast<const uint4*>(x_bf16), vec, static_cast<uint2*>(x_perm), x_perm_scale, x_perm_w,
      T * k, static_cast<uint2*>(x_q), x_q_w, inv_perm, T, k, T * k);
  return cudaGetLastError();
}

cudaError_t launch_permute(const int32_t* topk_idx, int T, int E, int k, const void* x,
                           int row_bytes, const float* x_scale, int scale_cols, void* x_perm,
                           float* x_perm_scale, int32_t* perm_token, int32_t* inv_perm,
                           int32_t* offsets, int32_t* chunk_counts, unsigned* done, int* status,
                           cudaStream_t s) {
  if (T == 0) {
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
  }
  cudaError_t err = launch_permute_index(topk_idx, T, E, k, perm_token, inv_perm, offsets,
                                         chunk_counts, done, status, s);
  if (err != cudaSuccess) return err;
  const int vec = row_bytes / 16;
  scatter_rows_kernel<<<copy_blocks(T, vec), 256, 0, s>>>(
      static_cast<const uint4*>(x), vec, x_scale, scale_cols, static_cast<uint4*>(x_perm),
      x_perm_scale, inv_perm, T, k, T * k);
  return cudaGetLastError();
}

}  // namespace moe
