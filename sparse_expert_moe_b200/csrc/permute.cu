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
//  3. gather: x_perm[r] = x[perm_token[r]], one warp per row, 16-byte vectors.
#include <cuda_runtime.h>

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

  // Last CTA: totals per expert, exclusive scan over experts, then per-chunk bases.
  // Thread i owns experts 4i..4i+3 (E <= 1024).
  const int tid = threadIdx.x;
  int tot[4];
  int local = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = tid * 4 + q;
    int s = 0;
    if (e < E)
      for (int c = 0; c < nch; ++c) s += __ldcg(chunk_counts + static_cast<size_t>(c) * E + e);
    tot[q] = s;
    local += s;
  }
  // block exclusive scan of `local`
  const int lane = tid & 31, warp = tid >> 5;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int warp_base = 0;
  for (int w = 0; w < warp; ++w) warp_base += warp_tot[w];
  int run = warp_base + incl - local;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = tid * 4 + q;
    if (e < E) {
      offsets[e] = run;
      int base = run;
      for (int c = 0; c < nch; ++c) {
        int32_t* p = chunk_counts + static_cast<size_t>(c) * E + e;
        const int cnt = __ldcg(p);
        *p = base;
        base += cnt;
      }
      run += tot[q];
    }
  }
  if (tid == blockDim.x - 1) offsets[E] = run;
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

// One warp per permuted row; rows past offsets[E] (dropped pairs) are skipped.  x is
// read k times (from L2 when it stays there) and x_perm is written once and not read
// again by this kernel, so the stores are streaming (evict-first): the T k rows passing
// through L2 on their way to HBM would otherwise push x out and turn its re-reads into
// DRAM reads.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x, int vec_per_row,
                                                          const float* __restrict__ x_scale,
                                                          int scale_cols, uint4* __restrict__ x_perm,
                                                          float* __restrict__ x_perm_scale,
                                                          const int32_t* __restrict__ perm_token,
                                                          const int32_t* __restrict__ total_ptr) {
  const int total = *total_ptr;
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < total; r += warps_total) {
    const int t = __ldg(perm_token + r);
    const uint4* src = x + static_cast<size_t>(t) * vec_per_row;
    uint4* dst = x_perm + static_cast<size_t>(r) * vec_per_row;
    int v = lane;
    for (; v + 96 < vec_per_row; v += 128) {
      const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64),
                  d = __ldg(src + v + 96);
      __stcs(dst + v, a);
      __stcs(dst + v + 32, b);
      __stcs(dst + v + 64, c);
      __stcs(dst + v + 96, d);
    }
    for (; v < vec_per_row; v += 32) __stcs(dst + v, __ldg(src + v));
    if (x_scale)
      for (int c = lane; c < scale_cols; c += 32)
        x_perm_scale[static_cast<size_t>(r) * scale_cols + c] =
            __ldg(x_scale + static_cast<size_t>(t) * scale_cols + c);
  }
}

}  // namespace

cudaError_t launch_permute(const int32_t* topk_idx, int T, int E, int k, const void* x,
                           int row_bytes, const float* x_scale, int scale_cols, void* x_perm,
                           float* x_perm_scale, int32_t* perm_token, int32_t* inv_perm,
                           int32_t* offsets, int32_t* chunk_counts, unsigned* done, int* status,
                           cudaStream_t s) {
  if (T == 0) {
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
  }
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
  const int rows = T * k;
  int blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  gather_rows_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(x), row_bytes / 16, x_scale,
                                            scale_cols, static_cast<uint4*>(x_perm), x_perm_scale,
                                            perm_token, offsets + E);
  return cudaGetLastError();
}

}  // namespace moe
