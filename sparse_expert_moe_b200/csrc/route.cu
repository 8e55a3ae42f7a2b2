// route.cu -- router top-k and gate weights, one warp per token.
//
// Follows the "topk_softmax" step of the moe_ffn pseudocode ("Decoding
// Trillion-Parameter MoE LLMs", section "Routing: Top-K Experts Plus a Shared
// Expert") and the sigmoid + selection-bias variant named "auxiliary-loss-free
// bias routing" ("Chapter 7: Serving Mega MoE at scale").
//
// Each lane holds experts lane, lane+32, ... of the token's logit row (coalesced
// 128-byte loads); when the router GEMM split K across CTAs, a CTA per token first
// sums the partial logits in a fixed order, so repeated runs are bit-identical.  k rounds
// of a warp-wide arg-max (shuffle butterfly; key descending, equal keys to the
// lower expert index) pick the slots in order; lane j keeps slot j and computes
// its gate with one more butterfly.  HBM-bound: the kernel reads
// n_partials * T * E * 4 bytes and writes T * k * 8.
#include <cfloat>
#include <climits>
#include <cuda_runtime.h>

#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

__device__ __forceinline__ bool better(float ka, int ea, float kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}

// Top-k of one token's logits, held by one warp (lane: experts lane, lane + 32, ...), and
// the gates of the selected experts; lanes 0..k-1 write slot `lane`.
template <int VPL>
__device__ __forceinline__ void select_and_gate(const float (&lg)[VPL], int lane, int E, int k,
                                                int score, const float* __restrict__ sel_bias,
                                                int token, int32_t* __restrict__ topk_idx,
                                                float* __restrict__ topk_w) {
  float key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    float kk = -FLT_MAX;
    if (e < E) kk = score == 0 ? lg[i] : sigmoidf_(lg[i]) + (sel_bias ? __ldg(sel_bias + e) : 0.f);
    key[i] = kk;
  }

  uint32_t taken = 0;
  int my_idx = 0;
  float my_logit = 0.f;
  for (int j = 0; j < k; ++j) {
    float bk = -FLT_MAX;
    int be = INT_MAX;
    float bl = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = i * 32 + lane;
      if (e < E && !((taken >> i) & 1u) && better(key[i], e, bk, be)) {
        bk = key[i];
        be = e;
        bl = lg[i];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      const float ol = __shfl_xor_sync(0xffffffffu, bl, off);
      if (better(ok, oe, bk, be)) {
        bk = ok;
        be = oe;
        bl = ol;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) {
      my_idx = be;
      my_logit = bl;
    }
  }

  // gates of the selected experts (lanes 0..k-1), fixed-order butterflies
  float v;
  if (score == 0) {
    float m = lane < k ? my_logit : -FLT_MAX;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    v = lane < k ? expf(my_logit - m) : 0.f;
  } else {
    v = lane < k ? sigmoidf_(my_logit) : 0.f;
  }
  float sum = v;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    topk_idx[static_cast<size_t>(token) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(token) * k + lane] = v / sum;
  }
}

// One warp per token on complete logits (n_partials == 1).
template <int VPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ sel_bias, int T, int E,
                                                    int k, int score, int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_w) {
  const int token = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (token >= T) return;
  const float* row = logits + static_cast<size_t>(token) * E;
  float lg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    lg[i] = e < E ? __ldg(row + e) : 0.f;
  }
  select_and_gate<VPL>(lg, lane, E, k, score, sel_bias, token, topk_idx, topk_w);
}

// One CTA per token on the partial logits of a split-K router: thread t sums the partials
// of experts t, t + 256, ... in the fixed order p0 + p1 + p2 + ... (all of a thread's loads
// in flight together: one round of latency instead of one per few partials), the sums go
// through shared memory, and warp 0 selects.
template <int VPL>
__global__ void __launch_bounds__(256) route_partials_kernel(const float* __restrict__ logits,
                                                             int n_partials, long long partial_stride,
                                                             const float* __restrict__ sel_bias,
                                                             int T, int E, int k, int score,
                                                             int32_t* __restrict__ topk_idx,
                                                             float* __restrict__ topk_w) {
  constexpr int kMaxPartials = 32;
  __shared__ float sums[32 * VPL];
  const int token = blockIdx.x;
  const float* row = logits + static_cast<size_t>(token) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float v[kMaxPartials];
#pragma unroll
    for (int q = 0; q < kMaxPartials; ++q)
      v[q] = q < n_partials ? __ldg(row + q * partial_stride + e) : 0.f;
    float l = v[0];
#pragma unroll
    for (int q = 1; q < kMaxPartials; ++q)
      if (q < n_partials) l += v[q];
    sums[e] = l;
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  float lg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = i * 32 + lane;
    lg[i] = e < E ? sums[e] : 0.f;
  }
  select_and_gate<VPL>(lg, lane, E, k, score, sel_bias, token, topk_idx, topk_w);
}

template <int VPL>
cudaError_t launch_route_vpl(const float* logits, int n_partials, long long partial_stride,
                             const float* sel_bias, int T, int E, int k, int score,
                             int32_t* topk_idx, float* topk_w, cudaStream_t s) {
  if (n_partials > 1) {
    route_partials_kernel<VPL><<<T, 256, 0, s>>>(logits, n_partials, partial_stride, sel_bias, T,
                                                 E, k, score, topk_idx, topk_w);
  } else {
    // small batches: 2 warps per block so that the tokens spread over many SMs
    const int threads = T >= 2048 ? 256 : 64;
    const int blocks = (T + threads / 32 - 1) / (threads / 32);
    route_kernel<VPL><<<blocks, threads, 0, s>>>(logits, sel_bias, T, E, k, score, topk_idx, topk_w);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const float* logits, int n_partials, long long partial_stride,
                         const float* sel_bias, int T, int E, int k, int score, int32_t* topk_idx,
                         float* topk_w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (n_partials < 1 || n_partials > 32) return cudaErrorInvalidValue;
  if (E <= 32) return launch_route_vpl<1>(logits, n_partials, partial_stride, sel_bias, T, E, k, score, topk_idx, topk_w, s);
  if (E <= 64) return launch_route_vpl<2>(logits, n_partials, partial_stride, sel_bias, T, E, k, score, topk_idx, topk_w, s);
  if (E <= 128) return launch_route_vpl<4>(logits, n_partials, partial_stride, sel_bias, T, E, k, score, topk_idx, topk_w, s);
  if (E <= 256) return launch_route_vpl<8>(logits, n_partials, partial_stride, sel_bias, T, E, k, score, topk_idx, topk_w, s);
  if (E <= 512) return launch_route_vpl<16>(logits, n_partials, partial_stride, sel_bias, T, E, k, score, topk_idx, topk_w, s);
  return launch_route_vpl<32>(logits, n_partials, partial_stride, sel_bias, T, E, k, score, topk_idx, topk_w, s);
}

}  // namespace moe
