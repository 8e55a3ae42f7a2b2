// combine.cu -- weighted un-permute: the `out += weights[..., k] * e(x)` and
// `out += s(x)` steps of the moe_ffn pseudocode ("Decoding Trillion-Parameter
// MoE LLMs", section "Routing: Top-K Experts Plus a Shared Expert").
//
//   out[t] = sum_j w[t, j] * y_perm[inv_perm[t, j]] + sum_s y_shared_s[t]
//
// One CTA per (token, 1024-column slice); each thread owns 8 consecutive columns
// (one 16-byte bf16 vector) and accumulates the k gathered rows in slot order in
// fp32 registers, then the shared rows, then rounds once.  No atomics: every
// output element has exactly one writer, so repeated runs are bit-identical.
// HBM-bound: reads (k + S) rows and writes one row per token.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& v, float w) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
  }
}

__device__ __forceinline__ void add_bf16x8_plain(float (&acc)[8], const uint4& v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

template <int KMAX>
__global__ void __launch_bounds__(128) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const float* __restrict__ topk_w,
                                                      const uint4* __restrict__ y_shared,
                                                      int n_shared, int T, int d, int k, int R,
                                                      bool out_f32, void* __restrict__ out) {
  const int t = blockIdx.x;
  const int vec = d / 8;
  const int v = blockIdx.y * blockDim.x + threadIdx.x;
  __shared__ int32_t rows[KMAX];
  __shared__ float ws[KMAX];
  if (threadIdx.x < k) {
    const int r = inv_perm[static_cast<size_t>(t) * k + threadIdx.x];
    rows[threadIdx.x] = (r >= 0 && r < R) ? r : -1;
    ws[threadIdx.x] = topk_w[static_cast<size_t>(t) * k + threadIdx.x];
  }
  __syncthreads();
  if (v < vec) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    uint4 buf[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k && rows[j] >= 0) buf[j] = __ldg(y_perm + static_cast<size_t>(rows[j]) * vec + v);
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k && rows[j] >= 0) add_bf16x8(acc, buf[j], ws[j]);
    for (int s = 0; s < n_shared; ++s)
      add_bf16x8_plain(acc, __ldg(y_shared + (static_cast<size_t>(s) * T + t) * vec + v));
    if (out_f32) {
      float4* o = static_cast<float4*>(out) + (static_cast<size_t>(t) * vec + v) * 2;
      o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint4 r;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      static_cast<uint4*>(out)[static_cast<size_t>(t) * vec + v] = r;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const void* y_perm, const int32_t* inv_perm, const float* topk_w,
                           const void* y_shared, int n_shared, int T, int d, int k, int R,
                           bool out_f32, void* y, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const uint4* yp = static_cast<const uint4*>(y_perm);
  const uint4* ys = static_cast<const uint4*>(y_shared);
  if (!y_shared) n_shared = 0;
  const dim3 grid(T, (d / 8 + 127) / 128);
  if (k <= 8)
    combine_kernel<8><<<grid, 128, 0, s>>>(yp, inv_perm, topk_w, ys, n_shared, T, d, k, R, out_f32, y);
  else
    combine_kernel<16><<<grid, 128, 0, s>>>(yp, inv_perm, topk_w, ys, n_shared, T, d, k, R, out_f32, y);
  return cudaGetLastError();
}

}  // namespace moe
