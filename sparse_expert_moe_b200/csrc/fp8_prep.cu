// fp8_prep.cu -- scale-factor and activation preparation for the FP8 block-scaled
// path ("GC-MoE: Overlapping Expert-Parallel Token Dispatch with FP8/FP4 Grouped GEMM
// via CUDA Green Contexts", key change on tcgen05 block-scaled MMA).
//
// The ABI takes fp32 power-of-two block scales; the tensor cores take UE8M0 scale
// factors (the fp32 exponent byte).  These kernels re-encode them in the layouts the
// grouped GEMM's scale warp copies from, and dequantise the e4m3 activations to bf16
// for the router GEMM (exact: 3 mantissa bits times a power of two fit in bf16).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

// UE8M0 code of a power-of-two fp32 scale, replicated into the 4 bytes of a word.  A scale
// that UE8M0 cannot hold exactly -- sign set, zero or subnormal, infinite or NaN, or any
// mantissa bit set -- records MOE_ERR_DEVICE_VALUE in the status word.
__device__ __forceinline__ uint32_t ue8m0x4(float s, int* status) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t e = (b >> 23) & 0xFFu;
  if ((b & 0x807FFFFFu) != 0u || e == 0u || e == 0xFFu) record_status(status, kStatusDeviceValue);
  return 0x01010101u * e;
}

// One thread per 16 activation bytes (16 e4m3 values, one 1x128 scale block).  x_lo
// (optional): v - bf16(v) rounded to bf16, so that x_bf16 + x_lo carries v = code x scale to
// ~2^-17 relative when the scale is not a power of two (x_bf16 alone is then rounded).
__global__ void act_prep_fp8_kernel(const uint4* __restrict__ x, const float* __restrict__ x_scale,
                                    int T, int d, uint4* __restrict__ x_bf16,
                                    uint4* __restrict__ x_lo, uint32_t* __restrict__ x_sf,
                                    int* status) {
  const int vec_per_row = d / 16;
  const size_t n = static_cast<size_t>(T) * vec_per_row;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / vec_per_row);
    const int v = static_cast<int>(i % vec_per_row);
    const int kb = v / 8;                         // 8 vectors of 16 bytes per 128 block
    const float s = x_scale[static_cast<size_t>(t) * (d / 128) + kb];
    if (x_bf16) {
      const uint4 q = x[i];
      const __nv_fp8x2_storage_t* p = reinterpret_cast<const __nv_fp8x2_storage_t*>(&q);
      uint4 o[2], lo[2];
      __nv_bfloat162* ob = reinterpret_cast<__nv_bfloat162*>(o);
      __nv_bfloat162* ol = reinterpret_cast<__nv_bfloat162*>(lo);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(p[j], __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        const float2 v = make_float2(f.x * s, f.y * s);
        ob[j] = __floats2bfloat162_rn(v.x, v.y);
        const float2 h = __bfloat1622float2(ob[j]);
        ol[j] = __floats2bfloat162_rn(v.x - h.x, v.y - h.y);
      }
      x_bf16[2 * i] = o[0];
      x_bf16[2 * i + 1] = o[1];
      if (x_lo) {
        x_lo[2 * i] = lo[0];
        x_lo[2 * i + 1] = lo[1];
      }
    }
    if (x_sf && (v % 8) == 0) x_sf[static_cast<size_t>(kb) * T + t] = ue8m0x4(s, status);
  }
}

__global__ void weight_sf_kernel(const float* __restrict__ s, size_t n, uint4* __restrict__ out,
                                 int* status) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint32_t w = ue8m0x4(s[i], status);
    out[i] = make_uint4(w, w, w, w);
  }
}

__global__ void gather_sf_kernel(const uint32_t* __restrict__ x_sf, int T, int kbs,
                                 const int32_t* __restrict__ perm_token,
                                 const int32_t* __restrict__ total_ptr, int R,
                                 uint32_t* __restrict__ x_perm_sf) {
  const int total = *total_ptr;
  const size_t n = static_cast<size_t>(kbs) * total;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int kb = static_cast<int>(i / total);
    const int r = static_cast<int>(i % total);
    x_perm_sf[static_cast<size_t>(kb) * R + r] = x_sf[static_cast<size_t>(kb) * T + perm_token[r]];
  }
}

unsigned grid_for(size_t n, int threads) {
  size_t b = (n + threads - 1) / threads;
  if (b > 148 * 16) b = 148 * 16;
  return static_cast<unsigned>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_act_prep_fp8(const uint8_t* x, const float* x_scale, int T, int d, void* x_bf16,
                                uint32_t* x_sf, int* status, cudaStream_t s, void* x_lo) {
  if (T == 0) return cudaSuccess;
  const size_t n = static_cast<size_t>(T) * (d / 16);
  act_prep_fp8_kernel<<<grid_for(n, 256), 256, 0, s>>>(reinterpret_cast<const uint4*>(x), x_scale, T,
                                                       d, static_cast<uint4*>(x_bf16),
                                                       static_cast<uint4*>(x_lo), x_sf, status);
  return cudaGetLastError();
}

cudaError_t launch_weight_sf(const float* scales, size_t n, uint4* out, int* status, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  weight_sf_kernel<<<grid_for(n, 256), 256, 0, s>>>(scales, n, out, status);
  return cudaGetLastError();
}

cudaError_t launch_gather_sf(const uint32_t* x_sf, int T, int kbs, const int32_t* perm_token,
                             const int32_t* total, int R, uint32_t* x_perm_sf, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  gather_sf_kernel<<<grid_for(static_cast<size_t>(kbs) * R, 256), 256, 0, s>>>(
      x_sf, T, kbs, perm_token, total, R, x_perm_sf);
  return cudaGetLastError();
}

}  // namespace moe
