// convert.cu -- fp32 -> bf16 (round to nearest even) for the f32 input family,
// 16-byte loads and 8-byte stores, grid-stride.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"

namespace moe {
namespace {

__global__ void f32_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, size_t n4) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = src[i];
    uint2 r;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
    h[0] = __floats2bfloat162_rn(v.x, v.y);
    h[1] = __floats2bfloat162_rn(v.z, v.w);
    dst[i] = r;
  }
}

}  // namespace

// n must be a multiple of 4 (every converted tensor has a multiple-of-128 dimension).
cudaError_t launch_f32_to_bf16(const float* src, void* dst, size_t n, cudaStream_t s) {
  const size_t n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  size_t blocks = (n4 + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  f32_to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      reinterpret_cast<const float4*>(src), static_cast<uint2*>(dst), n4);
  return cudaGetLastError();
}

}  // namespace moe
