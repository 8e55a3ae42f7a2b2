// permute_noalloc.cu -- moe_permute for callers that cannot hand the library a
// workspace: the scratch the permutation needs (per-chunk expert counts and the
// ticket of the last-block scan) lives in a fixed-size array in the library's
// own device memory instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it (kScratchInts * 4 bytes, about 1 MiB) until the process
// exits.  Host code may not use the variable's name as a device address; the
// device address is looked up once per device with cudaGetSymbolAddress.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {
namespace {

constexpr int kHeaderInts = 64;                    // [1] = scan ticket; rest reserved
constexpr int kMaxCountInts = 256 * 1024;          // ceil(T/256) * E <= 262144
constexpr int kScratchInts = kHeaderInts + kMaxCountInts;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

std::mutex g_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_permute_scratch on the current device (looked up on the
// first call made with that device current).  nullptr on failure.
int32_t* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                                          const void* x, const float* x_scale, void* x_perm,
                                          float* x_perm_scale, int32_t* perm_token,
                                          int32_t* inv_perm, int32_t* group_offsets,
                                          cudaStream_t stream) {
  using namespace moe;
  moe_status st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (!group_offsets) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_idx || !x || !x_perm || !perm_token || !inv_perm))
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_perm) & 15u))
    return MOE_ERR_INVALID_ARG;
  // bf16 rows for e4m3 / FP4 experts are quantised by moe_permute; not on this path
  if (cfg->act == MOE_BF16 && (cfg->weight == MOE_E4M3 || cfg->weight == MOE_E2M1))
    return MOE_ERR_UNSUPPORTED;
  // e4m3 rows come with one fp32 scale per 128 channels, permuted alongside the rows
  const bool fp8 = cfg->act == MOE_E4M3 || cfg->act == MOE_E4M3_FP32_SCALE;
  if (fp8 && cfg->T > 0 && (!x_scale || !x_perm_scale)) return MOE_ERR_INVALID_ARG;
  const int64_t counts = static_cast<int64_t>(permute_chunks(cfg->T)) * cfg->E;
  if (counts > kMaxCountInts) return MOE_ERR_UNSUPPORTED;   // beyond the fixed scratch
  int32_t* scratch = scratch_on_current_device();
  if (!scratch) return MOE_ERR_CUDA;
  // the scan ticket must start at zero; the array keeps whatever the last call left
  if (cudaMemsetAsync(scratch, 0, kHeaderInts * sizeof(int32_t), stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  // bytes per element of a row: f32 4, bf16 2, e4m3 1
  const int elem = cfg->act == MOE_F32 ? 4 : (fp8 ? 1 : 2);
  const cudaError_t e = launch_permute(topk_idx, cfg->T, cfg->E, cfg->top_k, x, cfg->d_model * elem,
                                       fp8 ? x_scale : nullptr, fp8 ? cfg->d_model / 128 : 0,
                                       x_perm, fp8 ? x_perm_scale : nullptr, perm_token, inv_perm,
                                       group_offsets, scratch + kHeaderInts,
                                       reinterpret_cast<unsigned*>(scratch + 1), nullptr, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
