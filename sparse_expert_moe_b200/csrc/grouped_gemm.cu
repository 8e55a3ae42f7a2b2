// grouped_gemm.cu -- the expert FFN GEMMs (and the router GEMM) on the 5th-
// generation tensor cores: TMA -> shared-memory ring -> tcgen05.mma -> TMEM ->
// epilogue registers -> global memory.
//
// Computes, per group g (one expert) and rows r of the group,
//   FFN1:  h[r] = silu(a[r] W1_g^T) * (a[r] W3_g^T)     (SwiGLU fused in the epilogue)
//   FFN2:  y[r] = h[r] W2_g^T
//   router: logits[t] = x[t] Wr^T  (fp32 out)
// -- the expert network `e(x)` of the moe_ffn pseudocode ("Decoding Trillion-
// Parameter MoE LLMs", section "Routing: Top-K Experts Plus a Shared Expert")
// with the SwiGLU and fused epilogue the GC-MoE radar item describes for
// Blackwell ("GC-MoE: Overlapping Expert-Parallel Token Dispatch with FP8/FP4
// Grouped GEMM via CUDA Green Contexts", key change on tcgen05 MMA with fused
// SwiGLU).
//
// Orientation ("swap AB"): the weight rows are the UMMA M side (128 rows per
// tile) and a group's tokens the N side (16..128 per tile, rounded up to 16).
// Decode groups hold a handful of tokens, so a 128-token M side would waste
// almost all of every MMA; with tokens on N the same kernel streams weights
// at N = 16 and reaches full 128x128 tiles on heavy prefill groups.  FFN1 keeps
// two accumulators per tile (gate rows and up rows of the same h columns), so
// SiLU(gate) * up happens in registers and h is written once.
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer (one lane)       -- fills a STAGES-deep smem ring
//   warp 1      TMEM owner + MMA issuer (one lane)
//   warps 2..5  epilogue: TMEM -> registers -> global (warp w reads TMEM lanes
//               32*(w%4)..+31, the sub-partition it may access)
// Two TMEM accumulator buffers let the epilogue of tile i overlap the MMAs of
// tile i+1.  Tiles are (chunk, 128-row weight block), weight block fastest, so
// CTAs running at the same time share a chunk's token rows through L2.
// Chunks come from the planner below, largest groups first.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;                  // weight rows per tile (UMMA M)
constexpr int kBK = 64;                   // K elements per stage (128 bytes of bf16)
constexpr int kNT = kChunkRows;           // token rows per tile (UMMA N max)
constexpr int kTokBox = 16;               // token rows per TMA box
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint32_t kBBytes = kNT * kBK * 2;
constexpr uint32_t kTokBoxBytes = kTokBox * kBK * 2;
constexpr int kThreads = 192;

struct DevParams {
  CUtensorMap wmap[2];
  CUtensorMap tmap[2];
  const Chunk* chunks;
  const int32_t* n_chunks;
  int router_T;
  int n_mblk;
  int k_blocks;
  int w_rows_per_group;
  int up_offset;
  int m_valid;
  void* out;
  int ld_out;
  int* status;
};

__device__ __forceinline__ Chunk get_chunk(const DevParams& p, int ci) {
  if (p.chunks) return p.chunks[ci];
  Chunk c;
  c.seg = 0;
  c.group = 0;
  c.b_row = ci * kNT;
  c.o_row = c.b_row;
  c.nrows = min(kNT, p.router_T - c.b_row);
  return c;
}

template <int MODE>
struct Cfg {
  static constexpr int kATiles = MODE == kFFN1 ? 2 : 1;
  static constexpr uint32_t kStageBytes = kATiles * kABytes + kBBytes;
  static constexpr int kStages = MODE == kFFN1 ? 4 : 6;
  static constexpr uint32_t kAccCols = MODE == kFFN1 ? 2 * kNT : kNT;   // per buffer
  static constexpr uint32_t kTmemCols = 2 * kAccCols;                  // 512 or 256
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 /*barriers*/ + 1024 /*align*/;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ DevParams p) {
  using C = Cfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty_bar = full_bar + C::kStages;
  uint64_t* tfull_bar = empty_bar + C::kStages;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.wmap[0]);
    tma_prefetch_desc(&p.tmap[0]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_chunks = p.chunks ? *p.n_chunks : (p.router_T + kNT - 1) / kNT;
  const int n_tiles = n_chunks * p.n_mblk;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const Chunk c = get_chunk(p, t / p.n_mblk);
        const int mb = t % p.n_mblk;
        const int a_row = c.group * p.w_rows_per_group + mb * kBM;
        const int nbox = (c.nrows + kTokBox - 1) / kTokBox;
        // FFN2 reads the h rows FFN1 wrote (output numbering); the others read b_row
        const int tok_row = MODE == kFFN2 ? c.o_row : c.b_row;
        const uint32_t bytes = C::kATiles * kABytes + nbox * kTokBoxBytes;
        const CUtensorMap* wm = &p.wmap[c.seg];
        const CUtensorMap* tm = &p.tmap[c.seg];
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* st = tiles + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          tma_load_2d(st, wm, &full_bar[stage], kb * kBK, a_row);
          if (MODE == kFFN1) tma_load_2d(st + kABytes, wm, &full_bar[stage], kb * kBK, a_row + p.up_offset);
          uint8_t* bt = st + C::kATiles * kABytes;
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(bt + i * kTokBoxBytes, tm, &full_bar[stage], kb * kBK, tok_row + i * kTokBox);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++it) {
        const Chunk c = get_chunk(p, t / p.n_mblk);
        const int n_pad = (c.nrows + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, n_pad);
        const uint32_t acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * C::kAccCols;
        const uint32_t d1 = d0 + kNT;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(tiles + stage * C::kStageBytes);
          const uint32_t bt = st + C::kATiles * kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t accum = (kb | kk) ? 1u : 0u;
            const uint64_t bdesc = umma_desc_sw128(bt + kk * 32);
            umma_bf16(d0, umma_desc_sw128(st + kk * 32), bdesc, idesc, accum);
            if (MODE == kFFN1) umma_bf16(d1, umma_desc_sw128(st + kABytes + kk * 32), bdesc, idesc, accum);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull_bar[acc]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;                 // TMEM lane quadrant of this warp
    const int m_local = sub * 32 + lane;      // weight row inside the tile
    int it = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
      const Chunk c = get_chunk(p, t / p.n_mblk);
      const int mb = t % p.n_mblk;
      const uint32_t acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      bool ok = mbar_wait(&tfull_bar[acc], acc_phase, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + acc * C::kAccCols;
      const int m = mb * kBM + m_local;       // output column
      for (int n0 = 0; n0 < c.nrows; n0 += 16) {
        if (MODE == kFFN1) {
          float g[16], u[16];
          tmem_ld16x2(tb + n0, tb + kNT + n0, g, u);
          __nv_bfloat16* h = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (n0 + i < c.nrows) {
              const float s = g[i] / (1.0f + __expf(-g[i]));
              h[static_cast<size_t>(c.o_row + n0 + i) * p.ld_out + m] = __float2bfloat16_rn(s * u[i]);
            }
          }
        } else if (MODE == kFFN2) {
          float v[16];
          tmem_ld16(tb + n0, v);
          __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n0 + i < c.nrows)
              y[static_cast<size_t>(c.o_row + n0 + i) * p.ld_out + m] = __float2bfloat16_rn(v[i]);
        } else {
          float v[16];
          tmem_ld16(tb + n0, v);
          float* lg = static_cast<float*>(p.out);
          if (m < p.m_valid) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n0 + i < c.nrows) lg[static_cast<size_t>(c.o_row + n0 + i) * p.ld_out + m] = v[i];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------- planner
// One CTA.  Validates the offsets, orders the groups by size (largest first,
// ties by index: routed before shared), splits each into chunks of at most
// kChunkRows rows and writes the chunk list and its length.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ offsets, int G,
                                                    int n_rows, int n_shared, int T,
                                                    int shared_o_row, Chunk* __restrict__ chunks,
                                                    int32_t* __restrict__ n_chunks, int* status) {
  __shared__ int32_t sz[kMaxGroups];
  __shared__ int32_t start[kMaxGroups];
  __shared__ int32_t order[kMaxGroups];
  __shared__ int32_t cbase[kMaxGroups + 1];
  __shared__ int bad;
  __shared__ int32_t warp_sum[32];
  const int NG = G + n_shared;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int g = tid; g < NG; g += blockDim.x) {
    int s, st;
    if (g < G) {
      const int lo = offsets[g], hi = offsets[g + 1];
      if (lo < 0 || hi < lo || hi > n_rows) bad = 1;
      s = hi - lo;
      st = lo;
    } else {
      s = T;
      st = 0;
    }
    sz[g] = s;
    start[g] = st;
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      record_status(status, kStatusDeviceIndex);
      *n_chunks = 0;
    }
    return;
  }
  for (int g = tid; g < NG; g += blockDim.x) {
    const int s = sz[g];
    int rank = 0;
    for (int j = 0; j < NG; ++j) {
      const int o = sz[j];
      rank += (o > s) || (o == s && j < g);
    }
    order[rank] = g;
  }
  __syncthreads();
  // exclusive scan of chunk counts in rank order; thread owns ranks 2*tid, 2*tid+1
  int c0 = 0, c1 = 0;
  const int r0 = 2 * tid, r1 = 2 * tid + 1;
  if (r0 < NG) c0 = (sz[order[r0]] + kChunkRows - 1) / kChunkRows;
  if (r1 < NG) c1 = (sz[order[r1]] + kChunkRows - 1) / kChunkRows;
  const int local = c0 + c1;
  const int lane = tid & 31, warp = tid >> 5;
  int incl = local;
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int wb = 0;
  for (int w = 0; w < warp; ++w) wb += warp_sum[w];
  const int excl = wb + incl - local;
  if (r0 < NG) cbase[r0] = excl;
  if (r1 < NG) cbase[r1] = excl + c0;
  if (tid == blockDim.x - 1) cbase[NG] = excl + local;
  __syncthreads();
  for (int r = tid; r < NG; r += blockDim.x) {
    const int g = order[r];
    const int s = sz[g];
    const bool shared = g >= G;
    int base = cbase[r];
    for (int c = 0; c * kChunkRows < s; ++c) {
      Chunk ch;
      ch.seg = shared ? 1 : 0;
      ch.group = shared ? g - G : g;
      ch.b_row = start[g] + c * kChunkRows;
      ch.o_row = shared ? shared_o_row + (g - G) * T + c * kChunkRows : ch.b_row;
      ch.nrows = min(kChunkRows, s - c * kChunkRows);
      ch.pad0 = ch.pad1 = ch.pad2 = 0;
      chunks[base + c] = ch;
    }
  }
  if (tid == 0) *n_chunks = cbase[NG];
}

}  // namespace

cudaError_t launch_plan(const int32_t* offsets, int G, int n_rows, int n_shared, int T,
                        int shared_o_row, Chunk* chunks, int32_t* n_chunks, int* status,
                        cudaStream_t s) {
  plan_kernel<<<1, 1024, 0, s>>>(offsets, G, n_rows, n_shared, T, shared_o_row, chunks, n_chunks,
                                 status);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t launch_mode(const GemmLaunch& g, cudaStream_t s) {
  using C = Cfg<MODE>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  DevParams p;
  p.wmap[0] = g.wmap[0];
  p.wmap[1] = g.wmap[1];
  p.tmap[0] = g.tmap[0];
  p.tmap[1] = g.tmap[1];
  p.chunks = g.chunks;
  p.n_chunks = g.n_chunks;
  p.router_T = g.router_T;
  p.n_mblk = g.n_mblk;
  p.k_blocks = g.k_blocks;
  p.w_rows_per_group = g.w_rows_per_group;
  p.up_offset = g.up_offset;
  p.m_valid = g.m_valid;
  p.out = g.out;
  p.ld_out = g.ld_out;
  p.status = g.status;
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::kSmemBytes));
  if (err != cudaSuccess) return err;
  int grid = g.num_sms;
  if (MODE == kRouter) {
    const int tiles = ((g.router_T + kNT - 1) / kNT) * g.n_mblk;
    if (tiles < grid) grid = tiles;
    if (grid == 0) return cudaSuccess;
  }
  grouped_gemm_kernel<MODE><<<grid, kThreads, C::kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t s) {
  switch (g.mode) {
    case kRouter: return launch_mode<kRouter>(g, s);
    case kFFN1: return launch_mode<kFFN1>(g, s);
    case kFFN2: return launch_mode<kFFN2>(g, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
