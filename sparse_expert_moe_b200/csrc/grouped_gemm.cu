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
// SiLU(gate) * up happens in registers and h is written once.  FFN2 likewise
// stages two 128-row weight blocks per K block (256 output columns, two
// accumulators): every stage then carries 32 KB of weights, as in FFN1, which the
// weight stream needs to reach the HBM roofline (one 16 KB block per stage left
// FFN2 at 77-91% of it).
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer (one lane)       -- fills a STAGES-deep smem ring
//   warp 1      TMEM owner + MMA issuer (one lane)
//   warps 2..5  epilogue: TMEM -> registers -> global (warp w reads TMEM lanes
//               32*(w%4)..+31, the sub-partition it may access)
// Two TMEM accumulator buffers let the epilogue of tile i overlap the MMAs of
// tile i+1.  Tiles are (token chunk, weight block) laid out group by group (see
// tile_coord); chunks come from the planner below, largest groups first.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;                  // weight rows per tile (UMMA M)
constexpr int kRowBytes = 128;            // K bytes per stage and row: one 128-byte swizzle row
constexpr uint32_t kABytes = kBM * kRowBytes;
constexpr uint32_t kSFAtomBytes = 512;    // 128 rows x 4 UE8M0 bytes (tcgen05.cp 32x128b source)

constexpr int kTokBoxes = 4;              // token boxes of 128, 64, 32, 16 rows
constexpr uint32_t kMaxSmem = 227 * 1024;  // opt-in dynamic shared memory per CTA
constexpr int kRingSlots = 16;            // stage barriers of a byte ring

struct DevParams {
  CUtensorMap wmap[2];        // weight maps per segment (boxes of 128 rows)
  CUtensorMap tmap[2][kTokBoxes];
  const Chunk* chunks;
  const int32_t* n_chunks;
  const int32_t* grp_cp;      // chunk prefix of the planned groups (largest first) [n_grp + 1],
                              // then their half-chunk prefix [n_grp + 1]
  const int32_t* n_grp;
  int halves;                 // chunks hold 2 x kNT rows: each tile takes one non-empty half
  int router_T;
  int n_mblk;
  int k_blocks;
  int k_splits;               // router: K split across CTAs (partial outputs, summed later)
  int k_per_split;            // k blocks per split
  long long split_stride;     // elements between the partial outputs of consecutive splits
  int w_rows_per_group;
  int up_offset;
  int m_valid;
  void* out;
  int ld_out;
  int* status;
  // FP8 block scaling
  const uint4* wsf[2];        // [groups][row blocks][k blocks] UE8M0 x16 per 128x128 weight block
  const uint4* wsc[2];        // FP4 weights: E8M0 codes in 512-byte scale atoms
                              // [groups][row blocks][k blocks][32 x uint4]
  int wsf_rb_per_group;       // 128-row blocks of the weight matrix per group
  const uint32_t* tsf[2];     // [k blocks][rows] UE8M0 x4 per (128-element block, token row)
  int tsf_ld[2];
  int tsf_rows[2];
  uint32_t* out_sf;           // FFN1 (FP8): [I / 128][rows] scales of the requantised h
  int ld_out_sf;
  // gather-on-load (first GEMM): token row n of a chunk is row gidx[b_row + n] of gsrc
  // (gidx null: row b_row + n), g_ld bytes apart
  const uint8_t* gsrc[2];
  const int32_t* gidx[2];
  int g_ld;
  // fp32-scale modes (kFFN1X / kFFN2X / kFFN2XM256): token scales fp32 [rows][fs_a_ld] per
  // segment (kFFN1X; the second GEMM reads h's UE8M0 words through tsf), weight scales fp32
  // [groups][row blocks][k blocks] per segment
  const float* fs_a[2];
  int fs_a_ld;
  const float* fs_w[2];
};

// NTW: token-tile width of the bf16 expert GEMMs.  128 by default -- half of a 256-row
// chunk once groups can exceed 128 rows (a 256-wide tile with two accumulators, gate
// and up or two output blocks, would need all 512 TMEM columns for one buffer, and its
// epilogue could no longer hide behind the next tile's MMAs); 32 for decode-sized
// batches (small token tiles leave shared memory to a deeper weight ring); 256 only for
// the single-block FFN2 used when d_model is not a multiple of 256.
// GATHER (first GEMM on wide token tiles, e4m3 token rows): the token tile of every stage
// is copied from the unpermuted activations by four gather warps (16-byte cp.async into
// the 128-byte swizzled layout) instead of TMA from a permuted copy; stages are then of
// fixed size.
template <int MODE, int NTW = kChunkRows, bool GATHER = false>
struct Cfg {
  // FP4 weights (MXFP4: E2M1, one E8M0 scale per 32 K-elements) with e4m3 tokens: the FP8
  // kernel with the weight operand unpacked by TMA into the e4m3 layout
  static constexpr bool kW4 = MODE == kFFN1F4 || MODE == kFFN2F4 || MODE == kFFN2F4M256;
  static constexpr bool kFP8 = MODE == kFFN1F8 || MODE == kFFN2F8 || MODE == kFFN2F8M256 || kW4;
  static constexpr bool kGLU = MODE == kFFN1 || MODE == kFFN1F8 || MODE == kFFN1F4;  // gate + up
  static constexpr bool kSecond = MODE == kFFN2 || MODE == kFFN2M256 || MODE == kFFN2M512 ||
                                  MODE == kFFN2F8 || MODE == kFFN2F4 || MODE == kFFN2F8M256 ||
                                  MODE == kFFN2F4M256;   // reads h (output rows)
  // FFN2: 128-row weight blocks (= 128 output columns each) per tile
  static constexpr int kOutBlocks =
      MODE == kFFN2M512 ? 4
                        : ((MODE == kFFN2M256 || MODE == kFFN2F8M256 || MODE == kFFN2F4M256) ? 2 : 1);
  static_assert(NTW == kChunkRows || MODE != kRouter, "router tiles are 128 tokens wide");
  static constexpr int kATiles = kGLU ? 2 : kOutBlocks;             // weight tiles per stage
  // FP8 tiles: 112 tokens (112 / 224 are passed in as NTW), leaving TMEM room for the
  // per-stage scale factors
  static constexpr int kNT = (kFP8 && NTW == kChunkRows) ? kChunkRowsFP8 : NTW;
  static constexpr int kSFBAtoms = (kNT + 127) / 128;               // 128 token rows per atom
  static constexpr int kAccBufs = (kGLU && kNT > 128) ? 1 : 2;
  static constexpr uint32_t kBBytes = kNT * kRowBytes;
  static constexpr uint32_t kSFBytes = kFP8 ? (kATiles + kSFBAtoms) * kSFAtomBytes : 0;
  static constexpr uint32_t kStageBytes =
      ((kATiles * kABytes + kBBytes + kSFBytes + 1023) / 1024) * 1024;
  static constexpr int kStagesFit = static_cast<int>((192u * 1024u) / kStageBytes);
  static constexpr int kStages = kStagesFit > 10 ? 10 : kStagesFit;
  static constexpr uint32_t kAccCols = kATiles * kNT;               // per accumulator buffer
  static constexpr uint32_t kSFColsPerStage = 16;                     // <= 4 atoms x 4 columns
  static_assert(!kFP8 || (kATiles + kSFBAtoms) * 4 <= 16, "scale atoms per stage");
  static constexpr uint32_t kSFCols = kFP8 ? kStages * kSFColsPerStage : 0;
  static constexpr uint32_t kColsUsed = kAccBufs * kAccCols + kSFCols;
  static constexpr uint32_t kTmemCols =
      kColsUsed <= 64 ? 64 : (kColsUsed <= 128 ? 128 : (kColsUsed <= 256 ? 256 : 512));
  static constexpr int kGatherWarp0 = kFP8 ? 7 : 6;                 // first gather warp
  static constexpr int kGatherThreads = 128;
  // + one scale-factor warp (FP8), + four gather warps (GATHER)
  static constexpr int kThreads = (kFP8 ? 224 : 192) + (GATHER ? kGatherThreads : 0);
  static constexpr bool kFixedStages = kFP8 || GATHER;
  static constexpr uint32_t kStagingBytes = 4 * 16 * 32 * 4;      // per epilogue warp: 16 x 32 x 4 B
  static constexpr uint32_t kGrpBytes = 2 * (kMaxGroups + 1) * 4;   // group (half-)chunk prefixes
  static constexpr uint32_t kRedBytes = kFP8 ? 2 * 4 * 128 * 4 : 0;  // FP8 amax exchange
  // Stage ring: FP8 keeps fixed stages (the scale warp and the per-stage TMEM scale
  // columns are indexed by stage); bf16 stages take their actual size out of a byte ring
  // filling the rest of shared memory.
  static constexpr uint32_t kFixedBytes = 1024 /*barriers*/ + kStagingBytes + kGrpBytes + 16 +
                                          kRedBytes + 1024 /*align*/;
  static constexpr int kSlots = kFixedStages ? kStages : kRingSlots;
  static constexpr uint32_t kRingBytes =
      kFixedStages ? kStages * kStageBytes : ((kMaxSmem - kFixedBytes) / 1024) * 1024;
  static constexpr uint32_t kSmemBytes = kRingBytes + kFixedBytes;
  static_assert(kSmemBytes <= kMaxSmem, "shared memory budget");
  static_assert(kColsUsed <= 512, "TMEM budget");
};

template <int MODE>
__device__ __forceinline__ Chunk get_chunk(const DevParams& p, int ci) {
  if (p.chunks) return p.chunks[ci];
  Chunk c;                                   // router: fixed chunks of kChunkRows tokens
  c.seg = 0;
  c.group = 0;
  c.b_row = ci * kChunkRows;
  c.o_row = c.b_row;
  c.nrows = min(kChunkRows, p.router_T - c.b_row);
  return c;
}

// Tile t -> (chunk, weight block, K split).
// Router (no chunk list): splits fastest, then weight blocks, then token chunks.
// Grouped GEMMs: tiles are laid out group by group (largest group first); inside a
// group of c chunks and n_mblk weight blocks, blocks of G weight blocks (G = 4 when
// it divides n_mblk) sweep all c chunks before the next G: CTAs running at the same
// time share a few weight blocks and many token chunks, both resident in L2, so an
// expert's weights and tokens come from HBM about once.

struct TileCoord {
  int chunk, mb, split, kb0, kb1, half;
};
__device__ __forceinline__ TileCoord tile_coord(const DevParams& p, int t, const int32_t* cp,
                                                int n_grp) {
  // cp: chunk prefix [n_grp + 1] followed by the half-chunk prefix [n_grp + 1]
  TileCoord tc;
  tc.half = 0;
  if (!p.chunks) {
    tc.split = t % p.k_splits;
    const int r = t / p.k_splits;
    tc.chunk = r / p.n_mblk;
    tc.mb = r % p.n_mblk;
    tc.kb0 = tc.split * p.k_per_split;
    tc.kb1 = min(p.k_blocks, tc.kb0 + p.k_per_split);
    return tc;
  }
  const int n = p.n_mblk;
  const int32_t* up = p.halves ? cp + n_grp + 1 : cp;   // units: chunks or half chunks
  int lo = 0, hi = n_grp;                                // up[lo] * n <= t < up[hi] * n
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (up[mid] * n <= t) lo = mid; else hi = mid;
  }
  const int cg = up[lo + 1] - up[lo];
  const int local = t - up[lo] * n;
  const int G = (n % 4 == 0) ? 4 : ((n % 2 == 0) ? 2 : 1);
  const int blk = cg * G;
  const int mbb = local / blk, rem = local - mbb * blk;
  const int unit = rem / G;                              // chunk (or half chunk) in the group
  tc.mb = mbb * G + rem % G;
  if (p.halves) {
    tc.chunk = cp[lo] + (unit >> 1);
    tc.half = unit & 1;
  } else {
    tc.chunk = cp[lo] + unit;
  }
  tc.split = 0;
  tc.kb0 = 0;
  tc.kb1 = p.k_blocks;
  return tc;
}

// The rows a tile covers: its chunk, or one half of it when chunks are twice the
// tile width (nrows <= 0: nothing to do -- every role skips the tile alike).
template <int MODE, int NTW>
__device__ __forceinline__ Chunk tile_rows(const DevParams& p, const TileCoord& tc) {
  Chunk c = get_chunk<MODE>(p, tc.chunk);
  if (p.halves) {
    constexpr int kNT = Cfg<MODE, NTW>::kNT;
    const int off = tc.half * kNT;
    c.b_row += off;
    c.o_row += off;
    c.nrows -= off;
    if (c.nrows > kNT) c.nrows = kNT;
  }
  return c;
}

// Pipeline stages of variable size in a byte ring of shared memory.  A stage takes the
// bytes right after the previous stage's, or offset 0 when it would run past the end of
// the ring, so a tile of few tokens keeps more K blocks of weights in flight than a tile
// of many.  The MMA thread releases stages in issue order, so the bytes in flight are
// those between the end of the released prefix and the head (counted mod 2^32, skipped
// ring tails included).  The producer thread keeps the counters in registers and each
// slot's end in shared memory (`end`); the consumer learns each stage's offset from
// `slot_off`, written before the stage's full-barrier arrive.
template <int kSlots, uint32_t kRing>
struct StageRing {
  uint32_t head = 0;       // bytes reserved so far, mod 2^32 (skipped tails included)
  uint32_t pos = 0;        // ring offset of the head
  uint32_t freed = 0;      // end of the released prefix, same count as head
  uint32_t issued = 0, released = 0;
  uint32_t* end;           // [kSlots] shared memory: each slot's end, same count as head

  // Reserves `bytes` (a multiple of 1024, at most kRing) for the next stage, waiting on
  // the empty barriers of the oldest stages as needed; false if a wait ran out.
  __device__ __forceinline__ bool acquire(uint32_t bytes, uint64_t* empty_bar,
                                          volatile int* abort_flag, int* status, uint32_t& slot,
                                          uint32_t& off) {
    uint32_t skip = 0;
    off = pos;
    if (off + bytes > kRing) {                          // skip the ring's tail
      skip = kRing - off;
      off = 0;
    }
    // [off, off + bytes) is free once at most this many bytes before it are in flight
    const int32_t allowed = max(0, static_cast<int32_t>(kRing - bytes - skip));
    while (issued - released >= static_cast<uint32_t>(kSlots) ||
           static_cast<int32_t>(head - freed) > allowed) {
      const uint32_t s = released % kSlots;
      if (!mbar_wait(&empty_bar[s], (released / kSlots) & 1u, abort_flag, status)) return false;
      freed = end[s];
      ++released;
    }
    slot = issued % kSlots;
    head += skip + bytes;
    pos = off + bytes;
    end[slot] = head;
    ++issued;
    return true;
  }
};

// Writes a warp's 16 (rows) x 32 (columns) output block: each lane holds one column's
// 16 values; they pass through the warp's shared-memory staging area so that global
// memory sees 16-byte vector stores (each row's 32 elements are contiguous), rows at
// or past `nvalid` skipped.  `g` points at element (row 0, column 0) of the block;
// `ld` is the row pitch in elements (the pitch and `g` must be 16-byte aligned).
template <typename T>
__device__ __forceinline__ void store_block_16x32(T* g, int ld, int nvalid, const T (&v)[16],
                                                  T* stage, int lane) {
#pragma unroll
  for (int i = 0; i < 16; ++i) stage[i * 32 + lane] = v[i];
  __syncwarp();
  constexpr int kVecPerRow = 32 * static_cast<int>(sizeof(T)) / 16;
  constexpr int kElemPerVec = 16 / static_cast<int>(sizeof(T));
#pragma unroll
  for (int q = lane; q < 16 * kVecPerRow; q += 32) {
    const int row = q / kVecPerRow, cv = q % kVecPerRow;
    if (row < nvalid)
      *reinterpret_cast<uint4*>(g + static_cast<size_t>(row) * ld + cv * kElemPerVec) =
          *reinterpret_cast<const uint4*>(stage + row * 32 + cv * kElemPerVec);
  }
  __syncwarp();
}

template <int MODE, int NTW, bool GATHER>
__global__ void __launch_bounds__(Cfg<MODE, NTW, GATHER>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ DevParams p) {
  using C = Cfg<MODE, NTW, GATHER>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kRingBytes);
  uint64_t* empty_bar = full_bar + C::kSlots;
  uint64_t* tfull_bar = empty_bar + C::kSlots;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* red_bar = tempty_bar + 2;                            // [2] FP8 amax exchange
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* slot_off = tmem_slot + 2;                            // [kSlots] stage offsets
  uint32_t* slot_end = slot_off + C::kSlots;                     // [kSlots] producer's ring state
  uint8_t* staging = smem + C::kRingBytes + 1024;                // [4 warps][16 x 32 x 4 B]
  int32_t* grp_cp = reinterpret_cast<int32_t*>(staging + C::kStagingBytes);
  // FP8: [2 buffers][4 warps][128 tokens] per-warp amax of the tile's h values
  uint32_t* red = reinterpret_cast<uint32_t*>(staging + C::kStagingBytes + C::kGrpBytes + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      // the producer's expect-tx arrive, + the scale warp's lanes, + the gather threads
      mbar_init(&full_bar[i], 1 + (C::kFP8 ? 32 : 0) + (GATHER ? C::kGatherThreads : 0));
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 128);
      mbar_init(&red_bar[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.wmap[0]);
    tma_prefetch_desc(&p.tmap[0][0]);
  }
  int n_grp = 0;
  if (p.chunks) {
    n_grp = *p.n_grp;
    for (int i = threadIdx.x; i < 2 * (n_grp + 1); i += blockDim.x) grp_cp[i] = p.grp_cp[i];
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_chunks = p.chunks ? *p.n_chunks : (p.router_T + kChunkRows - 1) / kChunkRows;
  const int n_units = !p.chunks ? n_chunks : (p.halves ? grp_cp[2 * n_grp + 1] : n_chunks);
  const int n_tiles = n_units * p.n_mblk * (p.chunks ? 1 : p.k_splits);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      StageRing<C::kSlots, C::kRingBytes> ring;
      ring.end = slot_end;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
        const Chunk c = tile_rows<MODE, NTW>(p, tc);
        if (c.nrows <= 0) continue;
        const int mb = tc.mb;
        // first weight row of the tile; FFN1's second weight tile holds the up rows of the
        // same h columns, FFN2's further tiles the next 128-row blocks
        const int a_row = c.group * p.w_rows_per_group + mb * kBM * C::kOutBlocks;
        const int n_pad = (c.nrows + 15) & ~15;
        // the second GEMM reads the h rows the first one wrote (output numbering)
        const int tok_row = C::kSecond ? c.o_row : c.b_row;
        // TMA bytes per stage: a packed FP4 weight box lands unpacked (16 KB of shared memory)
        // but completes its packed size in bytes (8 KB) on the barrier
        const uint32_t bytes = C::kATiles * (C::kW4 ? kABytes / 2 : kABytes) +
                               (GATHER ? 0u : static_cast<uint32_t>(n_pad) * kRowBytes);
        const uint32_t stage_bytes = C::kFixedStages ? C::kStageBytes : bytes;  // ring bytes per stage
        const CUtensorMap* wm = &p.wmap[c.seg];
        for (int kb = tc.kb0; kb < tc.kb1; ++kb) {
          uint32_t slot, soff;
          if (!ring.acquire(stage_bytes, empty_bar, abort_flag, p.status, slot, soff)) {
            ok = false;
            break;
          }
          uint8_t* st = tiles + soff;
          slot_off[slot] = soff;
          const int kx = kb * (C::kFP8 ? 128 : 64);   // element coordinate of this K block
          mbar_arrive_expect_tx(&full_bar[slot], bytes);
          tma_load_2d(st, wm, &full_bar[slot], kx, a_row);
          if (C::kGLU) tma_load_2d(st + kABytes, wm, &full_bar[slot], kx, a_row + p.up_offset);
#pragma unroll
          for (int j = 1; j < C::kOutBlocks; ++j)
            tma_load_2d(st + j * kABytes, wm, &full_bar[slot], kx, a_row + j * kBM);
          uint8_t* bt = st + C::kATiles * kABytes;
          // token rows as boxes of 128 / 64 / 32 / 16 rows covering n_pad (unless gathered)
          for (int bi = 0, off = 0; bi < kTokBoxes && !GATHER; ++bi) {
            const int rows = 128 >> bi;
            while (n_pad - off >= rows) {
              tma_load_2d(bt + off * kRowBytes, &p.tmap[c.seg][bi], &full_bar[slot], kx, tok_row + off);
              off += rows;
            }
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
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
        const Chunk c = tile_rows<MODE, NTW>(p, tc);
        if (c.nrows <= 0) continue;
        const int n_pad = (c.nrows + 15) & ~15;
        const uint32_t idesc = C::kFP8 ? idesc_e4m3_bs(kBM, n_pad) : idesc_bf16_f32(kBM, n_pad);
        // FP4 weights: MMA kk of a stage applies byte kk of each weight row's scale word
        const uint32_t idesc_w4 = idesc_mx_bs(kFmtE2M1, kFmtE4M3, kBM, n_pad, 0, 0);
        const uint32_t acc = it % C::kAccBufs;
        const uint32_t acc_phase = (it / C::kAccBufs) & 1;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * C::kAccCols;
        const uint32_t d1 = d0 + C::kNT;
        for (int kb = tc.kb0; kb < tc.kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(tiles) + slot_off[stage];
          const uint32_t bt = st + C::kATiles * kABytes;
          // rows written by cp.async (scale atoms, gathered tokens) before the async-proxy reads
          if (C::kFP8 || GATHER) fence_proxy_async_smem();
          if (C::kFP8) {
            // scale factors of this stage: smem (written by the scale warp) -> TMEM
            const uint32_t sf_smem = bt + C::kBBytes;
            const uint32_t sfa = tmem_base + C::kAccBufs * C::kAccCols + stage * C::kSFColsPerStage;
            const uint32_t sfb = sfa + C::kATiles * 4;
            // weight-side scales: one atom per weight tile (gate and up, or output blocks)
#pragma unroll
            for (int j = 0; j < C::kATiles; ++j)
              tmem_cp_32x128b_warpx4(sfa + 4 * j, smem_desc_noswizzle(sf_smem + j * kSFAtomBytes));
            // token-side scales: one atom per 128 token rows, in consecutive 4-column groups
#pragma unroll
            for (int a = 0; a < C::kSFBAtoms; ++a)
              tmem_cp_32x128b_warpx4(sfb + 4 * a,
                                     smem_desc_noswizzle(sf_smem + (C::kATiles + a) * kSFAtomBytes));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t accum = (kb > tc.kb0 || kk) ? 1u : 0u;
              const uint64_t bdesc = umma_desc_sw128(bt + kk * 32);
              const uint32_t id = C::kW4 ? (idesc_w4 | (static_cast<uint32_t>(kk) << 29)) : idesc;
#pragma unroll
              for (int j = 0; j < C::kATiles; ++j)
                umma_e4m3_bs(d0 + j * C::kNT, umma_desc_sw128(st + j * kABytes + kk * 32), bdesc, id,
                             sfa + 4 * j, sfb, accum);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t accum = (kb > tc.kb0 || kk) ? 1u : 0u;
              const uint64_t bdesc = umma_desc_sw128(bt + kk * 32);
              umma_bf16(d0, umma_desc_sw128(st + kk * 32), bdesc, idesc, accum);
#pragma unroll
              for (int j = 1; j < C::kATiles; ++j)
                umma_bf16(d0 + j * C::kNT, umma_desc_sw128(st + j * kABytes + kk * 32), bdesc, idesc, accum);
            }
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == C::kSlots) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull_bar[acc]);
        ++it;
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;                 // TMEM lane quadrant of this warp
    const int m_local = sub * 32 + lane;      // weight row inside the tile
    int it = 0;
    uint32_t rbuf = 0, rpar = 0;              // FP8 amax exchange: buffer and per-buffer parity bits
    bool epi_ok = true;
    for (int t = blockIdx.x; t < n_tiles && epi_ok; t += gridDim.x) {
      const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
      const Chunk c = tile_rows<MODE, NTW>(p, tc);
      if (c.nrows <= 0) continue;
      const int mb = tc.mb;
      const uint32_t acc = it % C::kAccBufs;
      const uint32_t acc_phase = (it / C::kAccBufs) & 1;
      bool ok = mbar_wait(&tfull_bar[acc], acc_phase, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + acc * C::kAccCols;
      const int m = mb * kBM + m_local;       // output column
      if (C::kGLU && C::kFP8) {
        // SwiGLU, then requantise h to e4m3 with one power-of-two scale per token per 128
        // h columns (this tile's columns).  Pass 1: per token, the maximum |h| of each
        // warp's 32 columns (redux.sync) into shared memory; one exchange between the
        // four epilogue warps (mbarrier, bounded wait); pass 2: reload the accumulators,
        // recompute h, scale, round to e4m3 and store with the scales.
        uint32_t* redt = red + rbuf * (4 * 128);
        for (int n0 = 0; n0 < c.nrows; n0 += 16) {
          float g[16], u[16];
          tmem_ld16x2(tb + n0, tb + C::kNT + n0, g, u);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float hv = g[i] / (1.0f + __expf(-g[i])) * u[i];
            const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(hv)));
            if (lane == 0) redt[sub * 128 + n0 + i] = wmax;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_bar[rbuf]);
        const bool rok = mbar_wait(&red_bar[rbuf], (rpar >> rbuf) & 1u, abort_flag, p.status);
        rpar ^= 1u << rbuf;
        if (!__all_sync(0xffffffffu, rok)) {
          epi_ok = false;
        } else {
          for (int n0 = 0; n0 < c.nrows; n0 += 16) {
            float g[16], u[16];
            tmem_ld16x2(tb + n0, tb + C::kNT + n0, g, u);
            uint8_t q[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float hv = g[i] / (1.0f + __expf(-g[i])) * u[i];
              const int n = n0 + i;
              const uint32_t amax = max(max(redt[n], redt[128 + n]), max(redt[256 + n], redt[384 + n]));
              const int e = e4m3_scale_exponent(amax);
              q[i] = __nv_cvt_float_to_fp8(scalbnf(hv, -e), __NV_SATFINITE, __NV_E4M3);
              if (m_local == 0 && n < c.nrows)
                p.out_sf[static_cast<size_t>(mb) * p.ld_out_sf + c.o_row + n] =
                    0x01010101u * static_cast<uint32_t>(e + 127);
            }
            store_block_16x32(static_cast<uint8_t*>(p.out) +
                                  static_cast<size_t>(c.o_row + n0) * p.ld_out + (m - lane),
                              p.ld_out, c.nrows - n0, q, staging + sub * 2048, lane);
          }
        }
        rbuf ^= 1u;
      }
      for (int n0 = 0; n0 < c.nrows && !(C::kGLU && C::kFP8); n0 += 16) {
        if (MODE == kFFN1) {
          float g[16], u[16];
          tmem_ld16x2(tb + n0, tb + C::kNT + n0, g, u);
          __nv_bfloat16 hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) hv[i] = __float2bfloat16_rn(g[i] / (1.0f + __expf(-g[i])) * u[i]);
          store_block_16x32(static_cast<__nv_bfloat16*>(p.out) +
                                static_cast<size_t>(c.o_row + n0) * p.ld_out + (m - lane),
                            p.ld_out, c.nrows - n0, hv,
                            reinterpret_cast<__nv_bfloat16*>(staging + sub * 2048), lane);
        } else if (MODE == kFFN2M256 || MODE == kFFN2M512 || MODE == kFFN2F8M256 ||
                   MODE == kFFN2F4M256) {
          // accumulator j holds output columns (mb * kOutBlocks + j) * 128 + (0..127)
          __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(p.out) + static_cast<size_t>(c.o_row + n0) * p.ld_out +
                                (mb * C::kOutBlocks * kBM + m_local - lane);
#pragma unroll
          for (int j = 0; j < C::kOutBlocks; j += 2) {
            float v0[16], v1[16];
            tmem_ld16x2(tb + j * C::kNT + n0, tb + (j + 1) * C::kNT + n0, v0, v1);
            __nv_bfloat16 yv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) yv[i] = __float2bfloat16_rn(v0[i]);
            store_block_16x32(yrow + j * kBM, p.ld_out, c.nrows - n0, yv,
                              reinterpret_cast<__nv_bfloat16*>(staging + sub * 2048), lane);
#pragma unroll
            for (int i = 0; i < 16; ++i) yv[i] = __float2bfloat16_rn(v1[i]);
            store_block_16x32(yrow + (j + 1) * kBM, p.ld_out, c.nrows - n0, yv,
                              reinterpret_cast<__nv_bfloat16*>(staging + sub * 2048), lane);
          }
        } else if (MODE == kFFN2 || MODE == kFFN2F8 || MODE == kFFN2F4) {
          float v[16];
          tmem_ld16(tb + n0, v);
          __nv_bfloat16 yv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) yv[i] = __float2bfloat16_rn(v[i]);
          store_block_16x32(static_cast<__nv_bfloat16*>(p.out) +
                                static_cast<size_t>(c.o_row + n0) * p.ld_out + (m - lane),
                            p.ld_out, c.nrows - n0, yv,
                            reinterpret_cast<__nv_bfloat16*>(staging + sub * 2048), lane);
        } else {
          float v[16];
          tmem_ld16(tb + n0, v);
          float* lg = static_cast<float*>(p.out) + tc.split * p.split_stride;
          if (m < p.m_valid) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n0 + i < c.nrows) lg[static_cast<size_t>(c.o_row + n0 + i) * p.ld_out + m] = v[i];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      ++it;
    }
  } else if (C::kFP8 && warp == 6) {
    // ------------------------------------------------------------ scale-factor warp (FP8)
    // Per stage: the 512-byte scale atoms of the weight tile(s) and of the token rows (row
    // n's 4 bytes at (n % 32) * 16 + (n / 32) * 4), copied with cp.async; each lane's
    // completion arrives on the stage's full barrier.  e4m3 weights: one UE8M0 value for
    // the whole 128x128 block, replicated.  FP4 weights: row r's 4 bytes are its E8M0
    // scales of the stage's four 32-element K runs, copied from the caller's atoms.
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    const int up_rb = p.up_offset / kBM;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
      const Chunk c = tile_rows<MODE, NTW>(p, tc);
      if (c.nrows <= 0) continue;
      const int mb = tc.mb;
      const int n_pad = (c.nrows + 15) & ~15;
      const int tok_row = C::kSecond ? c.o_row : c.b_row;
      const uint4* wsf = C::kW4 ? nullptr
                                : p.wsf[c.seg] + static_cast<size_t>(c.group) * p.wsf_rb_per_group * p.k_blocks;
      const uint32_t* tsf = p.tsf[c.seg];
      const int tld = p.tsf_ld[c.seg], trows = p.tsf_rows[c.seg];
      // the scale row of each of this lane's token rows, looked up once per tile
      int trow[4 * C::kSFBAtoms];
#pragma unroll
      for (int j = 0; j < 4 * C::kSFBAtoms; ++j) {
        const int n = lane + 32 * j;
        trow[j] = min(tok_row + n, trows - 1);
        if (GATHER) {                      // the token's own row of the unpermuted scales
          const int32_t* gi = p.gidx[c.seg];
          const int src = c.b_row + min(n, c.nrows - 1);
          trow[j] = gi ? __ldg(gi + src) : src;
        }
      }
      for (int kb = tc.kb0; kb < tc.kb1; ++kb) {
        const bool w = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        uint8_t* sf = tiles + stage * C::kStageBytes + C::kATiles * kABytes + C::kBBytes;
#pragma unroll
        for (int j = 0; j < C::kATiles; ++j) {
          // 128-row block of the weight matrix behind weight tile j: gate / up rows, or
          // consecutive output blocks
          const int rb = C::kGLU ? (j ? up_rb + mb : mb) : mb * C::kOutBlocks + j;
          if (C::kW4) {
            // the caller's atoms are already in the layout tcgen05.cp reads: 16 bytes per lane
            const uint4* wsc = p.wsc[c.seg] + static_cast<size_t>(c.group) * p.wsf_rb_per_group * p.k_blocks * 32;
            cp_async_16(sf + j * kSFAtomBytes + lane * 16,
                        wsc + (static_cast<size_t>(rb) * p.k_blocks + kb) * 32 + lane);
          } else {
            cp_async_16(sf + j * kSFAtomBytes + lane * 16, wsf + static_cast<size_t>(rb) * p.k_blocks + kb);
          }
        }
        uint8_t* sfb = sf + C::kATiles * kSFAtomBytes;
#pragma unroll
        for (int j = 0; j < 4 * C::kSFBAtoms; ++j) {
          const int n = lane + 32 * j;     // atom j / 4, in-atom row group j % 4
          if (n < n_pad) {
            const int row = trow[j];
            cp_async_4(sfb + (j >> 2) * kSFAtomBytes + lane * 16 + (j & 3) * 4,
                       tsf + static_cast<size_t>(kb) * tld + row);
          }
        }
        cp_async_mbar_arrive_noinc(&full_bar[stage]);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    __syncwarp();
  } else if (GATHER && warp >= C::kGatherWarp0) {
    // ------------------------------------------------------------ gather warps
    // Per stage: the tile's token rows, 128 bytes of K each, copied from the unpermuted
    // activations with 16-byte cp.async into the 128-byte swizzled layout (16-byte chunk j
    // of row n at n * 128 + ((j ^ (n % 8)) * 16), as TMA's 128-byte swizzle places it).
    // Thread g copies chunk g % 8 of rows g / 8 + 16 i: a warp instruction covers four
    // whole 128-byte rows.  Padding rows (past the chunk's rows) are not copied: their
    // products land only in output rows that are never stored.  Each thread's completion
    // arrives on the stage's full barrier.
    const int g = threadIdx.x - C::kGatherWarp0 * 32;
    const int j = g & 7, r0 = g >> 3;
    constexpr int kRowsPerThread = (C::kNT + 15) / 16;
    // source rows of this thread's token rows in the tile: looked up one tile ahead, so
    // that the index loads' latency hides behind the previous tile's stages
    auto rows_of = [&](int t, int (&rows)[kRowsPerThread], Chunk& c, TileCoord& tc) {
      tc = tile_coord(p, t, grp_cp, n_grp);
      c = tile_rows<MODE, NTW>(p, tc);
      const int32_t* gi = c.nrows > 0 ? p.gidx[c.seg] : nullptr;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int n = r0 + 16 * i;
        rows[i] = n < c.nrows ? (gi ? __ldg(gi + c.b_row + n) : c.b_row + n) : 0;
      }
    };
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    int rows[kRowsPerThread], next_rows[kRowsPerThread];
    Chunk c, next_c;
    TileCoord tc, next_tc;
    if (blockIdx.x < n_tiles) rows_of(blockIdx.x, next_rows, next_c, next_tc);
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      c = next_c;
      tc = next_tc;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) rows[i] = next_rows[i];
      if (t + static_cast<int>(gridDim.x) < n_tiles)
        rows_of(t + gridDim.x, next_rows, next_c, next_tc);
      if (c.nrows <= 0) continue;
      const uint8_t* src[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i)
        src[i] = p.gsrc[c.seg] + static_cast<size_t>(rows[i]) * p.g_ld + j * 16;
      for (int kb = tc.kb0; kb < tc.kb1; ++kb) {
        const bool w = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        uint8_t* bt = tiles + stage * C::kStageBytes + C::kATiles * kABytes;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          const int n = r0 + 16 * i;
          if (n < c.nrows)
            cp_async_16_cg(bt + n * kRowBytes + ((j ^ (n & 7)) << 4), src[i] + kb * kRowBytes);
        }
        cp_async_mbar_arrive_noinc(&full_bar[stage]);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}


// ---------------------------------------------------------------- fp32 block scales
// e4m3 expert GEMMs whose block scales are arbitrary positive fp32 values (not powers of
// two, which the tensor cores' UE8M0 scale factors cannot hold).  The MMAs run without
// block scaling (kind::f8f6f4); every 128-K block accumulates into its own TMEM buffer
// (several in rotation), and the epilogue warps fold it into fp32 register accumulators as
//   acc[r][n] += (s_w[block of r][kb] * s_a[n][kb]) * partial_kb[r][n]
// -- the block-scaled product summed exactly as its definition states, in fp32.  Tiles are
// NT = 32 tokens wide on decode-sized batches, else 64 (the accumulators of a tile live in
// registers: each epilogue warp holds 32 tokens of its 32 weight rows, so a 64-token tile
// has two sets of four epilogue warps), and 128 weight rows per weight tile (gate and up
// for the first GEMM; one or two output blocks for the second).
//   warp 0  TMA producer; warp 1  MMA issuer (also moves each block's scales from the stage
//   to a per-buffer slot the epilogue reads); warps 2 .. 2 + 4 NT / 32 - 1  epilogue; the
//   last warp  scale warp (cp.async of the stage's raw token and weight scales).
template <int MODE, int NT>
struct CfgFS {
  static constexpr bool kGLU = MODE == kFFN1X;
  static constexpr bool kSecond = MODE == kFFN2X || MODE == kFFN2XM256;   // reads h
  // FFN2: 128-row weight blocks (= 128 output columns each) per tile
  static constexpr int kOutBlocks = MODE == kFFN2XM256 ? 2 : 1;
  static constexpr int kATiles = kGLU ? 2 : kOutBlocks;
  static constexpr int kNT = NT;                                  // 32 or 64 tokens
  static_assert(NT == 32 || NT == 64, "token tile width");
  static constexpr int kEpiWarps = 4 * (kNT / 32);                // four per 32 tokens
  static constexpr int kScaleWarp = 2 + kEpiWarps;
  static constexpr uint32_t kBBytes = kNT * kRowBytes;
  static constexpr uint32_t kRawBytes = 1024;                     // [kNT] token + [2] weight scales
  static constexpr uint32_t kRawW = kNT * 4;                      // weight scales in the raw block
  static constexpr uint32_t kStageBytes = kATiles * kABytes + kBBytes + kRawBytes;
  static constexpr int kStages = (192u * 1024u) / kStageBytes > 10 ? 10 : (192u * 1024u) / kStageBytes;
  static constexpr uint32_t kPCols = kATiles * kNT;               // per partial buffer
  // partial buffers in flight (eight, or as many as TMEM holds): each K block's round trip
  // (MMAs, commit, the epilogue's TMEM loads and release) spans several K blocks of the
  // weight stream
  static constexpr int kPBufs = 512 / kPCols < 8 ? 512 / kPCols : 8;
  static constexpr uint32_t kTmemCols =
      kPBufs * kPCols <= 64 ? 64
                            : (kPBufs * kPCols <= 128 ? 128 : (kPBufs * kPCols <= 256 ? 256 : 512));
  static_assert(kPBufs * kPCols <= 512, "TMEM budget");
  static constexpr int kThreads = 32 * (3 + kEpiWarps);
  static constexpr uint32_t kStagingBytes = kEpiWarps * 16 * 32 * 4;
  static constexpr uint32_t kGrpBytes = (2 * (kMaxGroups + 1) * 4 + 15) & ~15u;   // 16-byte multiple
  static constexpr uint32_t kRedBytes = 2 * 4 * kNT * 4;          // [2][4 row quadrants][kNT]
  static constexpr int kSlot = kNT + 32;                          // floats per scale slot
  static constexpr uint32_t kPScaleBytes = kPBufs * kSlot * 4;    // [buffers][kNT token + 2 weight]
  static constexpr uint32_t kFixedBytes =
      1024 + kStagingBytes + kGrpBytes + kRedBytes + kPScaleBytes + 1024;
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + kFixedBytes;
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kSmemBytes <= kMaxSmem, "shared memory budget");
};

template <int MODE, int NT>
__global__ void __launch_bounds__(CfgFS<MODE, NT>::kThreads, 1)
    grouped_gemm_fs_kernel(const __grid_constant__ DevParams p) {
  using C = CfgFS<MODE, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty_bar = full_bar + C::kStages;
  uint64_t* pfull = empty_bar + C::kStages;                      // [kPBufs] partial buffer written
  uint64_t* pempty = pfull + C::kPBufs;                          // [kPBufs] partial buffer read
  uint64_t* red_bar = pempty + C::kPBufs;                        // [2] amax exchange
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* staging = smem + C::kStages * C::kStageBytes + 1024;
  int32_t* grp_cp = reinterpret_cast<int32_t*>(staging + C::kStagingBytes);
  uint32_t* red = reinterpret_cast<uint32_t*>(staging + C::kStagingBytes + C::kGrpBytes);
  float* pscale = reinterpret_cast<float*>(staging + C::kStagingBytes + C::kGrpBytes + C::kRedBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full_bar[i], 1 + 32);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < C::kPBufs; ++i) {
      mbar_init(&pfull[i], 2);        // the MMAs' commit + the scales' copy
      mbar_init(&pempty[i], C::kEpiWarps);   // one arrival per epilogue warp
    }
    for (int i = 0; i < 2; ++i) mbar_init(&red_bar[i], C::kEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.wmap[0]);
    tma_prefetch_desc(&p.tmap[0][0]);
  }
  const int n_grp = *p.n_grp;
  for (int i = threadIdx.x; i < 2 * (n_grp + 1); i += blockDim.x) grp_cp[i] = p.grp_cp[i];
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_tiles = *p.n_chunks * p.n_mblk;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
        const Chunk c = tile_rows<MODE, kChunkRowsNarrow>(p, tc);
        if (c.nrows <= 0) continue;
        const int a_row = c.group * p.w_rows_per_group + tc.mb * kBM * C::kOutBlocks;
        const int n_pad = (c.nrows + 15) & ~15;
        const int tok_row = C::kSecond ? c.o_row : c.b_row;
        const uint32_t bytes = C::kATiles * kABytes + n_pad * kRowBytes;
        const CUtensorMap* wm = &p.wmap[c.seg];
        for (int kb = tc.kb0; kb < tc.kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* st = tiles + stage * C::kStageBytes;
          const int kx = kb * 128;
          mbar_arrive_expect_tx(&full_bar[stage], bytes);
          tma_load_2d(st, wm, &full_bar[stage], kx, a_row);
          if (C::kGLU) tma_load_2d(st + kABytes, wm, &full_bar[stage], kx, a_row + p.up_offset);
#pragma unroll
          for (int j = 1; j < C::kOutBlocks; ++j)
            tma_load_2d(st + j * kABytes, wm, &full_bar[stage], kx, a_row + j * kBM);
          uint8_t* bt = st + C::kATiles * kABytes;
          for (int bi = 0, off = 0; bi < kTokBoxes; ++bi) {
            const int rows = 128 >> bi;
            while (n_pad - off >= rows) {
              tma_load_2d(bt + off * kRowBytes, &p.tmap[c.seg][bi], &full_bar[stage], kx, tok_row + off);
              off += rows;
            }
          }
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
    // The whole warp waits; lane n moves token n's scale, lane 0 issues the MMAs.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t kc = 0;                   // K blocks issued so far (partial buffer kc % kPBufs)
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
      const Chunk c = tile_rows<MODE, kChunkRowsNarrow>(p, tc);
      if (c.nrows <= 0) continue;
      const int n_pad = (c.nrows + 15) & ~15;
      const uint32_t idesc = idesc_e4m3_f32(kBM, n_pad);
      for (int kb = tc.kb0; kb < tc.kb1; ++kb, ++kc) {
        const uint32_t b = kc % C::kPBufs;
        const bool w = mbar_wait(&full_bar[stage], phase, abort_flag, p.status) &&
                       mbar_wait(&pempty[b], ((kc / C::kPBufs) & 1u) ^ 1u, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = tiles + stage * C::kStageBytes;
        const uint8_t* raw = st + C::kATiles * kABytes + C::kBBytes;
        float* ps = pscale + b * C::kSlot;
        // this K block's scales to the buffer's slot: token n's (fp32, or h's UE8M0 word
        // -> 2^(code - 127)) and each weight tile's fp32 block scale
#pragma unroll
        for (int n = lane; n < C::kNT; n += 32) {
          if (n >= c.nrows) break;
          if (C::kSecond) {
            const uint32_t code = reinterpret_cast<const uint32_t*>(raw)[n] & 0xFFu;
            ps[n] = code ? __uint_as_float(code << 23) : __uint_as_float(0x00400000u);
          } else {
            ps[n] = reinterpret_cast<const float*>(raw)[n];
          }
        }
        if (lane < C::kATiles) ps[C::kNT + lane] = reinterpret_cast<const float*>(raw + C::kRawW)[lane];
        __syncwarp();
        if (lane == 0) {
          fence_proxy_async_smem();    // the scale warp's cp.async rows before any async read
          const uint32_t sa = smem_u32(st), sb = sa + C::kATiles * kABytes;
          const uint32_t d0 = tmem_base + b * C::kPCols;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = umma_desc_sw128(sb + kk * 32);
#pragma unroll
            for (int j = 0; j < C::kATiles; ++j)
              umma_e4m3(d0 + j * C::kNT, umma_desc_sw128(sa + j * kABytes + kk * 32), bdesc, idesc,
                        kk ? 1u : 0u);
          }
          umma_commit(&empty_bar[stage]);   // the stage's operands and raw scales are consumed
          umma_commit(&pfull[b]);           // the partial sums are in TMEM
          mbar_arrive(&pfull[b]);           // the scales are in their slot
        }
        __syncwarp();
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    __syncwarp();
  } else if (warp < C::kScaleWarp) {
    // ------------------------------------------------------------ epilogue
    // Warp 2 + e: TMEM lane quadrant warp % 4 (32 weight rows), tokens 32 (e / 4) .. + 31.
    const int sub = warp & 3;
    const int e_warp = warp - 2;
    const int n_base = C::kNT > 32 ? (e_warp >> 2) * 32 : 0;   // this warp's first token
    const int m_local = sub * 32 + lane;      // weight row inside the tile
    uint8_t* stg = staging + e_warp * 2048;
    uint32_t kc = 0;
    uint32_t rbuf = 0, rpar = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
      const Chunk c = tile_rows<MODE, kChunkRowsNarrow>(p, tc);
      if (c.nrows <= 0) continue;
      const int rows = c.nrows - n_base;      // this warp's tokens (<= 0: none; warp-uniform)
      float acc[C::kATiles][32];
#pragma unroll
      for (int j = 0; j < C::kATiles; ++j)
#pragma unroll
        for (int n = 0; n < 32; ++n) acc[j][n] = 0.f;
      for (int kb = tc.kb0; kb < tc.kb1; ++kb, ++kc) {
        const uint32_t b = kc % C::kPBufs;
        const bool w = mbar_wait(&pfull[b], (kc / C::kPBufs) & 1u, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (rows > 0) {
          const float* ps = pscale + b * C::kSlot;
          const uint32_t tb =
              tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + b * C::kPCols + n_base;
#pragma unroll
          for (int j = 0; j < C::kATiles; ++j) {
            float v0[16], v1[16];
            tmem_ld16x2(tb + j * C::kNT, tb + j * C::kNT + 16, v0, v1);
            const float sw = ps[C::kNT + j];
#pragma unroll
            for (int n = 0; n < 16; ++n) {
              acc[j][n] = fmaf(sw * ps[n_base + n], v0[n], acc[j][n]);
              acc[j][16 + n] = fmaf(sw * ps[n_base + 16 + n], v1[n], acc[j][16 + n]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[b]);
      }
      if (!ok) break;
      const int mb = tc.mb;
      const int o_row = c.o_row + n_base;     // this warp's first output row
      if (MODE == kFFN1X) {
        // SwiGLU, then h requantised to e4m3 with one power-of-two scale per token per 128 h
        // columns, exchanged between the four warps of the token's rows (as the block-scaled
        // path does); every epilogue warp arrives on the exchange barrier
        constexpr int kRR = C::kNT;
        float h[32];
        uint32_t* redt = red + rbuf * (4 * kRR);
#pragma unroll
        for (int n = 0; n < 32; ++n) {
          h[n] = acc[0][n] / (1.0f + __expf(-acc[0][n])) * acc[1][n];
          const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h[n])));
          if (lane == 0) redt[sub * kRR + n_base + n] = wmax;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_bar[rbuf]);
        const bool rok = mbar_wait(&red_bar[rbuf], (rpar >> rbuf) & 1u, abort_flag, p.status);
        rpar ^= 1u << rbuf;
        if (!__all_sync(0xffffffffu, rok)) break;
#pragma unroll
        for (int n0 = 0; n0 < 32; n0 += 16) {
          uint8_t q[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = n_base + n0 + i;
            const uint32_t amax =
                max(max(redt[n], redt[kRR + n]), max(redt[2 * kRR + n], redt[3 * kRR + n]));
            const int e = e4m3_scale_exponent(amax);
            q[i] = __nv_cvt_float_to_fp8(scalbnf(h[n0 + i], -e), __NV_SATFINITE, __NV_E4M3);
            if (m_local == 0 && n0 + i < rows)
              p.out_sf[static_cast<size_t>(mb) * p.ld_out_sf + o_row + n0 + i] =
                  0x01010101u * static_cast<uint32_t>(e + 127);
          }
          if (n0 < rows)
            store_block_16x32(static_cast<uint8_t*>(p.out) + static_cast<size_t>(o_row + n0) * p.ld_out +
                                  (mb * kBM + sub * 32),
                              p.ld_out, rows - n0, q, stg, lane);
        }
        rbuf ^= 1u;
      } else {
        // accumulator j holds output columns (mb * kOutBlocks + j) * 128 + (0..127)
#pragma unroll
        for (int j = 0; j < C::kATiles; ++j) {
#pragma unroll
          for (int n0 = 0; n0 < 32; n0 += 16) {
            __nv_bfloat16 yv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) yv[i] = __float2bfloat16_rn(acc[j][n0 + i]);
            if (n0 < rows)
              store_block_16x32(static_cast<__nv_bfloat16*>(p.out) + static_cast<size_t>(o_row + n0) * p.ld_out +
                                    ((mb * C::kOutBlocks + j) * kBM + sub * 32),
                                p.ld_out, rows - n0, yv, reinterpret_cast<__nv_bfloat16*>(stg), lane);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ scale warp
    // Per stage: lanes copy the tile's token scales of this K block (token n by lane n % 32;
    // fp32, or h's UE8M0 word), lanes 0..kATiles-1 the weight tiles' fp32 block scales, with
    // cp.async; each lane's completion arrives on the stage's full barrier.
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    const int up_rb = p.up_offset / kBM;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      const TileCoord tc = tile_coord(p, t, grp_cp, n_grp);
      const Chunk c = tile_rows<MODE, kChunkRowsNarrow>(p, tc);
      if (c.nrows <= 0) continue;
      const int mb = tc.mb;
      const float* wsc = p.fs_w[c.seg] + static_cast<size_t>(c.group) * p.wsf_rb_per_group * p.k_blocks;
      for (int kb = tc.kb0; kb < tc.kb1; ++kb) {
        const bool w = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        uint8_t* raw = tiles + stage * C::kStageBytes + C::kATiles * kABytes + C::kBBytes;
#pragma unroll
        for (int n = lane; n < C::kNT; n += 32) {
          if (n >= c.nrows) break;
          if (C::kSecond)
            cp_async_4(raw + n * 4, p.tsf[c.seg] + static_cast<size_t>(kb) * p.tsf_ld[c.seg] + c.o_row + n);
          else
            cp_async_4(raw + n * 4, p.fs_a[c.seg] + static_cast<size_t>(c.b_row + n) * p.fs_a_ld + kb);
        }
        if (lane < C::kATiles) {
          const int rb = C::kGLU ? (lane ? up_rb + mb : mb) : mb * C::kOutBlocks + lane;
          cp_async_4(raw + C::kRawW + lane * 4, wsc + static_cast<size_t>(rb) * p.k_blocks + kb);
        }
        cp_async_mbar_arrive_noinc(&full_bar[stage]);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------- planner
// Exclusive block-wide scan (1024 threads, <= 2048 entries) of ceil(sz[order[r]] / rows)
// over ranks r, into base[0..NG].
__device__ void block_scan_counts(const int32_t* sz, const int32_t* order, int NG, int rows,
                                  int32_t* base, int32_t* warp_sum) {
  const int tid = threadIdx.x;
  int c0 = 0, c1 = 0;
  const int r0 = 2 * tid, r1 = 2 * tid + 1;
  if (r0 < NG) c0 = (sz[order[r0]] + rows - 1) / rows;
  if (r1 < NG) c1 = (sz[order[r1]] + rows - 1) / rows;
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
  if (r0 < NG) base[r0] = excl;
  if (r1 < NG) base[r1] = excl + c0;
  if (tid == blockDim.x - 1) base[NG] = excl + local;
  __syncthreads();
}

// One CTA.  Validates the offsets, orders the groups by size (largest first,
// ties by index: routed before shared), splits each into chunks of at most
// `cr` rows (the GEMM's token tile) and writes the chunk list and its length.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ offsets, int G,
                                                    int n_rows, int n_shared, int T,
                                                    int shared_o_row, int cr,
                                                    Chunk* __restrict__ chunks,
                                                    int32_t* __restrict__ n_chunks,
                                                    int32_t* __restrict__ grp_cp,
                                                    int32_t* __restrict__ n_grp, int* status) {
  __shared__ int32_t sz[kMaxGroups];
  __shared__ int32_t start[kMaxGroups];
  __shared__ int32_t order[kMaxGroups];
  __shared__ int32_t cbase[kMaxGroups + 1];
  __shared__ int32_t hbase[kMaxGroups + 1];
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
      *n_grp = 0;
      grp_cp[0] = 0;
      grp_cp[1] = 0;
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
  // exclusive scans, in rank order, of the chunk counts (chunks of cr rows) and of the
  // half-chunk counts (cr / 2 rows)
  block_scan_counts(sz, order, NG, cr, cbase, warp_sum);
  block_scan_counts(sz, order, NG, cr / 2, hbase, warp_sum);
  for (int r = tid; r < NG; r += blockDim.x) {
    const int g = order[r];
    const int s = sz[g];
    const bool shared = g >= G;
    int base = cbase[r];
    for (int c = 0; c * cr < s; ++c) {
      Chunk ch;
      ch.seg = shared ? 1 : 0;
      ch.group = shared ? g - G : g;
      ch.b_row = start[g] + c * cr;
      ch.o_row = shared ? shared_o_row + (g - G) * T + c * cr : ch.b_row;
      ch.nrows = min(cr, s - c * cr);
      ch.pad0 = ch.pad1 = ch.pad2 = 0;
      chunks[base + c] = ch;
    }
  }
  for (int r = tid; r <= NG; r += blockDim.x) {
    grp_cp[r] = cbase[r];
    grp_cp[NG + 1 + r] = hbase[r];
  }
  if (tid == 0) {
    *n_chunks = cbase[NG];
    *n_grp = NG;
  }
}

}  // namespace

cudaError_t launch_plan(const int32_t* offsets, int G, int n_rows, int n_shared, int T,
                        int shared_o_row, int chunk_rows, Chunk* chunks, int32_t* n_chunks,
                        int32_t* grp_cp, int32_t* n_grp, int* status, cudaStream_t s) {
  plan_kernel<<<1, 1024, 0, s>>>(offsets, G, n_rows, n_shared, T, shared_o_row, chunk_rows, chunks,
                                 n_chunks, grp_cp, n_grp, status);
  return cudaGetLastError();
}

template <int MODE, int NTW, bool GATHER = false>
static cudaError_t launch_mode(const GemmLaunch& g, cudaStream_t s) {
  using C = Cfg<MODE, NTW, GATHER>;
  static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
  DevParams p;
  for (int i = 0; i < 2; ++i) p.wmap[i] = g.wmap[i];
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < kTokBoxes; ++j) p.tmap[i][j] = g.tmap[i][j];
  p.chunks = g.chunks;
  p.n_chunks = g.n_chunks;
  p.grp_cp = g.grp_cp;
  p.n_grp = g.n_grp;
  p.halves = g.halves ? 1 : 0;
  p.router_T = g.router_T;
  p.n_mblk = g.n_mblk;
  p.k_blocks = g.k_blocks;
  p.k_splits = g.k_splits > 1 ? g.k_splits : 1;
  p.k_per_split = (g.k_blocks + p.k_splits - 1) / p.k_splits;
  p.split_stride = g.split_stride;
  p.w_rows_per_group = g.w_rows_per_group;
  p.up_offset = g.up_offset;
  p.m_valid = g.m_valid;
  p.out = g.out;
  p.ld_out = g.ld_out;
  p.status = g.status;
  for (int i = 0; i < 2; ++i) {
    p.wsf[i] = g.wsf[i];
    p.wsc[i] = g.wsc[i];
    p.tsf[i] = g.tsf[i];
    p.tsf_ld[i] = g.tsf_ld[i];
    p.tsf_rows[i] = g.tsf_rows[i];
  }
  p.wsf_rb_per_group = g.wsf_rb_per_group;
  p.out_sf = g.out_sf;
  p.ld_out_sf = g.ld_out_sf;
  for (int i = 0; i < 2; ++i) {
    p.gsrc[i] = static_cast<const uint8_t*>(g.gsrc[i]);
    p.gidx[i] = g.gidx[i];
  }
  p.g_ld = g.g_ld;
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, NTW, GATHER>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::kSmemBytes));
  if (err != cudaSuccess) return err;
  int grid = g.num_sms;
  if (MODE == kRouter) {
    const int tiles = ((g.router_T + kChunkRows - 1) / kChunkRows) * g.n_mblk * p.k_splits;
    if (tiles < grid) grid = tiles;
    if (grid == 0) return cudaSuccess;
  }
  grouped_gemm_kernel<MODE, NTW, GATHER><<<grid, C::kThreads, C::kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

template <int MODE, int NT>
static cudaError_t launch_fs(const GemmLaunch& g, cudaStream_t s) {
  using C = CfgFS<MODE, NT>;
  DevParams p;
  for (int i = 0; i < 2; ++i) p.wmap[i] = g.wmap[i];
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < kTokBoxes; ++j) p.tmap[i][j] = g.tmap[i][j];
  p.chunks = g.chunks;
  p.n_chunks = g.n_chunks;
  p.grp_cp = g.grp_cp;
  p.n_grp = g.n_grp;
  p.halves = 0;
  p.router_T = 0;
  p.n_mblk = g.n_mblk;
  p.k_blocks = g.k_blocks;
  p.k_splits = 1;
  p.k_per_split = g.k_blocks;
  p.split_stride = 0;
  p.w_rows_per_group = g.w_rows_per_group;
  p.up_offset = g.up_offset;
  p.m_valid = g.m_valid;
  p.out = g.out;
  p.ld_out = g.ld_out;
  p.status = g.status;
  p.wsf_rb_per_group = g.wsf_rb_per_group;
  p.out_sf = g.out_sf;
  p.ld_out_sf = g.ld_out_sf;
  for (int i = 0; i < 2; ++i) {
    p.tsf[i] = g.tsf[i];
    p.tsf_ld[i] = g.tsf_ld[i];
    p.tsf_rows[i] = g.tsf_rows[i];
    p.fs_a[i] = g.fs_a[i];
    p.fs_w[i] = g.fs_w[i];
  }
  p.fs_a_ld = g.fs_a_ld;
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_fs_kernel<MODE, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(C::kSmemBytes));
  if (err != cudaSuccess) return err;
  grouped_gemm_fs_kernel<MODE, NT><<<g.num_sms, C::kThreads, C::kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t s) {
  switch (g.mode) {
    // fp32-scale GEMMs: 32-token tiles on decode-sized batches, else 64
    case kFFN1X:
      return g.tile_tokens == 2 * kChunkRowsNarrow ? launch_fs<kFFN1X, 2 * kChunkRowsNarrow>(g, s)
                                                   : launch_fs<kFFN1X, kChunkRowsNarrow>(g, s);
    case kFFN2X:
      return g.tile_tokens == 2 * kChunkRowsNarrow ? launch_fs<kFFN2X, 2 * kChunkRowsNarrow>(g, s)
                                                   : launch_fs<kFFN2X, kChunkRowsNarrow>(g, s);
    case kFFN2XM256:
      return g.tile_tokens == 2 * kChunkRowsNarrow ? launch_fs<kFFN2XM256, 2 * kChunkRowsNarrow>(g, s)
                                                   : launch_fs<kFFN2XM256, kChunkRowsNarrow>(g, s);
    case kRouter: return launch_mode<kRouter, kChunkRows>(g, s);
    case kFFN1:
      if (g.tile_tokens == kChunkRowsNarrow) return launch_mode<kFFN1, kChunkRowsNarrow>(g, s);
      return launch_mode<kFFN1, kChunkRows>(g, s);
    case kFFN2M256:
      if (g.tile_tokens == kChunkRowsNarrow) return launch_mode<kFFN2M256, kChunkRowsNarrow>(g, s);
      return launch_mode<kFFN2M256, kChunkRows>(g, s);
    case kFFN2M512: return launch_mode<kFFN2M512, kChunkRowsNarrow>(g, s);
    case kFFN2:   // d_model not a multiple of 256: one 128-row weight block per tile
      if (g.tile_tokens == kChunkRowsNarrow) return launch_mode<kFFN2, kChunkRowsNarrow>(g, s);
      return launch_mode<kFFN2, kChunkRowsWide>(g, s);
    // FP8 / FP4-weight tiles: 32 tokens (decode-sized batches), else 112 (kChunkRows maps to
    // kChunkRowsFP8); the second GEMM takes 224-token tiles once chunks are 224 rows
    case kFFN1F8:
      if (g.tile_tokens == kChunkRowsNarrow) return launch_mode<kFFN1F8, kChunkRowsNarrow>(g, s);
      if (g.gather) return launch_mode<kFFN1F8, kChunkRows, true>(g, s);
      return launch_mode<kFFN1F8, kChunkRows>(g, s);
    case kFFN2F8:
      if (g.tile_tokens == kChunkRowsNarrow) return launch_mode<kFFN2F8, kChunkRowsNarrow>(g, s);
      if (g.tile_tokens == 2 * kChunkRowsFP8) return launch_mode<kFFN2F8, 2 * kChunkRowsFP8>(g, s);
      return launch_mode<kFFN2F8, kChunkRows>(g, s);
    case kFFN2F8M256: return launch_mode<kFFN2F8M256, kChunkRowsNarrow>(g, s);
    case kFFN2F4M256: return launch_mode<kFFN2F4M256, kChunkRowsNarrow>(g, s);
    case kFFN1F4:
      if (g.tile_tokens == kChunkRowsNarrow) return launch_mode<kFFN1F4, kChunkRowsNarrow>(g, s);
      if (g.gather) return launch_mode<kFFN1F4, kChunkRows, true>(g, s);
      return launch_mode<kFFN1F4, kChunkRows>(g, s);
    case kFFN2F4:
      if (g.tile_tokens == kChunkRowsNarrow) return launch_mode<kFFN2F4, kChunkRowsNarrow>(g, s);
      if (g.tile_tokens == 2 * kChunkRowsFP8) return launch_mode<kFFN2F4, 2 * kChunkRowsFP8>(g, s);
      return launch_mode<kFFN2F4, kChunkRows>(g, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
