// Block-scaled FP8 GEMM for sm_100a: Y[m, n] = bf16( sum_kb sa[m, kb] *
// sw[n/128, kb] * sum_{k in kb} Xq[m, k] * Wq[n, k] ), the fine-grained FP8
// linear layer ("Fine-grained FP8", introduction: 1x128 activation groups and
// 128x128 weight blocks; "UE8M0 scale format" for power-of-two scales).
//
// One CTA computes a 128 x BN output tile (BN = 128 or 256):
//   warp 0      TMA producer: per 128-wide K block, one 128x128 tile of Xq
//               and one BNx128 tile of Wq (128-byte swizzle) into a ring of
//               kStages shared-memory slots;
//   warp 1      owns TMEM and issues tcgen05.mma (kind::f8f6f4, E4M3 x E4M3
//               -> fp32), four K=32 steps per K block, into one of two TMEM
//               partial buffers (ping-pong), then commits once to the slot's
//               "empty" barrier, which also tells the promotion warps that
//               the block's partial is in TMEM;
//   warps 4..   promotion: each thread owns one output row and CW columns; it
//               loads the block partial from TMEM, multiplies by the product
//               of the two block scales and accumulates in fp32 registers
//               (packed fp32x2 FMAs), so the MMA of block kb+1 overlaps the
//               promotion of block kb.
// After the last K block each thread rounds its 128 accumulators to bf16
// (round-to-nearest-even) and stores them.
//
// Grouped variant (M-grouped MoE experts): rows of Xq are laid out per expert
// in contiguous segments whose lengths are multiples of 128, so every 128-row
// tile belongs to one expert e, found from group_offs; its B tile comes from
// rows e*N + n of the stacked [E*N, K] weight tensor and its weight scales
// from Ws[e].
//
// Every barrier wait is bounded: on expiry the CTA records a status code,
// stops issuing work, waits (bounded) for its own outstanding TMA copies and
// MMAs, frees TMEM and exits.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "quant.cuh"

namespace fgfp8 {

// Self-test of the bounded waits: one thread waits on an mbarrier that
// nothing completes.  The wait gives up after its limit, the status word
// records it and the kernel exits, so the context stays usable.
__global__ void selftest_expired_wait_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    if (!mbar_wait(&bar, 0)) record_status(kDevTimeoutSelftest);
  }
}

// Tile configuration of the dense / grouped kernel.  BN: output columns per
// tile; CW: columns per promotion warp (each warp owns 32 rows x CW columns).
template <int BN, int CW>
struct GemmCfg {
  static constexpr int kBM = 128;
  static constexpr int kBK = 128;
  static constexpr int kEpiWarps = 4 * (BN / CW);
  static constexpr int kThreads = 128 + kEpiWarps * 32;          // warpgroup 0: producer, MMA, 2 idle
  static constexpr int kNumBuf = (512 / BN) > 4 ? 4 : (512 / BN);  // TMEM partial buffers
  static constexpr uint32_t kTmemCols = kNumBuf * BN;
  static constexpr uint32_t kABytes = kBM * kBK;
  static constexpr uint32_t kBBytes = BN * kBK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  // Epilogue staging: each promotion warp transposes its 32 rows x 64
  // columns of bf16 (4 KB) per pass through its own slot.
  static constexpr uint32_t kWarpStageBytes = 32 * 128;
  static constexpr uint32_t kStagingBytes = kEpiWarps * kWarpStageBytes;
  static constexpr int kStages = (224 * 1024 - kStagingBytes) / kStageBytes;  // 6 (BN=128) or 4 (BN=256)
  static constexpr size_t kBarrierBytes = 256;
  static constexpr size_t kSmemBytes =
      1024 + kStages * static_cast<size_t>(kStageBytes) + kStagingBytes + kBarrierBytes;
  // The promotion warps need more than an even share of the register file
  // (CW fp32 accumulators per thread): warpgroup 0 gives registers back
  // (setmaxnreg.dec) to the promotion warpgroups (setmaxnreg.inc).  The
  // shares must sum to no more than the launch allocation (threads x the
  // kernel's register count); the host checks the compiled count before the
  // first launch.  384 threads x 168 = 128 x 24 + 256 x 240;
  // 640 threads x 96 >= 128 x 24 + 512 x 112.
  static constexpr int kLaunchRegs = (65536 / kThreads) & ~7;
  static constexpr bool kRegSplit = true;
  static constexpr int kRegsLow = 24;
  static constexpr int kRegsHigh = ((kThreads * kLaunchRegs - 128 * kRegsLow) / (kThreads - 128)) & ~7;
};

template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Block scales travel as raw 32-bit words (fp32 bits, or a UE8M0 byte) from
// their load until the K block that uses them, so the loads can be issued
// several K blocks ahead without stalling on them; combine_raw then forms
// sa[m, kb] * sw[nb, kb]: an fp32 product, or for UE8M0 exponent bytes
// 2^(ea-127) * 2^(eb-127) = 2^(ea+eb-254) built exactly from the biased
// exponent ea+eb-127 (ldexpf when that leaves the normal range).  A 0xFF
// (NaN) scale byte gives an unspecified product.
template <int FMT>
__device__ __forceinline__ uint32_t load_scale_raw(const void* __restrict__ p, uint64_t i) {
  if (FMT == 0) return __float_as_uint(__ldg(reinterpret_cast<const float*>(p) + i));
  return __ldg(reinterpret_cast<const uint8_t*>(p) + i);
}

template <int FMT>
__device__ __forceinline__ float combine_raw(uint32_t a, uint32_t w) {
  if (FMT == 0) return __uint_as_float(a) * __uint_as_float(w);
  const int e = static_cast<int>(a) + static_cast<int>(w) - 127;
  if (e >= 1 && e <= 254) return __int_as_float(e << 23);
  return ldexpf(1.0f, static_cast<int>(a) + static_cast<int>(w) - 254);
}

// Depth (in K blocks) of the scale prefetch ring of the promotion warps.
constexpr int kScaleAhead = 2;

// Dense tile f -> (M tile, N tile) in bands of group_m M tiles: within a
// band the M index runs fastest, then N; the bands follow each other.  A
// wave then covers about group_m M tiles x (wave / group_m) N tiles, so the
// activation and weight tiles it touches stay L2-resident together.  With
// group_m >= num_m this is the plain M-fastest order (the whole activation
// matrix resident while every weight tile is read once).
__device__ __forceinline__ void grouped_tile(int f, int num_m, int num_n, int group_m, int& mi, int& ni) {
  const int band_tiles = group_m * num_n;
  const int band = f / band_tiles;
  const int r = f - band * band_tiles;
  const int rows = min(group_m, num_m - band * group_m);
  mi = band * group_m + r % rows;
  ni = r / rows;
}

// Expert owning row m: the e with offs[e] <= m < offs[e+1] (binary search),
// or -1 when the offsets are inconsistent with m.
__device__ __forceinline__ int find_expert(const int32_t* __restrict__ offs, int E, int m) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offs + mid) <= m) lo = mid;
    else hi = mid - 1;
  }
  if (__ldg(offs + lo) <= m && m < __ldg(offs + lo + 1)) return lo;
  return -1;
}

// Masked expert layout (cap > 0): expert e owns rows [e * cap, e * cap + cap);
// its first counts[e] rows hold tokens and the rest are padding.  Returns the
// expert of the M tile starting at row m0 (cap is a multiple of the tile
// height, so a tile never straddles experts) and sets row_end to the end of
// its token rows; -2 marks a tile of padding rows only (skipped, not an
// error), -1 a count outside [0, cap] (skipped and recorded).
__device__ __forceinline__ int masked_expert(const int32_t* __restrict__ counts, int E, int cap, int m0,
                                             int& row_end) {
  const int e = m0 / cap;
  if (e >= E) return -1;
  const int cnt = __ldg(counts + e);
  if (cnt < 0 || cnt > cap) return -1;
  row_end = e * cap + cnt;
  return m0 < row_end ? e : -2;
}

// ---------------------------------------------------------------------------
// Pipeline roles shared by the GEMM kernels.
// ---------------------------------------------------------------------------

// TMA producer (one thread): per K block, a kABytes tile of operand A (rows
// a_row.., box from tmA) and a kBBytes tile of operand B into ring slot
// kb % kStages; waits for the slot to be released by the MMA first.  With
// early_a, the A tiles of the first kStages K blocks are requested before the
// wait for the preceding grid (A must not be written by it); every other
// load follows that wait.  Before returning it waits for every copy it
// issued to land.
template <int kStages, uint32_t kABytes, uint32_t kBBytes>
__device__ __forceinline__ void produce_tiles(const CUtensorMap* tmA, int a_row, const CUtensorMap* tmB, int b_row,
                                              int KB, uint8_t* sA, uint8_t* sB, uint64_t* full, uint64_t* empty,
                                              bool early_a) {
  const int pre = early_a ? (KB < kStages ? KB : kStages) : 0;
  for (int kb = 0; kb < pre; ++kb) {
    mbar_arrive_expect_tx(&full[kb], kABytes + kBBytes);
    tma_load_2d(sA + kb * kABytes, tmA, &full[kb], kb * 128, a_row);
  }
  griddep_wait();
  int issued = 0;
  for (int kb = 0; kb < KB; ++kb) {
    const int s = kb % kStages;
    const uint32_t use = kb / kStages;
    if (kb >= kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u)) {
      record_status(kDevTimeoutProducer);
      break;
    }
    if (kb >= pre) {
      mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
      tma_load_2d(sA + s * kABytes, tmA, &full[s], kb * 128, a_row);
    }
    tma_load_2d(sB + s * kBBytes, tmB, &full[s], kb * 128, b_row);
    issued = kb + 1;
  }
  for (int kb = (issued > kStages ? issued - kStages : 0); kb < issued; ++kb) {
    if (!mbar_wait(&full[kb % kStages], (kb / kStages) & 1u)) record_status(kDevTimeoutProducer);
  }
}

// MMA issuer (one thread): per K block, four K=32 tcgen05.mma (M=128, N=kN)
// into TMEM partial buffer kb % kNumBuf (columns [b*kN, b*kN + kN)),
// overwriting it on the first step; then frees the smem slot and publishes
// the buffer.  A buffer is reused only after the promotion warps released it.
// A final commit makes every MMA complete before the caller may free TMEM.
template <int kStages, uint32_t kABytes, uint32_t kBBytes, int kN, int kNumBuf>
__device__ __forceinline__ void issue_mmas(uint32_t a_base, uint32_t b_base, int KB, uint32_t tmem_base,
                                           uint64_t* full, uint64_t* empty, uint64_t* tfull, uint64_t* tempty,
                                           uint64_t* mma_done) {
  constexpr uint32_t idesc = idesc_e4m3_f32(128, kN);
  const uint64_t a_desc0 = smem_desc_k_sw128(a_base), b_desc0 = smem_desc_k_sw128(b_base);
  for (int kb = 0; kb < KB; ++kb) {
    const int s = kb % kStages;
    const int b = kb % kNumBuf;
    if (!mbar_wait(&full[s], (kb / kStages) & 1u)) {
      record_status(kDevTimeoutMma);
      break;
    }
    if (kb >= kNumBuf && !mbar_wait(&tempty[b], ((kb / kNumBuf) & 1u) ^ 1u)) {
      record_status(kDevTimeoutMma);
      break;
    }
    tc_fence_after();
    const uint32_t d = tmem_base + static_cast<uint32_t>(b * kN);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t ad = a_desc0 + ((s * kABytes + kk * 32) >> 4);
      const uint64_t bd = b_desc0 + ((s * kBBytes + kk * 32) >> 4);
      mma_f8f6f4(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
    mma_commit(&empty[s]);
    mma_commit(&tfull[b]);
  }
  mma_commit(mma_done);
  if (!mbar_wait(mma_done, 0)) record_status(kDevTimeoutMma);
}

// Dense 128 x 256 tiles may end with half tiles: work items t >= num_full
// split the remaining full tiles f = num_full + (t - num_full) / 2 into two
// 128 x 128 halves, loaded through tmBh (a 128-row box of the same weights)
// and promoted by all promotion warps at CW/2 columns each.  The host uses
// them when the last partial wave of full tiles fits twice into one wave, so
// that wave takes about half as long.
//
// kFuse (dense, fp32 scales, 128 x 256 tiles): the SwiGLU MLP's gate/up
// projection fused with the down projection's activation quantizer.  The
// weight holds gate and up rows interleaved in 128-row blocks (rows
// [256 j, 256 j + 128) are gate rows 128 j.., the next 128 the up rows), so a
// tile's columns [0, 128) are gate and [128, 256) up outputs for the
// intermediate indices i0 = n0 / 2 .. i0 + 127.  Instead of Y the epilogue
// writes the codes Hq [M, I] and MN-major scales Hs[(i0 / 128) * ld_h + m]
// of h = SiLU(gate) * up: the up warp of each TMEM lane quadrant hands its
// bf16 outputs to the gate warp through shared memory, and the gate warp's
// thread then holds one token's whole 1 x 128 group of h.
template <int BN, int CW, int FMT, bool kGrouped, bool kFuse = false>
__global__ void __launch_bounds__(GemmCfg<BN, CW>::kThreads, 1)
    gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmBh, const void* __restrict__ Xs, uint32_t ld_s,
                            const void* __restrict__ Ws, __nv_bfloat16* __restrict__ Y, int M, int N, int K,
                            const int32_t* __restrict__ group_offs, int E, int cap, int num_tiles, int num_full,
                            int early_b, uint8_t* __restrict__ Hq, float* __restrict__ Hs, uint32_t ld_h,
                            int withhold_kb, int group_m) {
  using C = GemmCfg<BN, CW>;
  static_assert(!kFuse || (BN == 256 && CW == 128 && FMT == 0 && !kGrouped), "fused SwiGLU: dense fp32 256-wide");
  static_assert(C::kStages > C::kNumBuf, "the promotion waits on the stage barriers (see the promotion loop)");
  static_assert((2 * C::kStages + C::kNumBuf + 1 + 8) * 8 + 4 <= C::kBarrierBytes, "barrier area");
  constexpr bool kHalfTiles = !kGrouped && BN == 256 && !kFuse;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint8_t* sStg = sB + C::kStages * C::kBBytes;       // epilogue staging, one slot per promotion warp
  uint64_t* full = reinterpret_cast<uint64_t*>(sStg + C::kStagingBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tempty = empty + C::kStages;
  uint64_t* mma_done = tempty + C::kNumBuf;
  uint64_t* xfull = mma_done + 1;                     // fused epilogue: halves exchanged, per quadrant
  uint64_t* xempty = xfull + 4;                       // fused epilogue: half-row amax exchanged, per quadrant
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xempty + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = K / C::kBK;
  const int NB = N / 128;
  const int num_m = (M + C::kBM - 1) / C::kBM;
  const int num_n = N / BN;

  // Work item t -> (m0, n0, expert, half, row_end).  Dense tiles run
  // M-fastest (the activation tile set stays L2-resident while a weight tile
  // is reused); grouped tiles run N-fastest (the CTAs of one expert share its
  // weights in L2).  Grouped rows come either as contiguous expert segments
  // (group_offs, cap == 0) or in the masked layout (per-expert counts in
  // group_offs, cap > 0).  An expert of -1 marks a tile whose rows no segment
  // covers (every role skips it and the status word records it), -2 a
  // masked tile of padding rows only (skipped).  Rows >= row_end of a tile
  // are not stored.
  auto coords = [&](int t, int& m0, int& n0, int& expert, bool& half, int& row_end) {
    half = false;
    row_end = M;
    if (!kGrouped) {
      int f = t, h = 0;
      if (kHalfTiles && t >= num_full) {
        f = num_full + ((t - num_full) >> 1);
        h = (t - num_full) & 1;
        half = true;
      }
      int mi, ni;
      grouped_tile(f, num_m, num_n, group_m, mi, ni);
      m0 = mi * C::kBM;
      n0 = ni * BN + h * (BN / 2);
      expert = 0;
    } else {
      n0 = (t % num_n) * BN;
      m0 = (t / num_n) * C::kBM;
      expert = cap > 0 ? masked_expert(group_offs, E, cap, m0, row_end) : find_expert(group_offs, E, m0);
    }
    FGFP8_DCHECK(t >= 0 && t < num_tiles && m0 >= 0 && m0 < M && n0 >= 0 && n0 + (half ? BN / 2 : BN) <= N &&
                 expert >= -2 && expert < (kGrouped ? E : 1) && row_end <= M);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kNumBuf; ++b) mbar_init(&tempty[b], C::kEpiWarps);
    mbar_init(mma_done, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&xfull[q], 64);                       // both warps of the quadrant's pair
      mbar_init(&xempty[q], 64);
    }
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (kHalfTiles) tma_prefetch_desc(&tmBh);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Dependency on the preceding grid (programmatic launch): the producer may
  // request the first weight tiles before it; every other access follows it.
  if (threadIdx.x != 0) griddep_wait();

  if (warp < 4) {
    if (C::kRegSplit) setmaxnreg_dec<C::kRegsLow>();
    if (warp == 0 && lane == 0) {
      // ================= TMA producer
      // early_b (dense): the weight tiles of the first tile's first kStages K
      // blocks are requested before the wait (the weights must not be
      // written by the preceding grid).
      int pre = 0;
      bool half0 = true;
      int m0p = 0, n0p = 0, ep = 0, rep_end = 0;
      if (static_cast<int>(blockIdx.x) < num_tiles) coords(blockIdx.x, m0p, n0p, ep, half0, rep_end);
      if (!kGrouped && early_b && static_cast<int>(blockIdx.x) < num_tiles && !half0) {
        const int n0 = n0p;
        pre = KB < C::kStages ? KB : C::kStages;
        for (int kb = 0; kb < pre; ++kb) {
          mbar_arrive_expect_tx(&full[kb], C::kStageBytes);
          tma_load_2d(sB + kb * C::kBBytes, &tmB, &full[kb], kb * C::kBK, n0);
        }
      }
      griddep_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int m0, n0, expert, row_end;
        bool half;
        coords(t, m0, n0, expert, half, row_end);
        if (expert < 0) {
          if (expert == -1) record_status(kDevBadGroupOffsets);
          continue;
        }
        const int b_row = expert * N + n0;
        const CUtensorMap* mapB = (kHalfTiles && half) ? &tmBh : &tmB;
        const uint32_t stage_tx = (kHalfTiles && half) ? C::kABytes + C::kBBytes / 2 : C::kStageBytes;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kStages;
          if (it >= static_cast<uint32_t>(C::kStages) && !mbar_wait(&empty[s], ((it / C::kStages) & 1u) ^ 1u)) {
            record_status(kDevTimeoutProducer);
            ok = false;
            break;
          }
          // fault injection (self-test only, withhold_kb < 0 in every product
          // launch): work item 0 never requests K block withhold_kb, so the
          // MMA's wait for it expires and every role unwinds
          if (t == 0 && kb == withhold_kb) continue;
          if (it >= static_cast<uint32_t>(pre)) {
            mbar_arrive_expect_tx(&full[s], stage_tx);
            tma_load_2d(sB + s * C::kBBytes, mapB, &full[s], kb * C::kBK, b_row);
          }
          tma_load_2d(sA + s * C::kABytes, &tmA, &full[s], kb * C::kBK, m0);
        }
      }
      // every copy issued must land before the CTA may exit
      for (uint32_t j = (it > static_cast<uint32_t>(C::kStages) ? it - C::kStages : 0); j < it; ++j)
        if (!mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1u)) record_status(kDevTimeoutProducer);
    } else if (warp == 1 && lane == 0) {
      // ================= MMA issuer
      constexpr uint32_t idesc_full = idesc_e4m3_f32(128, BN);
      constexpr uint32_t idesc_half = idesc_e4m3_f32(128, BN / 2);
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      // descriptors differ per stage / K step only in the start-address field
      const uint64_t a_desc0 = smem_desc_k_sw128(a_base), b_desc0 = smem_desc_k_sw128(b_base);
      uint32_t it = 0, bt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int m0, n0, expert, row_end;
        bool half;
        coords(t, m0, n0, expert, half, row_end);
        if (expert < 0) continue;
        const uint32_t idesc = (kHalfTiles && half) ? idesc_half : idesc_full;
        for (int kb = 0; kb < KB; ++kb, ++it, ++bt) {
          const int s = it % C::kStages;
          const int buf = bt % C::kNumBuf;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1u)) {
            record_status(kDevTimeoutMma);
            ok = false;
            break;
          }
          if (bt >= static_cast<uint32_t>(C::kNumBuf) &&
              !mbar_wait(&tempty[buf], ((bt / C::kNumBuf) & 1u) ^ 1u)) {
            record_status(kDevTimeoutMma);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = a_desc0 + ((s * C::kABytes + kk * 32) >> 4);
            const uint64_t bd = b_desc0 + ((s * C::kBBytes + kk * 32) >> 4);
            mma_f8f6f4(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          // one commit per K block: the stage's "empty" barrier also tells
          // the promotion warps that the partial of this K block is in TMEM
          mma_commit(&empty[s]);
        }
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) record_status(kDevTimeoutMma);
    }
  } else {
    if (C::kRegSplit) setmaxnreg_inc<C::kRegsHigh>();
    // ================= promotion / epilogue
    const int ew = warp - 4;
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int grp = ew >> 2;                   // column group: columns [grp * cols, grp * cols + cols)
    const int row = quad * 32 + lane;
    // raw scale words for K blocks kb .. kb+kScaleAhead-1, ring slot kb % kScaleAhead
    uint32_t ra[kScaleAhead], rw[kScaleAhead];
    auto fetch = [&](int kb, int m, bool live, uint64_t ws_row, uint32_t& a, uint32_t& w) {
      if (live && kb < KB) {
        a = load_scale_raw<FMT>(Xs, static_cast<uint64_t>(kb) * ld_s + m);
        w = load_scale_raw<FMT>(Ws, ws_row + kb);
      } else {
        a = 0u;
        w = 0u;
      }
    };
    // This thread's row, first column, liveness and weight-scale row in work
    // item t (expert < 0: skipped tile).  A warp covers CW columns of a full
    // tile, CW/2 of a half tile; either way they lie in one 128-column
    // weight block.
    auto tile_rows = [&](int t, int& m0, int& n0, int& expert, bool& half, int& col0, int& m, bool& live,
                         uint64_t& ws_row, int& row_end) {
      coords(t, m0, n0, expert, half, row_end);
      col0 = grp * ((kHalfTiles && half) ? CW / 2 : CW);
      m = m0 + row;
      live = (m < row_end) && (n0 + col0 < N);
      ws_row = (static_cast<uint64_t>(expert < 0 ? 0 : expert) * NB + (n0 + col0) / 128) * KB;
    };
    int pref_t = -1;                           // tile whose first scale words are in the ring
    uint32_t bt = 0;
    uint32_t xt = 0;                           // fused epilogue: tiles handed over so far
    bool ok = true;

    // Fused SwiGLU epilogue (kFuse).  The gate warp (grp 0) and the up warp
    // (grp 1) of quadrant `quad` hold the same 32 rows: gate columns and up
    // columns of the same 128 intermediate indices.  They split the work by
    // halves: the gate warp sends g for columns 64..127 and the up warp u for
    // columns 0..63 through the quadrant's shared-memory region (bf16, 16-byte
    // chunk c of lane l at position c ^ (l % 8)), each forms h = bf16(silu(g)
    // * u) for its 64 columns with g, u the bf16-rounded outputs and silu(g) =
    // g / (1 + exp(-g)) in fp32 (hardware exponential and divide, a few fp32
    // ulps), the two half-row amax values meet through the region, and each
    // warp quantizes its 64 values with the row's scale exactly as the
    // activation quantizer does.  Both meetings are bounded mbarrier waits on
    // which all 64 lanes of the pair arrive.
    auto fused_swiglu_epilogue = [&](float2 (&acc2)[CW / 2], int m0, int n0) {
      uint8_t* region = sStg + quad * 8192;       // [0, 4 KB): g half, [4, 8 KB): u half
      const uint32_t par = xt & 1u;
      // kGate: this is the gate warp (keeps columns 0..63, sends g of 64..127)
      // or the up warp (keeps 64..127, sends u of 0..63).  Once read, the
      // partner's half carries this warp's half-row amax (slot = lane).
      auto run = [&](auto gate_tag) -> bool {
        constexpr bool kGate = decltype(gate_tag)::value;
        constexpr int kSend0 = kGate ? 32 : 0, kOwn0 = kGate ? 0 : 32;
        uint8_t* out = region + (kGate ? 0 : 4096);
        uint8_t* in = region + (kGate ? 4096 : 0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v;
          uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            __nv_bfloat162 b = __floats2bfloat162_rn(acc2[kSend0 + 4 * c + q].x, acc2[kSend0 + 4 * c + q].y);
            w[q] = *reinterpret_cast<uint32_t*>(&b);
          }
          *reinterpret_cast<uint4*>(out + lane * 128 + ((c ^ (lane & 7)) << 4)) = v;
        }
        mbar_arrive(&xfull[quad]);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&xfull[quad], par))) return false;
        uint32_t hw[32];                           // h of my 64 columns as bf16 pairs
        uint32_t a2 = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(in + lane * 128 + ((c ^ (lane & 7)) << 4));
          const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float p0 = __uint_as_float(w[q] << 16), p1 = __uint_as_float(w[q] & 0xFFFF0000u);
            const float o0 = __bfloat162float(__float2bfloat16_rn(acc2[kOwn0 + 4 * c + q].x));
            const float o1 = __bfloat162float(__float2bfloat16_rn(acc2[kOwn0 + 4 * c + q].y));
            const float g0 = kGate ? o0 : p0, g1 = kGate ? o1 : p1;
            const float u0 = kGate ? p0 : o0, u1 = kGate ? p1 : o1;
            const float s0 = __fdividef(g0, __fadd_rn(1.0f, __expf(-g0)));
            const float s1 = __fdividef(g1, __fadd_rn(1.0f, __expf(-g1)));
            __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(s0, u0), __fmul_rn(s1, u1));
            hw[4 * c + q] = *reinterpret_cast<uint32_t*>(&h);
            a2 = __vmaxu2(a2, hw[4 * c + q] & 0x7FFF7FFFu);
          }
        }
        const uint32_t mine = max(a2 & 0xFFFFu, a2 >> 16);
        __syncwarp();                              // every lane has read its row of `in`
        reinterpret_cast<uint32_t*>(in)[lane] = mine;
        mbar_arrive(&xempty[quad]);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&xempty[quad], par))) return false;
        // the partner's half-row amax sits in the half this warp sent; its next
        // overwrite follows the next tile's first meeting
        const uint32_t amax = max(mine, reinterpret_cast<const uint32_t*>(out)[lane]);
        const int m = m0 + row;
        if (m < M) {
          const GroupScale gs = make_scale<0>(amax);
          const int i0 = n0 / 2;
          FGFP8_DCHECK(i0 + 128 <= N / 2 && m < M);
          uint8_t* dst = Hq + static_cast<uint64_t>(m) * (N / 2) + i0 + (kGate ? 0 : 64);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 o;
            o.x = quant4<0>(hw[8 * c + 0], hw[8 * c + 1], gs);
            o.y = quant4<0>(hw[8 * c + 2], hw[8 * c + 3], gs);
            o.z = quant4<0>(hw[8 * c + 4], hw[8 * c + 5], gs);
            o.w = quant4<0>(hw[8 * c + 6], hw[8 * c + 7], gs);
            *reinterpret_cast<uint4*>(dst + 16 * c) = o;
          }
          if (kGate) Hs[static_cast<uint64_t>(i0 / 128) * ld_h + m] = gs.s;
        }
        return true;
      };
      const bool done = (grp == 0) ? run(std::true_type{}) : run(std::false_type{});
      if (!done) {
        if (lane == 0) record_status(kDevTimeoutEpilogue);
        ok = false;
        return;
      }
      ++xt;
    };

    // One work item with COLS columns per warp: per K block, the partial from
    // TMEM times sa * sw into the accumulators, then the bf16 epilogue.
    auto promote = [&](auto cols_tag, int t, int m0, int n0, int col0, int m, bool live, uint64_t ws_row,
                       int row_end) {
      constexpr int COLS = decltype(cols_tag)::value;
      const uint32_t lane_base =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(col0);
      // fp32 accumulators as pairs: columns 2j, 2j+1 in acc2[j]
      float2 acc2[COLS / 2];
#pragma unroll
      for (int j = 0; j < COLS / 2; ++j) acc2[j] = make_float2(0.0f, 0.0f);
      for (int kb0 = 0; kb0 < KB && ok; kb0 += kScaleAhead) {
#pragma unroll
        for (int d = 0; d < kScaleAhead; ++d) {
          const int kb = kb0 + d;
          if (kb >= KB) break;
          const float sc = live ? combine_raw<FMT>(ra[d], rw[d]) : 0.0f;
          fetch(kb + kScaleAhead, m, live, ws_row, ra[d], rw[d]);
          const int buf = bt % C::kNumBuf;
          // The partial of K block bt is complete when the MMAs' commit to
          // stage bt % kStages lands (phase bt / kStages of its "empty"
          // barrier).  That barrier cannot run a phase ahead of this wait:
          // its next phase is the commit of K block bt + kStages, whose MMAs
          // need buffer (bt + kStages) % kNumBuf back from a later K block's
          // promotion (kStages > kNumBuf).  Warp-uniform outcome: the TMEM
          // loads below are .sync.aligned.
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[bt % C::kStages], (bt / C::kStages) & 1u))) {
            if (lane == 0) record_status(kDevTimeoutEpilogue);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = lane_base + static_cast<uint32_t>(buf * BN);
          // Two halves of COLS/2 columns, each one TMEM load round trip and
          // packed fp32x2 FMAs (fma.rn per element, as a scalar FMA).  The
          // buffer is handed back as soon as the second half is in
          // registers; that half's FMAs run while the next MMA fills it.
          constexpr int kHalf = COLS / 2;
          const float2 sc2 = make_float2(sc, sc);
          uint32_t p[kHalf];
          tmem_ld_cols<kHalf>(taddr, p);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < kHalf / 2; ++j)
            acc2[j] = __ffma2_rn(make_float2(__uint_as_float(p[2 * j]), __uint_as_float(p[2 * j + 1])), sc2, acc2[j]);
          tmem_ld_cols<kHalf>(taddr + kHalf, p);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
#pragma unroll
          for (int j = 0; j < kHalf / 2; ++j)
            acc2[kHalf / 2 + j] =
                __ffma2_rn(make_float2(__uint_as_float(p[2 * j]), __uint_as_float(p[2 * j + 1])), sc2, acc2[kHalf / 2 + j]);
          ++bt;
        }
      }
      if (!ok) return;

      // The next tile's first scale words: their latency overlaps the epilogue.
      pref_t = -1;
      if (t + static_cast<int>(gridDim.x) < num_tiles) {
        const int tn = t + static_cast<int>(gridDim.x);
        int m0n, n0n, en, c0n, mn, ren;
        bool hn, liven;
        uint64_t wsn;
        tile_rows(tn, m0n, n0n, en, hn, c0n, mn, liven, wsn, ren);
        if (en >= 0) {
#pragma unroll
          for (int d = 0; d < kScaleAhead; ++d) fetch(d, mn, liven, wsn, ra[d], rw[d]);
          pref_t = tn;
        }
      }

      if constexpr (kFuse) {
        if constexpr (COLS == CW) {
          fused_swiglu_epilogue(acc2, m0, n0);
          return;
        }
      }

      // Epilogue: bf16 (round-to-nearest-even), transposed through the warp's
      // shared-memory slot so that each store instruction writes four whole
      // 128-byte row segments.  Per 64-column pass, lane l writes its row's
      // eight 16-byte chunks (chunk c at position c ^ (l % 8): conflict-free),
      // then reads back row 4i + l / 8, chunk l % 8, for i = 0..7.
      uint8_t* slot = sStg + ew * C::kWarpStageBytes;
#pragma unroll
      for (int p = 0; p < COLS / 64; ++p) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int j = p * 64 + c * 8;
          uint4 v;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(acc2[j / 2 + 0].x, acc2[j / 2 + 0].y);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(acc2[j / 2 + 1].x, acc2[j / 2 + 1].y);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(acc2[j / 2 + 2].x, acc2[j / 2 + 2].y);
          __nv_bfloat162 h3 = __floats2bfloat162_rn(acc2[j / 2 + 3].x, acc2[j / 2 + 3].y);
          v.x = *reinterpret_cast<uint32_t*>(&h0);
          v.y = *reinterpret_cast<uint32_t*>(&h1);
          v.z = *reinterpret_cast<uint32_t*>(&h2);
          v.w = *reinterpret_cast<uint32_t*>(&h3);
          *reinterpret_cast<uint4*>(slot + lane * 128 + ((c ^ (lane & 7)) << 4)) = v;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + (lane >> 3), c = lane & 7;
          const uint4 v = *reinterpret_cast<const uint4*>(slot + r * 128 + ((c ^ (r & 7)) << 4));
          const int mr = m0 + quad * 32 + r;
          if (mr < row_end) {
            FGFP8_DCHECK(mr < M && n0 + col0 + p * 64 + c * 8 + 8 <= N);
            *reinterpret_cast<uint4*>(Y + static_cast<uint64_t>(mr) * N + n0 + col0 + p * 64 + c * 8) = v;
          }
        }
        __syncwarp();
      }
    };

    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      int m0, n0, expert, col0, m, row_end;
      bool half, live;
      uint64_t ws_row;
      tile_rows(t, m0, n0, expert, half, col0, m, live, ws_row, row_end);
      if (expert < 0) continue;
      if (pref_t != t) {
#pragma unroll
        for (int d = 0; d < kScaleAhead; ++d) fetch(d, m, live, ws_row, ra[d], rw[d]);
      }
      if constexpr (kHalfTiles) {
        if (half) {
          promote(std::integral_constant<int, CW / 2>{}, t, m0, n0, col0, m, live, ws_row, row_end);
          continue;
        }
      }
      promote(std::integral_constant<int, CW>{}, t, m0, n0, col0, m, live, ws_row, row_end);
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------------------
// UE8M0 variant with hardware block scaling ("UE8M0 scale format": scales are
// powers of two, which the tensor core can apply itself).  Per 128-wide K
// block the MMA takes one UE8M0 scale per row of Xq and one per row of Wq
// (the 128x128 weight block's scale, shared by its 128 rows) from TMEM
// (kind::mxf8f6f4.block_scale, one scale per 32-element K slice; the four
// slices of a 128 block use the same scale), so the whole K reduction
// accumulates in TMEM and no promotion step runs per K block.  The scales
// travel in groups of four K blocks: byte b of each 32-bit TMEM scale word
// belongs to K block 4g + b, and the MMAs of that block select it through
// the scale-factor ids of the instruction descriptor, so one copy into TMEM
// serves four K blocks.
//   warp 0      TMA for the operand tiles (lane 0);
//   warp 1      owns TMEM; per scale group tcgen05.cp of the group's slot
//               into TMEM, then per K block four block-scaled MMAs; after the
//               tile's last K block it publishes the accumulator.  The copies
//               stay on this thread: the tensor pipe runs them in issue order
//               with the MMAs, so no wait separates a copy from its MMAs;
//   warp 2      the scale words of two groups at a time written to
//               shared-memory slots in the TMEM scale layout (lane l: words
//               of rows l, l+32, l+64, l+96; a weight tile: its block's word
//               everywhere), one proxy fence per two groups, so the scale
//               loads never delay a TMA or MMA issue;
//   warps 4..   epilogue: TMEM -> registers -> bf16 -> global.
// TMEM: BN = 128: two accumulators in columns [0, 256); BN = 256: one in
// [0, 256).  Scale factors follow, two slots of 4 columns for A and BN / 32
// for B.
// ---------------------------------------------------------------------------
template <int BN>
struct MxCfg {
  static constexpr int kBM = 128, kBN = BN, kBK = 128;
  static constexpr int kEpiWarps = 4 * (BN / 128);                 // one warp per 32 rows x 128 columns
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  static constexpr int kNumAcc = (BN == 128) ? 2 : 1;             // accumulator buffers in TMEM
  static constexpr uint32_t kABytes = kBM * kBK;
  static constexpr uint32_t kBBytes = kBN * kBK;
  static constexpr uint32_t kSfABytes = 512;                      // 32 rows x 16 bytes (128 rows of A)
  static constexpr uint32_t kSfBBytes = 512 * (BN / 128);         // one 32 x 16 tile per 128 rows of B
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;      // TMA bytes per stage
  static constexpr int kStages = (BN == 128) ? 6 : 4;
  static constexpr int kSfGroup = 4;                              // K blocks per scale group (bytes of a word)
  static constexpr int kSfBatch = 2;                              // groups written per shared-memory fence
  static constexpr int kSfSlots = 2 * kSfBatch;                   // scale groups in flight
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSfCol = kNumAcc * BN;                // scale factors after the accumulators
  static constexpr uint32_t kSfColsPerSlot = 4 + BN / 32;         // A: 4 columns, B: BN/32 columns
  static constexpr size_t kBarrierBytes = 256;
  static constexpr size_t kSmemBytes = 1024 + kStages * static_cast<size_t>(kStageBytes) +
                                       kSfSlots * static_cast<size_t>(kSfABytes + kSfBBytes) + kBarrierBytes;
};

template <int BN, bool kGrouped>
__global__ void __launch_bounds__(MxCfg<BN>::kThreads, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmBh, const uint8_t* __restrict__ Xs, uint32_t ld_s,
                   const uint8_t* __restrict__ Ws, __nv_bfloat16* __restrict__ Y, int M, int N, int K,
                   const int32_t* __restrict__ group_offs, int E, int cap, int num_tiles, int num_full,
                   int early_b, int withhold_kb, int group_m) {
  using C = MxCfg<BN>;
  constexpr bool kHalfTiles = !kGrouped && BN == 256;
  static_assert(C::kSfCol + C::kSfSlots * C::kSfColsPerSlot <= C::kTmemCols, "TMEM columns");
  static_assert((2 * C::kStages + 4 + 1 + 2 * C::kSfSlots) * 8 + 4 <= C::kBarrierBytes, "barrier area");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::kStages * C::kABytes;
  uint8_t* sSfA = sB + C::kStages * C::kBBytes;
  uint8_t* sSfB = sSfA + C::kSfSlots * C::kSfABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSfB + C::kSfSlots * C::kSfBBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* sf_full = mma_done + 1;                  // a scale group written to its shared-memory slot
  uint64_t* sf_empty = sf_full + C::kSfSlots;        // the slot copied into TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + C::kSfSlots);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = K / C::kBK;
  const int NB = N / 128;
  const int num_m = (M + C::kBM - 1) / C::kBM;
  const int num_n = N / C::kBN;

  // as in the fp32-scale kernel: expert -1 = uncovered rows (recorded),
  // -2 = masked padding tile (skipped); rows >= row_end are not stored;
  // dense work items t >= num_full are 128 x 128 halves of the last full
  // tiles (half = true: a 128-row weight box, an N = 128 MMA)
  auto coords = [&](int t, int& m0, int& n0, int& expert, int& row_end, bool& half) {
    row_end = M;
    half = false;
    if (!kGrouped) {
      int f = t, h = 0;
      if (kHalfTiles && t >= num_full) {
        f = num_full + ((t - num_full) >> 1);
        h = (t - num_full) & 1;
        half = true;
      }
      int mi, ni;
      grouped_tile(f, num_m, num_n, group_m, mi, ni);
      m0 = mi * C::kBM;
      n0 = ni * C::kBN + h * (C::kBN / 2);
      expert = 0;
    } else {
      n0 = (t % num_n) * C::kBN;
      m0 = (t / num_n) * C::kBM;
      expert = cap > 0 ? masked_expert(group_offs, E, cap, m0, row_end) : find_expert(group_offs, E, m0);
    }
    FGFP8_DCHECK(t >= 0 && t < num_tiles && m0 >= 0 && m0 < M && n0 >= 0 &&
                 n0 + (half ? C::kBN / 2 : C::kBN) <= N && expert >= -2 && expert < (kGrouped ? E : 1) &&
                 row_end <= M);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::kEpiWarps);
    }
    for (int b = 0; b < C::kSfSlots; ++b) {
      mbar_init(&sf_full[b], 1);
      mbar_init(&sf_empty[b], 1);
    }
    mbar_init(mma_done, 1);
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (kHalfTiles) tma_prefetch_desc(&tmBh);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Dependency on the preceding grid (programmatic launch): the producer may
  // request the first weight tiles before it; every other access follows it.
  if (warp != 0) griddep_wait();

  if (warp == 0) {
    // ================= producer: TMA (lane 0)
    // early_b (dense): the weight tiles of the first tile's first kStages K
    // blocks are requested before the wait (the weights must not be written
    // by the preceding grid).
    if (lane == 0) {
      int pre = 0;
      bool half0 = true;
      int m0p = 0, n0p = 0, ep = 0, rep_end = 0;
      if (static_cast<int>(blockIdx.x) < num_tiles) coords(blockIdx.x, m0p, n0p, ep, rep_end, half0);
      if (!kGrouped && early_b && static_cast<int>(blockIdx.x) < num_tiles && !half0) {
        const int n0 = n0p;
        pre = KB < C::kStages ? KB : C::kStages;
        for (int kb = 0; kb < pre; ++kb) {
          mbar_arrive_expect_tx(&full[kb], C::kStageBytes);
          tma_load_2d(sB + kb * C::kBBytes, &tmB, &full[kb], kb * C::kBK, n0);
        }
      }
      griddep_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int m0, n0, expert, row_end;
        bool half;
        coords(t, m0, n0, expert, row_end, half);
        if (expert < 0) {
          if (expert == -1) record_status(kDevBadGroupOffsets);
          continue;
        }
        const CUtensorMap* mapB = (kHalfTiles && half) ? &tmBh : &tmB;
        const uint32_t stage_tx = (kHalfTiles && half) ? C::kABytes + C::kBBytes / 2 : C::kStageBytes;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kStages;
          if (it >= static_cast<uint32_t>(C::kStages) && !mbar_wait(&empty[s], ((it / C::kStages) & 1u) ^ 1u)) {
            record_status(kDevTimeoutProducer);
            ok = false;
            break;
          }
          if (t == 0 && kb == withhold_kb) continue;     // fault injection, as in the fp32-scale kernel
          if (it >= static_cast<uint32_t>(pre)) {
            mbar_arrive_expect_tx(&full[s], stage_tx);
            tma_load_2d(sB + s * C::kBBytes, mapB, &full[s], kb * C::kBK, expert * N + n0);
          }
          tma_load_2d(sA + s * C::kABytes, &tmA, &full[s], kb * C::kBK, m0);
        }
      }
      for (uint32_t j = (it > static_cast<uint32_t>(C::kStages) ? it - C::kStages : 0); j < it; ++j)
        if (!mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1u)) record_status(kDevTimeoutProducer);
    }
  } else if (warp == 2) {
    // ================= scale groups into shared memory (all lanes)
    uint32_t grp = 0;                          // scale groups issued so far
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      int m0, n0, expert, row_end;
      bool half;
      coords(t, m0, n0, expert, row_end, half);
      if (expert < 0) continue;
      const int nblk = (kHalfTiles && half) ? 1 : BN / 128;   // weight blocks the tile covers
      const uint64_t ws_row = (static_cast<uint64_t>(expert) * NB + n0 / 128) * KB;
      // Scale group g = K blocks 4g .. 4g+3, byte b of every word for K block
      // 4g + b: rows lane + 32 j of the tile's A rows (ra[.][j][b]) and the
      // scale of the tile's 128-row weight block h (rw[.][h][b]).  Groups go
      // out kSfBatch at a time (one proxy fence per batch); the raw bytes
      // are fetched one batch ahead and packed only when written.
      uint32_t ra[C::kSfBatch][4][C::kSfGroup], rw[C::kSfBatch][BN / 128][C::kSfGroup];
      auto fetch = [&](int g0) {
#pragma unroll
        for (int q = 0; q < C::kSfBatch; ++q) {
#pragma unroll
          for (int b = 0; b < C::kSfGroup; ++b) {
            const int kb = (g0 + q) * C::kSfGroup + b;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int m = m0 + lane + 32 * j;
              ra[q][j][b] = (kb < KB && m < row_end) ? __ldg(Xs + static_cast<uint64_t>(kb) * ld_s + m) : 127u;
            }
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              rw[q][h][b] = (kb < KB && h < nblk) ? __ldg(Ws + ws_row + static_cast<uint64_t>(h) * KB + kb) : 127u;
          }
        }
      };
      auto pack = [](const uint32_t (&v)[C::kSfGroup]) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < C::kSfGroup; ++b) word |= v[b] << (8 * b);
        return word;
      };
      const int groups = (KB + C::kSfGroup - 1) / C::kSfGroup;
      fetch(0);
      for (int g0 = 0; g0 < groups; g0 += C::kSfBatch) {
        const int nb = groups - g0 < C::kSfBatch ? groups - g0 : C::kSfBatch;
        // slot (grp + q) % kSfSlots is free once the copy of group
        // grp + q - kSfSlots is done
        bool free = true;
        for (int q = 0; q < nb; ++q) {
          const uint32_t gq = grp + q;
          free = free && (gq < static_cast<uint32_t>(C::kSfSlots) ||
                          mbar_wait(&sf_empty[gq % C::kSfSlots], ((gq / C::kSfSlots) & 1u) ^ 1u));
        }
        if (!__all_sync(0xFFFFFFFFu, free)) {
          if (lane == 0) record_status(kDevTimeoutProducer);
          ok = false;
          break;
        }
        // the TMEM scale layout: lane l holds rows l + 32 j (word j), a
        // weight tile its block's word in every position
#pragma unroll
        for (int q = 0; q < C::kSfBatch; ++q) {
          if (q < nb) {
            const int sl = static_cast<int>((grp + q) % C::kSfSlots);
            *reinterpret_cast<uint4*>(sSfA + sl * C::kSfABytes + lane * 16) =
                make_uint4(pack(ra[q][0]), pack(ra[q][1]), pack(ra[q][2]), pack(ra[q][3]));
#pragma unroll
            for (int h = 0; h < BN / 128; ++h) {
              const uint32_t w = pack(rw[q][h]);
              *reinterpret_cast<uint4*>(sSfB + sl * C::kSfBBytes + h * 512 + lane * 16) = make_uint4(w, w, w, w);
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
          for (int q = 0; q < nb; ++q) mbar_arrive(&sf_full[(grp + q) % C::kSfSlots]);
        grp += nb;
        fetch(g0 + C::kSfBatch);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= MMA issuer
      // K block kb reads byte kb % 4 of its group's scale words (scale
      // factor ids in the instruction descriptor: A bits 29-30, B bits 4-5)
      constexpr uint32_t idesc0 = idesc_mx_e4m3_ue8m0(128, C::kBN);
      constexpr uint32_t idesc_half = idesc_mx_e4m3_ue8m0(128, C::kBN / 2);
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      // descriptors differ per stage / K step only in the start-address field
      const uint64_t a_desc0 = smem_desc_k_sw128(a_base), b_desc0 = smem_desc_k_sw128(b_base);
      const uint64_t sfa_desc0 = smem_desc_rows16(smem_u32(sSfA)), sfb_desc0 = smem_desc_rows16(smem_u32(sSfB));
      uint32_t it = 0, grp = 0, tile_no = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int m0, n0, expert, row_end;
        bool half;
        coords(t, m0, n0, expert, row_end, half);
        if (expert < 0) continue;
        const uint32_t idesc_t = (kHalfTiles && half) ? idesc_half : idesc0;
        const int ab = tile_no % C::kNumAcc;            // accumulator buffer
        const int tb = tile_no & 1;                      // tfull / tempty barrier of this tile
        if (tile_no >= static_cast<uint32_t>(C::kNumAcc) &&
            !mbar_wait(&tempty[(tile_no - C::kNumAcc) & 1], ((tile_no - C::kNumAcc) >> 1) & 1u)) {
          record_status(kDevTimeoutMma);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(ab * C::kBN);
        // per scale group: its copy into TMEM slot grp % kSfSlots (in issue
        // order with the MMAs, which read the previous group's slot), then the
        // group's K blocks; K block kb reads byte kb % 4 of the scale words
        for (int kb0 = 0; kb0 < KB && ok; kb0 += C::kSfGroup, ++grp) {
          const int sl = static_cast<int>(grp % C::kSfSlots);
          if (!mbar_wait(&sf_full[sl], (grp / C::kSfSlots) & 1u)) {
            record_status(kDevTimeoutMma);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa = tmem_base + C::kSfCol + static_cast<uint32_t>(sl * C::kSfColsPerSlot);
          const uint32_t sfb = sfa + 4;
          tmem_cp_32x128b_x4(sfa, sfa_desc0 + ((sl * C::kSfABytes) >> 4));
#pragma unroll
          for (int h = 0; h < BN / 128; ++h)
            tmem_cp_32x128b_x4(sfb + 4 * h, sfb_desc0 + ((sl * C::kSfBBytes + h * 512) >> 4));
          mma_commit(&sf_empty[sl]);                     // the slot may be refilled once copied
          const int kb1 = kb0 + C::kSfGroup < KB ? kb0 + C::kSfGroup : KB;
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % C::kStages;
            if (!mbar_wait(&full[s], (it / C::kStages) & 1u)) {
              record_status(kDevTimeoutMma);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sf_id = static_cast<uint32_t>(kb - kb0);
            const uint32_t idesc = idesc_t | (sf_id << 29) | (sf_id << 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t adesc = a_desc0 + ((s * C::kABytes + kk * 32) >> 4);
              const uint64_t bdesc = b_desc0 + ((s * C::kBBytes + kk * 32) >> 4);
              mma_mxf8f6f4(d, adesc, bdesc, idesc, sfa, sfb, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
          }
        }
        if (ok) mma_commit(&tfull[tb]);
        ++tile_no;
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) record_status(kDevTimeoutMma);
    }
  } else if (warp >= 4) {
    // ================= epilogue: TMEM -> bf16 -> global
    const int ew = warp - 4;
    const int quad = warp & 3;
    const int col0 = (ew >> 2) * 128;
    const int row = quad * 32 + lane;
    uint32_t tile_no = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int m0, n0, expert, row_end;
      bool half;
      coords(t, m0, n0, expert, row_end, half);
      if (expert < 0) continue;
      const int ab = tile_no % C::kNumAcc;
      const int tb = tile_no & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[tb], (tile_no >> 1) & 1u))) {
        if (lane == 0) record_status(kDevTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      if (kHalfTiles && half && col0 >= C::kBN / 2) {
        // no columns of this half tile: hand the accumulator back at once
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[tb]);
        ++tile_no;
        continue;
      }
      const int m = m0 + row;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(ab * C::kBN + col0);
      FGFP8_DCHECK(m >= row_end || (m < M && n0 + col0 + 128 <= N));
      __nv_bfloat16* yrow = Y + static_cast<uint64_t>(m) * N + n0 + col0;
      // the whole 128-column slice into registers first, so the accumulator
      // is handed back to the MMA before the (slower) global stores
      uint32_t p[128];
#pragma unroll
      for (int h = 0; h < 128 / 32; ++h) tmem_ld_32x32b_x32(taddr + h * 32, *reinterpret_cast<uint32_t(*)[32]>(&p[h * 32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[tb]);
      if (m < row_end) {
#pragma unroll
        for (int j = 0; j < 128; j += 8) {
          uint4 v;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(p[j + 0]), __uint_as_float(p[j + 1]));
          __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(p[j + 2]), __uint_as_float(p[j + 3]));
          __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(p[j + 4]), __uint_as_float(p[j + 5]));
          __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(p[j + 6]), __uint_as_float(p[j + 7]));
          v.x = *reinterpret_cast<uint32_t*>(&h0);
          v.y = *reinterpret_cast<uint32_t*>(&h1);
          v.z = *reinterpret_cast<uint32_t*>(&h2);
          v.w = *reinterpret_cast<uint32_t*>(&h3);
          *reinterpret_cast<uint4*>(yrow + j) = v;
        }
      }
      ++tile_no;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------------------
// Row/column-scaled GEMM ("FP8 W8A8", "Applying quantization": the
// FP8_DYNAMIC scheme, per-output-channel weight scales and per-token
// activation scales; or one static scale for a whole tensor):
//   Y[m, n] = bf16( sx[m] * sw[n] * sum_k Xq[m, k] * Wq[n, k] )
// with sx[0] for every m when x_per_tensor, sw[0] for every n when
// w_per_tensor.  No scale changes along K, so the whole K reduction
// accumulates in TMEM and the scales are applied once, in the epilogue:
//   warp 0      TMA producer: one 128x128 Xq tile and one BNx128 Wq tile per
//               K block into a kStages ring (128-byte swizzle);
//   warp 1      TMEM owner and MMA issuer: four K=32 tcgen05.mma
//               (kind::f8f6f4) per K block into the tile's accumulator; two
//               accumulators, so one tile's epilogue overlaps the next tile's
//               MMAs;
//   warps 4..   epilogue: each thread one row and 128 columns; TMEM ->
//               registers, times sx[m] * sw[n] (an fp32 product, then an fp32
//               multiply), bf16 (round-to-nearest-even), global.
// ---------------------------------------------------------------------------
template <int BN>
struct RowColCfg {
  static constexpr int kBM = 128, kBN = BN, kBK = 128;
  static constexpr int kEpiWarps = 4 * (BN / 128);
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  static constexpr int kNumAcc = 2;
  static constexpr uint32_t kABytes = kBM * kBK;
  static constexpr uint32_t kBBytes = kBN * kBK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (BN == 128) ? 6 : 4;
  static constexpr uint32_t kTmemCols = kNumAcc * BN;
  static constexpr size_t kSmemBytes = 1024 + kStages * static_cast<size_t>(kStageBytes) + 256;
};

template <int BN>
__global__ void __launch_bounds__(RowColCfg<BN>::kThreads, 1)
    gemm_rowcol_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmBh, const float* __restrict__ sx, int x_per_tensor,
                       const float* __restrict__ sw, int w_per_tensor, __nv_bfloat16* __restrict__ Y, int M, int N,
                       int K, int num_tiles, int num_full, int group_m) {
  using C = RowColCfg<BN>;
  constexpr bool kHalfTiles = BN == 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::kStages * C::kBBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = K / C::kBK;
  const int num_m = (M + C::kBM - 1) / C::kBM;
  const int num_n = N / C::kBN;
  // work item t -> (m0, n0, half) in the banded order of grouped_tile; items
  // t >= num_full are the 128 x 128 halves of the remaining full tiles (as in
  // the fp32-scale kernel)
  auto coords = [&](int t, int& m0, int& n0, bool& half) {
    int f = t, h = 0;
    half = false;
    if (kHalfTiles && t >= num_full) {
      f = num_full + ((t - num_full) >> 1);
      h = (t - num_full) & 1;
      half = true;
    }
    int mi, ni;
    grouped_tile(f, num_m, num_n, group_m, mi, ni);
    m0 = mi * C::kBM;
    n0 = ni * C::kBN + h * (C::kBN / 2);
    FGFP8_DCHECK(t >= 0 && t < num_tiles && m0 >= 0 && m0 < M && n0 >= 0 && n0 + (half ? C::kBN / 2 : C::kBN) <= N);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::kEpiWarps);
    }
    mbar_init(mma_done, 1);
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (kHalfTiles) tma_prefetch_desc(&tmBh);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // programmatic launch: every access follows the preceding grid
  griddep_wait();

  if (warp == 0) {
    if (lane == 0) {
      // ================= TMA producer
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int m0, n0;
        bool half;
        coords(t, m0, n0, half);
        const CUtensorMap* mapB = (kHalfTiles && half) ? &tmBh : &tmB;
        const uint32_t stage_tx = (kHalfTiles && half) ? C::kABytes + C::kBBytes / 2 : C::kStageBytes;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kStages;
          if (it >= static_cast<uint32_t>(C::kStages) && !mbar_wait(&empty[s], ((it / C::kStages) & 1u) ^ 1u)) {
            record_status(kDevTimeoutProducer);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], stage_tx);
          tma_load_2d(sB + s * C::kBBytes, mapB, &full[s], kb * C::kBK, n0);
          tma_load_2d(sA + s * C::kABytes, &tmA, &full[s], kb * C::kBK, m0);
        }
      }
      // every copy issued must land before the CTA may exit
      for (uint32_t j = (it > static_cast<uint32_t>(C::kStages) ? it - C::kStages : 0); j < it; ++j)
        if (!mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1u)) record_status(kDevTimeoutProducer);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= MMA issuer
      constexpr uint32_t idesc_full = idesc_e4m3_f32(128, C::kBN);
      constexpr uint32_t idesc_half = idesc_e4m3_f32(128, C::kBN / 2);
      const uint64_t a_desc0 = smem_desc_k_sw128(smem_u32(sA)), b_desc0 = smem_desc_k_sw128(smem_u32(sB));
      uint32_t it = 0, tile_no = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tile_no) {
        int m0, n0;
        bool half;
        coords(t, m0, n0, half);
        const uint32_t idesc = (kHalfTiles && half) ? idesc_half : idesc_full;
        const int ab = tile_no & 1;                      // accumulator and its tfull / tempty barriers
        if (tile_no >= 2 && !mbar_wait(&tempty[ab], ((tile_no - 2) >> 1) & 1u)) {
          record_status(kDevTimeoutMma);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(ab * C::kBN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kStages;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1u)) {
            record_status(kDevTimeoutMma);
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = a_desc0 + ((s * C::kABytes + kk * 32) >> 4);
            const uint64_t bdesc = b_desc0 + ((s * C::kBBytes + kk * 32) >> 4);
            mma_f8f6f4(d, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&tfull[ab]);
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) record_status(kDevTimeoutMma);
    }
  } else if (warp >= 4) {
    // ================= epilogue: TMEM -> scales -> bf16 -> global
    const int ew = warp - 4;
    const int quad = warp & 3;
    const int col0 = (ew >> 2) * 128;
    const int row = quad * 32 + lane;
    uint32_t tile_no = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tile_no) {
      int m0, n0;
      bool half;
      coords(t, m0, n0, half);
      const int ab = tile_no & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[ab], (tile_no >> 1) & 1u))) {
        if (lane == 0) record_status(kDevTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      if (kHalfTiles && half && col0 >= C::kBN / 2) {
        // no columns of this half tile: hand the accumulator back at once
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[ab]);
        continue;
      }
      const int m = m0 + row;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(ab * C::kBN + col0);
      // the whole 128-column slice into registers, then the accumulator is
      // handed back before the scale multiplies and the stores
      uint32_t p[128];
#pragma unroll
      for (int h = 0; h < 4; ++h) tmem_ld_32x32b_x32(taddr + h * 32, *reinterpret_cast<uint32_t(*)[32]>(&p[h * 32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
      if (m < M) {
        const float a = __ldg(sx + (x_per_tensor ? 0 : m));
        const float w0 = w_per_tensor ? __ldg(sw) : 0.0f;
        FGFP8_DCHECK(n0 + col0 + 128 <= N);
        __nv_bfloat16* yrow = Y + static_cast<uint64_t>(m) * N + n0 + col0;
        const float4* swv = reinterpret_cast<const float4*>(sw + n0 + col0);
#pragma unroll
        for (int j = 0; j < 128; j += 8) {
          float c[8];
          if (w_per_tensor) {
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] = __fmul_rn(a, w0);
          } else {
            const float4 u = __ldg(swv + j / 4), v = __ldg(swv + j / 4 + 1);
            c[0] = __fmul_rn(a, u.x); c[1] = __fmul_rn(a, u.y); c[2] = __fmul_rn(a, u.z); c[3] = __fmul_rn(a, u.w);
            c[4] = __fmul_rn(a, v.x); c[5] = __fmul_rn(a, v.y); c[6] = __fmul_rn(a, v.z); c[7] = __fmul_rn(a, v.w);
          }
          uint4 o;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(p[j + 0]), c[0]),
                                                    __fmul_rn(__uint_as_float(p[j + 1]), c[1]));
          __nv_bfloat162 h1 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(p[j + 2]), c[2]),
                                                    __fmul_rn(__uint_as_float(p[j + 3]), c[3]));
          __nv_bfloat162 h2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(p[j + 4]), c[4]),
                                                    __fmul_rn(__uint_as_float(p[j + 5]), c[5]));
          __nv_bfloat162 h3 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(p[j + 6]), c[6]),
                                                    __fmul_rn(__uint_as_float(p[j + 7]), c[7]));
          o.x = *reinterpret_cast<uint32_t*>(&h0);
          o.y = *reinterpret_cast<uint32_t*>(&h1);
          o.z = *reinterpret_cast<uint32_t*>(&h2);
          o.w = *reinterpret_cast<uint32_t*>(&h3);
          *reinterpret_cast<uint4*>(yrow + j) = o;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------------------
// Few-token variant with fp32 scales (M <= 64, decode; UE8M0 scales take
// gemm_decode_mx_kernel below): operands swapped so the weight supplies the
// MMA's 128 rows and the tokens its N dimension (BNT = M rounded up to
// 16/32/64).  One CTA streams one 128-row weight slab through a deep TMA ring
// (the layer is bound by reading Wq from HBM).  TMEM holds D^T: lane = output
// column n, column = token m.  Each promotion thread owns one n and BNT
// accumulators; the token scales sa[m, kb] are fetched once per warp
// (one per lane) and broadcast with shuffles.
// ---------------------------------------------------------------------------
template <int BNT>
struct DecodeCfg {
  static constexpr uint32_t kABytes = 128 * 128;             // weight tile
  static constexpr uint32_t kBBytes = BNT * 128;             // token tile
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 12 ? 12 : (200 * 1024) / kStageBytes;
  static constexpr int kThreads = 6 * 32;                    // producer, MMA, 4 promotion warps
  static constexpr int kNumBuf = 4;                          // TMEM partial buffers
  static constexpr uint32_t kTmemCols = (kNumBuf * BNT < 32) ? 32 : kNumBuf * BNT;
  static constexpr size_t kSmemBytes = 1024 + kStages * static_cast<size_t>(kStageBytes) + 256;
};

template <int BNT, int FMT>
__global__ void __launch_bounds__(DecodeCfg<BNT>::kThreads, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const void* __restrict__ Xs, uint32_t ld_s, const void* __restrict__ Ws,
                       __nv_bfloat16* __restrict__ Y, int M, int N, int K, int early_w) {
  using C = DecodeCfg<BNT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + C::kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + C::kStages * C::kBBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + C::kNumBuf;
  uint64_t* mma_done = tempty + C::kNumBuf;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = K / 128;
  const int n0 = blockIdx.x * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kNumBuf; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(mma_done, 1);
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Dependency on the preceding grid (programmatic launch): the producer may
  // request the first weight tiles before it; every other access follows it.
  if (threadIdx.x != 0) griddep_wait();
  if (warp == 0) {
    if (lane == 0)
      produce_tiles<C::kStages, C::kABytes, C::kBBytes>(&tmW, n0, &tmX, 0, KB, sW, sX, full, empty, early_w != 0);
  } else if (warp == 1) {
    if (lane == 0)
      issue_mmas<C::kStages, C::kABytes, C::kBBytes, BNT, C::kNumBuf>(smem_u32(sW), smem_u32(sX), KB, tmem_base,
                                                                      full, empty, tfull, tempty, mma_done);
  } else {
    const int quad = warp & 3;
    const int n = n0 + quad * 32 + lane;
    const uint64_t ws_row = static_cast<uint64_t>(n0 / 128) * KB;
    const uint32_t taddr0 = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    constexpr int kT = (BNT + 31) / 32;              // scale words per lane

    float acc[BNT];
#pragma unroll
    for (int j = 0; j < BNT; ++j) acc[j] = 0.0f;

    // raw scale words of block kb: lane l holds the token scales l, l+32
    // (0 for tokens >= M) and the weight scale; ring slot kb % kScaleAhead
    uint32_t ra[kScaleAhead][kT], rw[kScaleAhead];
    auto fetch = [&](int kb, uint32_t (&a)[kT], uint32_t& w) {
      const bool in = kb < KB;
      w = in ? load_scale_raw<FMT>(Ws, ws_row + kb) : 0u;
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int m = t * 32 + lane;
        a[t] = (in && m < M) ? load_scale_raw<FMT>(Xs, static_cast<uint64_t>(kb) * ld_s + m) : 0u;
      }
    };
#pragma unroll
    for (int d = 0; d < kScaleAhead; ++d) fetch(d, ra[d], rw[d]);

    bool ok = true;
    for (int kb0 = 0; kb0 < KB && ok; kb0 += kScaleAhead) {
#pragma unroll
      for (int d = 0; d < kScaleAhead; ++d) {
        const int kb = kb0 + d;
        if (kb >= KB) break;
        float sc[kT];
#pragma unroll
        for (int t = 0; t < kT; ++t) sc[t] = (t * 32 + lane < M) ? combine_raw<FMT>(ra[d][t], rw[d]) : 0.0f;
        fetch(kb + kScaleAhead, ra[d], rw[d]);
        const int b = kb % C::kNumBuf;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], (kb / C::kNumBuf) & 1u))) {
          if (lane == 0) record_status(kDevTimeoutEpilogue);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = taddr0 + static_cast<uint32_t>(b * BNT);
        uint32_t p[BNT];
#pragma unroll
        for (int c = 0; c < BNT / 16; ++c)
          tmem_ld_32x32b_x16(taddr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&p[c * 16]));
        tmem_wait_ld();
#pragma unroll
        for (int mm = 0; mm < BNT; ++mm) {
          const float a = __shfl_sync(0xFFFFFFFFu, sc[mm / 32], mm % 32);
          acc[mm] = __fmaf_rn(__uint_as_float(p[mm]), a, acc[mm]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
      }
    }
    if (ok && n < N) {
#pragma unroll
      for (int m = 0; m < BNT; ++m)
        if (m < M) {
          FGFP8_DCHECK(m < BNT);
          Y[static_cast<uint64_t>(m) * N + n] = __float2bfloat16_rn(acc[m]);
        }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ---------------------------------------------------------------------------
// Few-token GEMM with UE8M0 scales on the block-scaled MMA ("UE8M0 scale
// format": power-of-two scales the tensor core applies itself).  Operands
// swapped as in gemm_decode_kernel: the CTA's 128 weight rows are the MMA's
// M, the BNT token rows its N.  Every A row takes the weight block's scale,
// every B row its token's 1x128 group scale, so the whole K reduction
// accumulates in TMEM and nothing but the scale words runs per K block off
// the tensor pipe (groups of four K blocks, byte b of each word for K block
// 4g + b, as in gemm_mx_kernel).
//   warp 0      TMA: per K block the 128-row weight tile and the token tile
//               (rows >= M read as zeros);
//   warp 1      TMEM owner and MMA issuer: per scale group tcgen05.cp of
//               the two scale tiles, per K block four block-scaled MMAs;
//   warp 2      the scale words into shared memory, two groups per fence;
//   warps 4..7  epilogue: the BNT finished columns of their 32 weight rows,
//               stored transposed into Y[m, n].
// ---------------------------------------------------------------------------
template <int BNT>
struct DecodeMxCfg {
  static constexpr uint32_t kABytes = 128 * 128;             // weight tile
  static constexpr uint32_t kBBytes = BNT * 128;             // token tile
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024) / kStageBytes > 12 ? 12 : (192 * 1024) / kStageBytes;
  static constexpr int kSfGroup = 4;                         // K blocks per scale word
  static constexpr int kSfBatch = 2;                         // groups per shared-memory fence
  static constexpr int kSfSlots = 2 * kSfBatch;
  static constexpr uint32_t kSfTileBytes = 512;              // one 32 x 16-byte scale tile
  static constexpr int kThreads = 8 * 32;
  static constexpr uint32_t kSfCol = BNT < 32 ? 32 : BNT;    // scale slots after the accumulator
  static constexpr uint32_t kSfColsPerSlot = 8;              // A: 4 columns, B: 4 columns
  static constexpr uint32_t kTmemCols = (kSfCol + kSfSlots * kSfColsPerSlot) <= 64 ? 64 : 128;
  static constexpr size_t kBarrierBytes = 256;
  static constexpr size_t kSmemBytes =
      1024 + kStages * static_cast<size_t>(kStageBytes) + kSfSlots * 2 * static_cast<size_t>(kSfTileBytes) + kBarrierBytes;
};

template <int BNT>
__global__ void __launch_bounds__(DecodeMxCfg<BNT>::kThreads, 1)
    gemm_decode_mx_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                          const uint8_t* __restrict__ Xs, uint32_t ld_s, const uint8_t* __restrict__ Ws,
                          __nv_bfloat16* __restrict__ Y, int M, int N, int K, int early_w) {
  using C = DecodeMxCfg<BNT>;
  static_assert(C::kSfCol + C::kSfSlots * C::kSfColsPerSlot <= C::kTmemCols, "TMEM columns");
  static_assert((2 * C::kStages + 1 + 1 + 2 * C::kSfSlots) * 8 + 4 <= C::kBarrierBytes, "barrier area");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + C::kStages * C::kABytes;
  uint8_t* sSfA = sX + C::kStages * C::kBBytes;                 // weight-block scale tiles, per slot
  uint8_t* sSfB = sSfA + C::kSfSlots * C::kSfTileBytes;         // token scale tiles, per slot
  uint64_t* full = reinterpret_cast<uint64_t*>(sSfB + C::kSfSlots * C::kSfTileBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* mma_done = tfull + 1;
  uint64_t* sf_full = mma_done + 1;
  uint64_t* sf_empty = sf_full + C::kSfSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + C::kSfSlots);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = K / 128;
  const int n0 = blockIdx.x * 128;
  const int groups = (KB + C::kSfGroup - 1) / C::kSfGroup;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(mma_done, 1);
    for (int b = 0; b < C::kSfSlots; ++b) {
      mbar_init(&sf_full[b], 1);
      mbar_init(&sf_empty[b], 1);
    }
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Dependency on the preceding grid (programmatic launch): the producer may
  // request the first weight tiles before it; every other access follows it.
  if (threadIdx.x != 0) griddep_wait();
  if (warp == 0) {
    if (lane == 0)
      produce_tiles<C::kStages, C::kABytes, C::kBBytes>(&tmW, n0, &tmX, 0, KB, sW, sX, full, empty, early_w != 0);
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= MMA issuer
      constexpr uint32_t idesc0 = idesc_mx_e4m3_ue8m0(128, BNT);
      const uint64_t a_desc0 = smem_desc_k_sw128(smem_u32(sW)), b_desc0 = smem_desc_k_sw128(smem_u32(sX));
      const uint64_t sfa_desc0 = smem_desc_rows16(smem_u32(sSfA)), sfb_desc0 = smem_desc_rows16(smem_u32(sSfB));
      bool ok = true;
      uint32_t it = 0;
      for (int g = 0; g < groups && ok; ++g) {
        const int sl = g % C::kSfSlots;
        if (!mbar_wait(&sf_full[sl], (g / C::kSfSlots) & 1u)) {
          record_status(kDevTimeoutMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sfa = tmem_base + C::kSfCol + static_cast<uint32_t>(sl * C::kSfColsPerSlot);
        const uint32_t sfb = sfa + 4;
        tmem_cp_32x128b_x4(sfa, sfa_desc0 + ((sl * C::kSfTileBytes) >> 4));
        tmem_cp_32x128b_x4(sfb, sfb_desc0 + ((sl * C::kSfTileBytes) >> 4));
        mma_commit(&sf_empty[sl]);                     // the slot may be refilled once copied
        const int kb0 = g * C::kSfGroup, kb1 = kb0 + C::kSfGroup < KB ? kb0 + C::kSfGroup : KB;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::kStages;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1u)) {
            record_status(kDevTimeoutMma);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf_id = static_cast<uint32_t>(kb - kb0);
          const uint32_t idesc = idesc0 | (sf_id << 29) | (sf_id << 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = a_desc0 + ((s * C::kABytes + kk * 32) >> 4);
            const uint64_t bdesc = b_desc0 + ((s * C::kBBytes + kk * 32) >> 4);
            mma_mxf8f6f4(tmem_base, adesc, bdesc, idesc, sfa, sfb, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
      }
      if (ok) mma_commit(tfull);
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) record_status(kDevTimeoutMma);
    }
  } else if (warp == 2) {
    // ================= scale words into shared memory (all lanes)
    // Group g: the weight block's word (byte b: K block 4g + b) in every
    // position of the A tile; B tile lane l, word j: token l + 32 j (127 =
    // 2^0 past M; rows >= BNT are never read).  Raw bytes one batch ahead.
    const uint64_t ws_row = static_cast<uint64_t>(n0 / 128) * KB;
    uint32_t ra[C::kSfBatch][4][C::kSfGroup], rw[C::kSfBatch][C::kSfGroup];
    auto fetch = [&](int g0) {
#pragma unroll
      for (int q = 0; q < C::kSfBatch; ++q) {
#pragma unroll
        for (int b = 0; b < C::kSfGroup; ++b) {
          const int kb = (g0 + q) * C::kSfGroup + b;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = lane + 32 * j;
            ra[q][j][b] = (kb < KB && m < M && m < BNT) ? __ldg(Xs + static_cast<uint64_t>(kb) * ld_s + m) : 127u;
          }
          rw[q][b] = kb < KB ? __ldg(Ws + ws_row + kb) : 127u;
        }
      }
    };
    auto pack = [](const uint32_t (&v)[C::kSfGroup]) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < C::kSfGroup; ++b) word |= v[b] << (8 * b);
      return word;
    };
    fetch(0);
    for (int g0 = 0; g0 < groups; g0 += C::kSfBatch) {
      const int nb = groups - g0 < C::kSfBatch ? groups - g0 : C::kSfBatch;
      bool free = true;
      for (int q = 0; q < nb; ++q) {
        const int gq = g0 + q;
        free = free && (gq < C::kSfSlots || mbar_wait(&sf_empty[gq % C::kSfSlots], ((gq / C::kSfSlots) & 1) ^ 1));
      }
      if (!__all_sync(0xFFFFFFFFu, free)) {
        if (lane == 0) record_status(kDevTimeoutProducer);
        break;
      }
#pragma unroll
      for (int q = 0; q < C::kSfBatch; ++q) {
        if (q < nb) {
          const int sl = (g0 + q) % C::kSfSlots;
          const uint32_t w = pack(rw[q]);
          *reinterpret_cast<uint4*>(sSfA + sl * C::kSfTileBytes + lane * 16) = make_uint4(w, w, w, w);
          *reinterpret_cast<uint4*>(sSfB + sl * C::kSfTileBytes + lane * 16) =
              make_uint4(pack(ra[q][0]), pack(ra[q][1]), pack(ra[q][2]), pack(ra[q][3]));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0)
        for (int q = 0; q < nb; ++q) mbar_arrive(&sf_full[(g0 + q) % C::kSfSlots]);
      fetch(g0 + C::kSfBatch);
    }
  } else if (warp >= 4) {
    // ================= epilogue
    const int quad = warp & 3;
    const int n = n0 + quad * 32 + lane;
    if (__all_sync(0xFFFFFFFFu, mbar_wait(tfull, 0))) {
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      uint32_t p[BNT];
#pragma unroll
      for (int c = 0; c < BNT / 16; ++c)
        tmem_ld_32x32b_x16(taddr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&p[c * 16]));
      tmem_wait_ld();
      if (n < N) {
#pragma unroll
        for (int m = 0; m < BNT; ++m)
          if (m < M) {
            FGFP8_DCHECK(m < BNT);
            Y[static_cast<uint64_t>(m) * N + n] = __float2bfloat16_rn(__uint_as_float(p[m]));
          }
      }
    } else if (lane == 0) {
      record_status(kDevTimeoutEpilogue);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

}  // namespace fgfp8
