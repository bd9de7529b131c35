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
//               partial buffers (ping-pong), then commits to the slot's
//               "empty" barrier and the buffer's "full" barrier;
//   warps 2..   promotion: each thread owns one output row and 128 columns; it
//               loads the block partial from TMEM, multiplies by the product
//               of the two block scales and accumulates in fp32 registers, so
//               the MMA of block kb+1 overlaps the promotion of block kb.
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

#include "ptx.cuh"

namespace fgfp8 {

__device__ int g_device_status;

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_device_status, 0, code); }

template <int BN>
struct GemmCfg {
  static constexpr int kBM = 128;
  static constexpr int kBK = 128;
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr int kEpiWarps = BN / 32;                  // one warp per 32 rows x 128 columns
  static constexpr int kThreads = (2 + kEpiWarps) * 32;
  static constexpr uint32_t kTmemCols = 2 * BN;              // two partial buffers
  static constexpr uint32_t kABytes = kBM * kBK;
  static constexpr uint32_t kBBytes = BN * kBK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr size_t kBarrierBytes = 256;
  static constexpr size_t kSmemBytes = 1024 + kStages * static_cast<size_t>(kStageBytes) + kBarrierBytes;
};

// Combined block scale sa[m, kb] * sw[nb, kb] for one K block.  fp32 scales
// multiply in fp32; UE8M0 scales are exponent bytes: 2^(ea-127) * 2^(eb-127)
// = 2^(ea+eb-254), built exactly from the biased exponent ea+eb-127 (or by
// ldexpf when that leaves the normal range).  A 0xFF (NaN) scale byte gives
// an unspecified product.
template <int FMT>
__device__ __forceinline__ float block_scale(const void* __restrict__ Xs, uint64_t ia, const void* __restrict__ Ws,
                                             uint64_t iw) {
  if (FMT == 0) return __ldg(reinterpret_cast<const float*>(Xs) + ia) * __ldg(reinterpret_cast<const float*>(Ws) + iw);
  const int ea = __ldg(reinterpret_cast<const uint8_t*>(Xs) + ia);
  const int eb = __ldg(reinterpret_cast<const uint8_t*>(Ws) + iw);
  const int e = ea + eb - 127;
  if (e >= 1 && e <= 254) return __int_as_float(e << 23);
  return ldexpf(1.0f, ea + eb - 254);
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

template <int BN, int FMT, bool kGrouped>
__global__ void __launch_bounds__(GemmCfg<BN>::kThreads, 1)
    gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const void* __restrict__ Xs, uint32_t ld_s, const void* __restrict__ Ws,
                            __nv_bfloat16* __restrict__ Y, int M, int N, int K,
                            const int32_t* __restrict__ group_offs, int E) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::kStages * C::kBBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = K / C::kBK;
  const int NB = N / 128;

  // ---- tile coordinates
  int m_tile, n_tile;
  if (!kGrouped) {
    const int num_m = (M + C::kBM - 1) / C::kBM;
    m_tile = blockIdx.x % num_m;
    n_tile = blockIdx.x / num_m;
  } else {
    const int num_n = N / BN;
    n_tile = blockIdx.x % num_n;
    m_tile = blockIdx.x / num_n;
  }
  const int m0 = m_tile * C::kBM;
  const int n0 = n_tile * BN;
  int expert = 0;
  if (kGrouped) {
    expert = find_expert(group_offs, E, m0);
    if (expert < 0) {                        // uniform across the CTA
      if (threadIdx.x == 0) record_status(kDevBadGroupOffsets);
      return;
    }
  }

  // ---- setup: barriers (thread 0), TMEM (warp 1)
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
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer
    if (lane == 0) {
      const int b_row0 = expert * N + n0;
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % C::kStages;
        const uint32_t use = kb / C::kStages;
        if (kb >= C::kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u)) {
          record_status(kDevTimeoutProducer);
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        tma_load_2d(sA + s * C::kABytes, &tmA, &full[s], kb * C::kBK, m0);
        tma_load_2d(sB + s * C::kBBytes, &tmB, &full[s], kb * C::kBK, b_row0);
        issued = kb + 1;
      }
      // every copy issued must have landed before the CTA may exit
      for (int kb = (issued > C::kStages ? issued - C::kStages : 0); kb < issued; ++kb) {
        if (!mbar_wait(&full[kb % C::kStages], (kb / C::kStages) & 1u)) record_status(kDevTimeoutProducer);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(128, BN);
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % C::kStages;
        const int b = kb & 1;
        if (!mbar_wait(&full[s], (kb / C::kStages) & 1u)) {
          record_status(kDevTimeoutMma);
          break;
        }
        if (kb >= 2 && !mbar_wait(&tempty[b], ((kb >> 1) & 1u) ^ 1u)) {
          record_status(kDevTimeoutMma);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * BN);
#pragma unroll
        for (int kk = 0; kk < C::kBK / 32; ++kk) {
          const uint64_t ad = smem_desc_k_sw128(a_base + s * C::kABytes + kk * 32);
          const uint64_t bd = smem_desc_k_sw128(b_base + s * C::kBBytes + kk * 32);
          mma_f8f6f4(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[b]);
      }
      // all MMAs of this thread complete before TMEM may be freed
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) record_status(kDevTimeoutMma);
    }
  } else {
    // ================= promotion / epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int col0 = (ew >> 2) * 128;          // column half (BN = 256) or 0
    const int row = quad * 32 + lane;
    const int m = m0 + row;
    const bool row_ok = m < M;
    const bool col_ok = n0 + col0 < N;
    const uint64_t ws_row = (static_cast<uint64_t>(expert) * NB + (n0 + col0) / 128) * KB;
    const uint32_t taddr0 = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(col0);

    float acc[128];
#pragma unroll
    for (int j = 0; j < 128; ++j) acc[j] = 0.0f;

    auto scale_of = [&](int kb) -> float {
      return (row_ok && col_ok) ? block_scale<FMT>(Xs, static_cast<uint64_t>(kb) * ld_s + m, Ws, ws_row + kb)
                                : 0.0f;
    };

    bool ok = true;
    float s_next = scale_of(0);
    for (int kb = 0; kb < KB; ++kb) {
      const int b = kb & 1;
      const float s = s_next;
      if (kb + 1 < KB) s_next = scale_of(kb + 1);
      // the outcome is made warp-uniform: the TMEM loads below are .sync.aligned
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], (kb >> 1) & 1u))) {
        if (lane == 0) record_status(kDevTimeoutEpilogue);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = taddr0 + static_cast<uint32_t>(b * BN);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t p[32];
        tmem_ld_32x32b_x32(taddr + c * 32, p);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[c * 32 + j] = __fmaf_rn(__uint_as_float(p[j]), s, acc[c * 32 + j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
    }

    if (ok && row_ok && col_ok) {
      __nv_bfloat16* yrow = Y + static_cast<uint64_t>(m) * N + n0 + col0;
#pragma unroll
      for (int j = 0; j < 128; j += 8) {
        uint4 v;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j + 0], acc[j + 1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
        v.x = *reinterpret_cast<uint32_t*>(&h0);
        v.y = *reinterpret_cast<uint32_t*>(&h1);
        v.z = *reinterpret_cast<uint32_t*>(&h2);
        v.w = *reinterpret_cast<uint32_t*>(&h3);
        *reinterpret_cast<uint4*>(yrow + j) = v;
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

}  // namespace fgfp8
