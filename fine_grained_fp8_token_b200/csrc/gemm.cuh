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

// ---------------------------------------------------------------------------
// Pipeline roles shared by the GEMM kernels.
// ---------------------------------------------------------------------------

// TMA producer (one thread): per K block, a kABytes tile of operand A (rows
// a_row.., box from tmA) and a kBBytes tile of operand B into ring slot
// kb % kStages; waits for the slot to be released by the MMA first.  Before
// returning it waits for every copy it issued to land.
template <int kStages, uint32_t kABytes, uint32_t kBBytes>
__device__ __forceinline__ void produce_tiles(const CUtensorMap* tmA, int a_row, const CUtensorMap* tmB, int b_row,
                                              int KB, uint8_t* sA, uint8_t* sB, uint64_t* full, uint64_t* empty) {
  int issued = 0;
  for (int kb = 0; kb < KB; ++kb) {
    const int s = kb % kStages;
    const uint32_t use = kb / kStages;
    if (kb >= kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u)) {
      record_status(kDevTimeoutProducer);
      break;
    }
    mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
    tma_load_2d(sA + s * kABytes, tmA, &full[s], kb * 128, a_row);
    tma_load_2d(sB + s * kBBytes, tmB, &full[s], kb * 128, b_row);
    issued = kb + 1;
  }
  for (int kb = (issued > kStages ? issued - kStages : 0); kb < issued; ++kb) {
    if (!mbar_wait(&full[kb % kStages], (kb / kStages) & 1u)) record_status(kDevTimeoutProducer);
  }
}

// MMA issuer (one thread): per K block, four K=32 tcgen05.mma (M=128, N=kN)
// into TMEM partial buffer kb & 1 (columns [b*kN, b*kN + kN)), overwriting it
// on the first step; then frees the smem slot and publishes the buffer.  The
// buffer is reused only after the promotion warps released it.  A final
// commit makes every MMA complete before the caller may free TMEM.
template <int kStages, uint32_t kABytes, uint32_t kBBytes, int kN>
__device__ __forceinline__ void issue_mmas(uint32_t a_base, uint32_t b_base, int KB, uint32_t tmem_base,
                                           uint64_t* full, uint64_t* empty, uint64_t* tfull, uint64_t* tempty,
                                           uint64_t* mma_done) {
  constexpr uint32_t idesc = idesc_e4m3_f32(128, kN);
  for (int kb = 0; kb < KB; ++kb) {
    const int s = kb % kStages;
    const int b = kb & 1;
    if (!mbar_wait(&full[s], (kb / kStages) & 1u)) {
      record_status(kDevTimeoutMma);
      break;
    }
    if (kb >= 2 && !mbar_wait(&tempty[b], ((kb >> 1) & 1u) ^ 1u)) {
      record_status(kDevTimeoutMma);
      break;
    }
    tc_fence_after();
    const uint32_t d = tmem_base + static_cast<uint32_t>(b * kN);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t ad = smem_desc_k_sw128(a_base + s * kABytes + kk * 32);
      const uint64_t bd = smem_desc_k_sw128(b_base + s * kBBytes + kk * 32);
      mma_f8f6f4(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
    mma_commit(&empty[s]);
    mma_commit(&tfull[b]);
  }
  mma_commit(mma_done);
  if (!mbar_wait(mma_done, 0)) record_status(kDevTimeoutMma);
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
    if (lane == 0)
      produce_tiles<C::kStages, C::kABytes, C::kBBytes>(&tmA, m0, &tmB, expert * N + n0, KB, sA, sB, full, empty);
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0)
      issue_mmas<C::kStages, C::kABytes, C::kBBytes, BN>(smem_u32(sA), smem_u32(sB), KB, tmem_base, full, empty,
                                                         tfull, tempty, mma_done);
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


// ---------------------------------------------------------------------------
// Few-token variant (M <= 64, decode): operands swapped so the weight supplies
// the MMA's 128 rows and the tokens its N dimension (BNT = M rounded up to
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
  static constexpr uint32_t kTmemCols = (2 * BNT < 32) ? 32 : 2 * BNT;
  static constexpr size_t kSmemBytes = 1024 + kStages * static_cast<size_t>(kStageBytes) + 256;
};

template <int FMT>
__device__ __forceinline__ uint32_t load_scale_raw(const void* __restrict__ p, uint64_t i) {
  if (FMT == 0) return __float_as_uint(__ldg(reinterpret_cast<const float*>(p) + i));
  return __ldg(reinterpret_cast<const uint8_t*>(p) + i);
}

// sa * sw from raw scale words (fp32 bits or UE8M0 bytes).
template <int FMT>
__device__ __forceinline__ float combine_raw(uint32_t a, uint32_t w) {
  if (FMT == 0) return __uint_as_float(a) * __uint_as_float(w);
  const int e = static_cast<int>(a) + static_cast<int>(w) - 127;
  if (e >= 1 && e <= 254) return __int_as_float(e << 23);
  return ldexpf(1.0f, static_cast<int>(a) + static_cast<int>(w) - 254);
}

template <int BNT, int FMT>
__global__ void __launch_bounds__(DecodeCfg<BNT>::kThreads, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const void* __restrict__ Xs, uint32_t ld_s, const void* __restrict__ Ws,
                       __nv_bfloat16* __restrict__ Y, int M, int N, int K) {
  using C = DecodeCfg<BNT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sX = smem + C::kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + C::kStages * C::kBBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
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
    for (int b = 0; b < 2; ++b) {
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

  if (warp == 0) {
    if (lane == 0)
      produce_tiles<C::kStages, C::kABytes, C::kBBytes>(&tmW, n0, &tmX, 0, KB, sW, sX, full, empty);
  } else if (warp == 1) {
    if (lane == 0)
      issue_mmas<C::kStages, C::kABytes, C::kBBytes, BNT>(smem_u32(sW), smem_u32(sX), KB, tmem_base, full, empty,
                                                          tfull, tempty, mma_done);
  } else {
    const int quad = warp & 3;
    const int n = n0 + quad * 32 + lane;
    const uint64_t ws_row = static_cast<uint64_t>(n0 / 128) * KB;
    const uint32_t taddr0 = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    constexpr int kT = (BNT + 31) / 32;              // scale words per lane

    float acc[BNT];
#pragma unroll
    for (int j = 0; j < BNT; ++j) acc[j] = 0.0f;

    // raw scales of block kb: lane l holds the token scales l, l+32 (if < M)
    auto load_scales = [&](int kb, uint32_t (&sa)[kT], uint32_t& sw) {
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int m = t * 32 + lane;
        sa[t] = m < M ? load_scale_raw<FMT>(Xs, static_cast<uint64_t>(kb) * ld_s + m) : 0u;
      }
      sw = load_scale_raw<FMT>(Ws, ws_row + kb);
    };

    bool ok = true;
    uint32_t sa_next[kT], sw_next;
    load_scales(0, sa_next, sw_next);
    for (int kb = 0; kb < KB; ++kb) {
      const int b = kb & 1;
      uint32_t sa[kT];
#pragma unroll
      for (int t = 0; t < kT; ++t) sa[t] = sa_next[t];
      const uint32_t sw = sw_next;
      if (kb + 1 < KB) load_scales(kb + 1, sa_next, sw_next);
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[b], (kb >> 1) & 1u))) {
        if (lane == 0) record_status(kDevTimeoutEpilogue);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = taddr0 + static_cast<uint32_t>(b * BNT);
#pragma unroll
      for (int c = 0; c < BNT / 16; ++c) {
        uint32_t p[16];
        tmem_ld_32x32b_x16(taddr + c * 16, p);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = c * 16 + j;
          const uint32_t a = __shfl_sync(0xFFFFFFFFu, sa[m / 32], m % 32);
          const float sc = (m < M) ? combine_raw<FMT>(a, sw) : 0.0f;
          acc[m] = __fmaf_rn(__uint_as_float(p[j]), sc, acc[m]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
    }
    if (ok && n < N) {
#pragma unroll
      for (int m = 0; m < BNT; ++m)
        if (m < M) Y[static_cast<uint64_t>(m) * N + n] = __float2bfloat16_rn(acc[m]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

}  // namespace fgfp8
