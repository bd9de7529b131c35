// Dynamic per-token (1x128) activation quantization and 128x128 block weight
// quantization to FP8 E4M3 with fp32 or UE8M0 scales.
//
// Method ("Fine-grained FP8", introduction and "UE8M0 scale format"; E4M3
// range from "FP8 W8A8", "Two FP8 representations"):
//   amax  = max |x| over the group or block (NaN propagates), raised to 1e-4
//   fp32  : s = amax / 448 (IEEE division), code = E4M3_rne_satfinite(x / s)
//   UE8M0 : s = 2^ceil(log2(amax / 448)), stored as its biased exponent byte
//
// Divisions are evaluated without a division routine: with r = RN(1/d),
// q0 = RN(a r), e = fma(-q0, d, a), q = fma(e, r, q0) is the correctly
// rounded a/d (Markstein's theorem, "IA-64 and Elementary Functions", 2000;
// Muller et al., "Handbook of Floating-Point Arithmetic", the FMA-based
// division section).  It is used for amax/448 (r = RN(1/448), a constant) and
// for |x|/s (r = RN(1/s) once per group).  A host-side test checks both
// against IEEE division on every input the kernel can meet: every bf16 amax,
// and every (bf16 element, bf16 amax) pair.  For UE8M0 the quotient is
// |x| * 2^-p, exact.  The sign of x is applied to the E4M3 code afterwards,
// so -0 and tiny negatives keep it.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cmath>
#include <cstdint>

#include "ptx.cuh"

namespace fgfp8 {

constexpr int kGroup = 128;

// Unsigned 32-bit division by a runtime-invariant divisor, by multiplication
// (Granlund & Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994, the round-up variant for N = 32).
struct FastDiv {
  uint32_t d, mult, sh1, sh2;
  __host__ __device__ explicit FastDiv(uint32_t divisor) : d(divisor) {
    uint32_t l = 0;
    while ((1ull << l) < divisor) ++l;                      // l = ceil(log2 d)
    mult = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - divisor)) / divisor + 1);
    sh1 = l < 1 ? l : 1;
    sh2 = l > 1 ? l - 1 : 0;
  }
  __host__ __device__ __forceinline__ uint32_t div(uint32_t n) const {
#ifdef __CUDA_ARCH__
    const uint32_t t = __umulhi(mult, n);
#else
    const uint32_t t = static_cast<uint32_t>((static_cast<uint64_t>(mult) * n) >> 32);
#endif
    return (t + ((n - t) >> sh1)) >> sh2;
  }
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// max |x| bits over 8 packed bf16 (sign masked; NaN patterns compare above
// every finite value and infinity, so they propagate).
__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
  const uint32_t m = 0x7FFF7FFFu;
  uint32_t a = __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
  return max(a & 0xFFFFu, a >> 16);
}

struct GroupScale {
  float s;        // the scale (fp32 path) or 2^p (UE8M0 path)
  float r;        // RN(1/s) (fp32 path) or the exact 2^-p (UE8M0 path)
  uint32_t e8;    // UE8M0 byte
};

template <int FMT>
__device__ __forceinline__ GroupScale make_scale(uint32_t amax_bits) {
  const float amax = __uint_as_float(amax_bits << 16);
  const float amax_c = amax < 1e-4f ? 1e-4f : amax;    // NaN stays NaN
  constexpr float kR448 = 1.0f / 448.0f;               // RN(1/448), folded at compile time
  const float q0 = __fmul_rn(amax_c, kR448);
  const float t = __fmaf_rn(__fmaf_rn(-q0, 448.0f, amax_c), kR448, q0);   // = RN(amax_c / 448)
  GroupScale g;
  if (FMT == 0) {
    g.s = t;
    g.r = __frcp_rn(t);
    g.e8 = 0;
  } else {
    uint32_t b = __float_as_uint(t);
    uint32_t e = b >> 23;                                // t > 0: sign bit clear
    if ((b & 0x7FFFFFu) != 0u && e < 255u) e += 1u;      // round up to a power of two
    g.e8 = e;
    g.s = 0.0f;
    g.r = (e >= 1u && e <= 253u) ? __uint_as_float((254u - e) << 23) : 0.0f;   // 2^(127-e)
  }
  return g;
}

// Four bf16 (two packed words) -> four E4M3 codes in one word (element 0 in
// the low byte).  Magnitudes are quantized (div(x) = |x| / s); the four sign
// bits (bit 7 of the bf16 bytes 1 and 3 of each word) are gathered with one
// byte permute.
template <typename Div>
__device__ __forceinline__ uint32_t quant4_by(uint32_t w0, uint32_t w1, const Div& div) {
  const uint32_t c0 = __nv_cvt_float2_to_fp8x2(
      make_float2(div(__uint_as_float(w0 << 16)), div(__uint_as_float(w0 & 0xFFFF0000u))), __NV_SATFINITE, __NV_E4M3);
  const uint32_t c1 = __nv_cvt_float2_to_fp8x2(
      make_float2(div(__uint_as_float(w1 << 16)), div(__uint_as_float(w1 & 0xFFFF0000u))), __NV_SATFINITE, __NV_E4M3);
  const uint32_t codes = __byte_perm(c0, c1, 0x5410);
  const uint32_t signs = __byte_perm(w0, w1, 0x7531) & 0x80808080u;
  return codes | signs;
}

// Four bf16 -> four E4M3 codes with the group's scale, in packed fp32x2
// arithmetic (two elements per instruction).  Per element: |x| (the bf16
// sign bit cleared before the widening), then for fp32 scales the FMA form
// of Markstein's correctly rounded division, q0 = RN(|x| r),
// q = RN(fma(RN(fma(-q0, s, |x|)), r, q0)) with r = RN(1/s); for UE8M0
// scales the exact product |x| * 2^-p.  Signs and byte order as in quant4_by.
template <int FMT>
__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, const GroupScale& g) {
  const float2 r2 = make_float2(g.r, g.r);
  auto q2 = [&](uint32_t w) {
    const float2 a = make_float2(__uint_as_float((w << 16) & 0x7FFFFFFFu), __uint_as_float(w & 0x7FFF0000u));
    const float2 q0 = __fmul2_rn(a, r2);
    if (FMT != 0) return q0;
    const float2 ns2 = make_float2(-g.s, -g.s);
    return __ffma2_rn(__ffma2_rn(q0, ns2, a), r2, q0);
  };
  const uint32_t c0 = __nv_cvt_float2_to_fp8x2(q2(w0), __NV_SATFINITE, __NV_E4M3);
  const uint32_t c1 = __nv_cvt_float2_to_fp8x2(q2(w1), __NV_SATFINITE, __NV_E4M3);
  const uint32_t codes = __byte_perm(c0, c1, 0x5410);
  const uint32_t signs = __byte_perm(w0, w1, 0x7531) & 0x80808080u;
  return codes | signs;
}

// |x| / s for a caller-given scale s > 0 (static quantization), correctly
// rounded wherever the E4M3 code depends on it.  Unlike the dynamic scales
// (amax/448 with |x| <= amax, so the quotient stays below 449), a given scale
// can meet any bf16 |x|, and the FMA form above fails at the ends of the
// range: RN(|x| r) overflows to infinity for |x|/s > 2^128 (the correction
// then gives inf - inf = NaN), and r = RN(1/s) itself overflows or loses
// precision for s below 2^-126.  So:
//  * kFast (s in [2^-92, 2^126], checked once per launch): the FMA form.  In
//    that window 1/s is a normal number, and every quotient >= 2^-11 has
//    |x| >= 2^-103, so the residual fma(-q0, s, |x|) is exact and Markstein's
//    theorem gives RN(|x|/s).  Quotients below 2^-11 come out below 2^-10 and
//    encode to a zero code either way.  When the first approximation q0
//    reaches 1024 the quotient exceeds 448 and saturates whatever its last
//    bits: q0 itself is returned (also when it is infinite).
//  * otherwise: the IEEE quotient (__fdiv_rn) for every element.
// Host code gets the same operations from the host compiler's IEEE fp32
// arithmetic, so the host checks run this very function.
template <bool kFast>
__host__ __device__ __forceinline__ float static_quotient(float a, float s, float r) {
#ifdef __CUDA_ARCH__
  if (kFast) {
    const float q0 = __fmul_rn(a, r);
    const float q = __fmaf_rn(__fmaf_rn(-q0, s, a), r, q0);
    return q0 < 1024.0f ? q : q0;
  }
  return __fdiv_rn(a, s);
#else
  if (kFast) {
    const float q0 = a * r;
    const float q = std::fmaf(std::fmaf(-q0, s, a), r, q0);
    return q0 < 1024.0f ? q : q0;
  }
  return a / s;
#endif
}

// The window of given scales in which static_quotient<true> is exact.
__host__ __device__ __forceinline__ bool static_scale_fast(float s) { return s >= 0x1p-92f && s <= 0x1p126f; }

template <int FMT>
__device__ __forceinline__ uint2 quant8(const uint4& v, const GroupScale& g) {
  return make_uint2(quant4<FMT>(v.x, v.y, g), quant4<FMT>(v.z, v.w, g));
}

// ---------------------------------------------------------------------------
// Activation quantization.  Eight lanes per 128-element group, 16 elements
// (two 16-byte loads) per lane, UNROLL groups in flight per lane group, over
// the M*K/128 groups in row-major order.  The host sizes the grid to cover
// every group in one pass where it can; the loop strides over what a capped
// grid leaves, and never wraps past the 32-bit group count.
// X bf16 [M, K] row stride ldx  ->  Xq u8 [M, K] row stride K,
// scales Xs[g * ld_s + m] (fp32 or UE8M0 byte).
// ---------------------------------------------------------------------------
template <int FMT, int UNROLL>
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ X, uint32_t M, uint32_t K,
                                                        uint64_t ldx, uint8_t* __restrict__ Xq,
                                                        void* __restrict__ Xs, uint64_t ld_s, FastDiv kb_div) {
  // a GEMM launched after this kernel with programmatic serialization may be
  // scheduled now; it waits for this grid's completion before reading Xq / Xs
  griddep_launch_dependents();
  const uint32_t total = M * kb_div.d;
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t sub = lane & 7u;
  const uint32_t gmask = 0xFFu << (lane & 24u);            // the 8 lanes sharing a group
  const uint32_t grp = (blockIdx.x * blockDim.x + threadIdx.x) >> 3;
  const uint32_t ngrp = (gridDim.x * blockDim.x) >> 3;
  const uint32_t step = ngrp * UNROLL;

  for (uint32_t base = grp; base < total; base = (total - base > step) ? base + step : total) {
    uint4 v[UNROLL][2];
    uint32_t m[UNROLL], g[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const uint32_t gi = base + u * ngrp;
      if (gi < total) {
        m[u] = kb_div.div(gi);
        g[u] = gi - m[u] * kb_div.d;
        const uint16_t* src = X + m[u] * ldx + g[u] * kGroup + sub * 16u;
        v[u][0] = ld_stream_v4(src);
        v[u][1] = ld_stream_v4(src + 8);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const uint32_t gi = base + u * ngrp;
      if (gi < total) {
        uint32_t a = max(absmax_bits8(v[u][0]), absmax_bits8(v[u][1]));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(gmask, a, o));
        const GroupScale gs = make_scale<FMT>(a);
        uint4 codes;
        codes.x = quant4<FMT>(v[u][0].x, v[u][0].y, gs);
        codes.y = quant4<FMT>(v[u][0].z, v[u][0].w, gs);
        codes.z = quant4<FMT>(v[u][1].x, v[u][1].y, gs);
        codes.w = quant4<FMT>(v[u][1].z, v[u][1].w, gs);
        FGFP8_DCHECK(m[u] < M && g[u] < kb_div.d);
        *reinterpret_cast<uint4*>(Xq + static_cast<uint64_t>(m[u]) * K + g[u] * kGroup + sub * 16u) = codes;
        if (sub == 0) {
          const uint64_t si = static_cast<uint64_t>(g[u]) * ld_s + m[u];
          if (FMT == 0) reinterpret_cast<float*>(Xs)[si] = gs.s;
          else reinterpret_cast<uint8_t*>(Xs)[si] = static_cast<uint8_t>(gs.e8);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Activation quantization in the masked expert layout: expert e's tokens are
// rows [e * cap, e * cap + counts[e]) of X; only those rows are quantized
// (the padding rows' codes and scales are left as they are: the masked GEMM
// loads whole 128-row tiles, padding rows included, but every output row
// depends on its own input row only and rows past the count are never
// stored).  blockIdx.y = expert; the blocks of an expert stride over its
// count * K/128 groups, 8 lanes per group as above.  A count outside
// [0, cap] is clamped to it here and recorded in the status word
// (kDevBadGroupOffsets), as the masked GEMM does.
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(256) quant_act_masked_kernel(const uint16_t* __restrict__ X,
                                                               const int32_t* __restrict__ counts, uint32_t cap,
                                                               uint32_t K, uint64_t ldx, uint8_t* __restrict__ Xq,
                                                               void* __restrict__ Xs, uint64_t ld_s, FastDiv kb_div) {
  griddep_launch_dependents();
  const uint32_t e = blockIdx.y;
  const int32_t c = __ldg(counts + e);
  if ((c < 0 || static_cast<uint32_t>(c) > cap) && blockIdx.x == 0 && threadIdx.x == 0)
    record_status(kDevBadGroupOffsets);
  const uint32_t rows = c <= 0 ? 0u : (static_cast<uint32_t>(c) < cap ? static_cast<uint32_t>(c) : cap);
  const uint32_t total = rows * kb_div.d;
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t sub = lane & 7u;
  const uint32_t gmask = 0xFFu << (lane & 24u);
  const uint32_t row0 = e * cap;
  const uint32_t gstep = (gridDim.x * blockDim.x) >> 3;
  // the increment never wraps past the 32-bit count (a wrapped index would
  // restart the pass)
  for (uint32_t gi = (blockIdx.x * blockDim.x + threadIdx.x) >> 3; gi < total;
       gi = (total - gi > gstep) ? gi + gstep : total) {
    const uint32_t r = kb_div.div(gi);
    const uint32_t g = gi - r * kb_div.d;
    const uint32_t m = row0 + r;
    const uint16_t* src = X + m * ldx + g * kGroup + sub * 16u;
    const uint4 v0 = ld_stream_v4(src), v1 = ld_stream_v4(src + 8);
    uint32_t a = max(absmax_bits8(v0), absmax_bits8(v1));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(gmask, a, o));
    const GroupScale gs = make_scale<FMT>(a);
    uint4 codes;
    codes.x = quant4<FMT>(v0.x, v0.y, gs);
    codes.y = quant4<FMT>(v0.z, v0.w, gs);
    codes.z = quant4<FMT>(v1.x, v1.y, gs);
    codes.w = quant4<FMT>(v1.z, v1.w, gs);
    FGFP8_DCHECK(r < cap && g < kb_div.d);
    *reinterpret_cast<uint4*>(Xq + static_cast<uint64_t>(m) * K + g * kGroup + sub * 16u) = codes;
    if (sub == 0) {
      const uint64_t si = static_cast<uint64_t>(g) * ld_s + m;
      if (FMT == 0) reinterpret_cast<float*>(Xs)[si] = gs.s;
      else reinterpret_cast<uint8_t*>(Xs)[si] = static_cast<uint8_t>(gs.e8);
    }
  }
}

// ---------------------------------------------------------------------------
// Weight quantization.  One 256-thread CTA per 128x128 block: half-warp h
// owns rows h, h+16, ..., h+112 of the block; every thread keeps its eight
// 16-byte chunks in registers across the block-wide amax reduction.
// W bf16 [N, K] row stride ldw -> Wq u8 [N, K] row stride K,
// Ws[nb * KB + kb] (row-major [N/128, K/128]).
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t* __restrict__ W, uint32_t K,
                                                           uint64_t ldw, uint8_t* __restrict__ Wq,
                                                           void* __restrict__ Ws, FastDiv kb_div) {
  __shared__ uint32_t s_max[8];
  const uint32_t blk = blockIdx.x;
  const uint32_t nb = kb_div.div(blk);
  const uint32_t kb = blk - nb * kb_div.d;
  const uint32_t t = threadIdx.x;
  const uint32_t h = t >> 4, sub = t & 15u;
  const uint64_t row0 = static_cast<uint64_t>(nb) * kGroup;
  const uint32_t col = kb * kGroup + sub * 8u;

  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = ld_stream_v4(W + (row0 + h + 16u * i) * ldw + col);
  uint32_t a = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = max(a, absmax_bits8(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if ((t & 31u) == 0) s_max[t >> 5] = a;
  __syncthreads();
  a = s_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) a = max(a, s_max[i]);

  const GroupScale gs = make_scale<FMT>(a);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint2 codes = quant8<FMT>(v[i], gs);
    *reinterpret_cast<uint2*>(Wq + (row0 + h + 16u * i) * K + col) = codes;
  }
  if (t == 0) {
    if (FMT == 0) reinterpret_cast<float*>(Ws)[blk] = gs.s;
    else reinterpret_cast<uint8_t*>(Ws)[blk] = static_cast<uint8_t>(gs.e8);
  }
}

// ---------------------------------------------------------------------------
// Row and tensor scale granularity ("FP8 W8A8", "Applying quantization": the
// FP8_DYNAMIC scheme, per-output-channel weights and per-token activations;
// static per-tensor AbsMax scales).  The scale and code rules are those of
// the 1x128 groups above, with the group widened to a whole row of K or to
// the whole tensor; scales are fp32.
// ---------------------------------------------------------------------------

// One CTA of kRowThreads per row r of X [R, K]: pass 1 takes the row's amax
// (the first kRowRegChunks 16-byte chunks of each thread stay in registers),
// the CTA reduces it, pass 2 writes the codes (chunks beyond the register
// cache are read again, from L2).  Thread 0 stores the row's scale.
constexpr int kRowThreads = 256;
constexpr int kRowRegChunks = 8;     // rows up to 256 * 8 * 8 = 16384 elements in one read

__global__ void __launch_bounds__(kRowThreads) quant_rows_kernel(const uint16_t* __restrict__ X, uint32_t K,
                                                                 uint64_t ldx, uint8_t* __restrict__ Xq,
                                                                 float* __restrict__ scales) {
  __shared__ uint32_t s_max[kRowThreads / 32];
  griddep_launch_dependents();
  const uint32_t r = blockIdx.x;
  const uint16_t* xr = X + static_cast<uint64_t>(r) * ldx;
  uint8_t* qr = Xq + static_cast<uint64_t>(r) * K;
  const uint32_t chunks = K / 8;                       // 16-byte chunks in the row
  uint4 v[kRowRegChunks];
  uint32_t a = 0;
#pragma unroll
  for (int i = 0; i < kRowRegChunks; ++i) {
    const uint32_t c = threadIdx.x + i * kRowThreads;
    if (c < chunks) {
      v[i] = ld_stream_v4(xr + c * 8u);
      a = max(a, absmax_bits8(v[i]));
    }
  }
  for (uint32_t c = threadIdx.x + kRowRegChunks * kRowThreads; c < chunks; c += kRowThreads)
    a = max(a, absmax_bits8(ld_stream_v4(xr + c * 8u)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if ((threadIdx.x & 31u) == 0) s_max[threadIdx.x >> 5] = a;
  __syncthreads();
  a = s_max[0];
#pragma unroll
  for (int i = 1; i < kRowThreads / 32; ++i) a = max(a, s_max[i]);
  const GroupScale gs = make_scale<0>(a);
#pragma unroll
  for (int i = 0; i < kRowRegChunks; ++i) {
    const uint32_t c = threadIdx.x + i * kRowThreads;
    if (c < chunks) *reinterpret_cast<uint2*>(qr + c * 8u) = quant8<0>(v[i], gs);
  }
  for (uint32_t c = threadIdx.x + kRowRegChunks * kRowThreads; c < chunks; c += kRowThreads)
    *reinterpret_cast<uint2*>(qr + c * 8u) = quant8<0>(ld_stream_v4(xr + c * 8u), gs);
  if (threadIdx.x == 0) scales[r] = gs.s;
}

// Rows of up to kWarpRowChunks * 32 * 8 = 4096 elements: one warp per row,
// eight rows per CTA, every chunk held in registers between the warp's amax
// reduction and the codes.  Same arithmetic as quant_rows_kernel.
constexpr int kWarpRowChunks = 16;

__global__ void __launch_bounds__(256) quant_rows_warp_kernel(const uint16_t* __restrict__ X, uint32_t R,
                                                              uint32_t K, uint64_t ldx, uint8_t* __restrict__ Xq,
                                                              float* __restrict__ scales) {
  griddep_launch_dependents();
  const uint32_t r = blockIdx.x * 8u + (threadIdx.x >> 5);
  const uint32_t lane = threadIdx.x & 31u;
  if (r >= R) return;
  const uint16_t* xr = X + static_cast<uint64_t>(r) * ldx;
  uint8_t* qr = Xq + static_cast<uint64_t>(r) * K;
  const uint32_t chunks = K / 8;
  uint4 v[kWarpRowChunks];
  uint32_t a = 0;
#pragma unroll
  for (int i = 0; i < kWarpRowChunks; ++i) {
    const uint32_t c = lane + i * 32u;
    if (c < chunks) {
      v[i] = ld_stream_v4(xr + c * 8u);
      a = max(a, absmax_bits8(v[i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  const GroupScale gs = make_scale<0>(a);
#pragma unroll
  for (int i = 0; i < kWarpRowChunks; ++i) {
    const uint32_t c = lane + i * 32u;
    if (c < chunks) *reinterpret_cast<uint2*>(qr + c * 8u) = quant8<0>(v[i], gs);
  }
  if (lane == 0) scales[r] = gs.s;
}

// amax over a whole tensor: each thread folds 16-byte chunks of its
// grid-stride share, the warp reduces, lane 0 raises *amax_bits (bf16
// magnitude bits; NaN patterns order above infinity) with atomicMax.
// *amax_bits must be zero beforehand.
__global__ void __launch_bounds__(256) tensor_amax_kernel(const uint16_t* __restrict__ X, uint32_t R, uint32_t K,
                                                          uint64_t ldx, FastDiv chunk_div,
                                                          uint32_t* __restrict__ amax_bits) {
  const uint32_t total = R * chunk_div.d;              // 16-byte chunks
  uint32_t a = 0;
  const uint32_t istep = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i = (total - i > istep) ? i + istep : total) {
    const uint32_t row = chunk_div.div(i);
    const uint32_t c = i - row * chunk_div.d;
    a = max(a, absmax_bits8(ld_stream_v4(X + static_cast<uint64_t>(row) * ldx + c * 8u)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if ((threadIdx.x & 31u) == 0 && a != 0u) atomicMax(amax_bits, a);
}

// The tensor's scale from its amax bits, in place: the word holding the
// bits becomes the fp32 scale max(amax, 1e-4) / 448.
__global__ void tensor_scale_finish_kernel(uint32_t* __restrict__ word) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    const GroupScale gs = make_scale<0>(*word);
    *reinterpret_cast<float*>(word) = gs.s;
  }
}

// Static quantization with a given fp32 scale *scale (device):
// code = E4M3(x / scale) over X [R, K], 16 bytes of input per thread step.
// A scale that is not positive (<= 0 or NaN) is rejected: nothing is
// written and the status word records kDevBadScale.  +inf is a valid scale
// (every code becomes a signed zero).
template <bool kFast>
__device__ __forceinline__ void quant_static_run(const uint16_t* __restrict__ X, uint32_t R, uint64_t ldx, uint32_t K,
                                                 const FastDiv& chunk_div, float s, uint8_t* __restrict__ Xq) {
  const float r = kFast ? __frcp_rn(s) : 0.0f;
  const auto div = [s, r](float x) { return static_quotient<kFast>(fabsf(x), s, r); };
  const uint32_t total = R * chunk_div.d;
  const uint32_t istep = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i = (total - i > istep) ? i + istep : total) {
    const uint32_t row = chunk_div.div(i);
    const uint32_t c = i - row * chunk_div.d;
    const uint4 v = ld_stream_v4(X + static_cast<uint64_t>(row) * ldx + c * 8u);
    *reinterpret_cast<uint2*>(Xq + static_cast<uint64_t>(row) * K + c * 8u) =
        make_uint2(quant4_by(v.x, v.y, div), quant4_by(v.z, v.w, div));
  }
}

__global__ void __launch_bounds__(256) quant_static_kernel(const uint16_t* __restrict__ X, uint32_t R, uint32_t K,
                                                           uint64_t ldx, FastDiv chunk_div,
                                                           const float* __restrict__ scale,
                                                           uint8_t* __restrict__ Xq) {
  griddep_launch_dependents();
  const float s = __ldg(scale);
  if (!(s > 0.0f)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(kDevBadScale);
    return;
  }
  if (static_scale_fast(s)) quant_static_run<true>(X, R, ldx, K, chunk_div, s, Xq);
  else quant_static_run<false>(X, R, ldx, K, chunk_div, s, Xq);
}

}  // namespace fgfp8
