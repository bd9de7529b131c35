// Host-only checks of the integer / floating-point arithmetic the quantizers
// rely on (compiled with nvcc, run on the CPU):
//  1. FastDiv (Granlund-Montgomery) equals integer division for every
//     divisor 1..65536 on edge and random numerators;
//  2. the FMA-based quotient q = fma(fma(-q0, s, a), r, q0), q0 = a*r,
//     r = RN(1/s) equals the IEEE quotient RN(a/s) for EVERY pair the kernel
//     meets: a = |x| for a bf16 x, s = RN(amax_c/448) for a bf16 amax >= |x|
//     (amax_c = max(amax, 1e-4)), wherever the quotient can reach a nonzero
//     E4M3 code.  E4M3 rounds every |v| <= 2^-10 to zero (2^-10 is halfway to
//     the smallest subnormal 2^-9 and ties go to the even code 0), so below
//     that only "both quotients <= 2^-10" is required; there the FMA residual
//     of a subnormal |x| may be inexact.  Host fmaf/division/multiplication
//     are IEEE round-to-nearest, like the device intrinsics the kernel uses;
//  3. amax / 448 by the same FMA form with the constant RN(1/448);
//  4. the static quantizer's quotient for caller-given scales (below).
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <random>
#include <vector>

#include "quant.cuh"

static float bf16_bits_to_float(uint32_t h) {
  uint32_t u = h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

static uint32_t fbits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

int main() {
  long bad = 0;
  // ---- 1. FastDiv
  std::mt19937_64 rng(1);
  for (uint32_t d = 1; d <= 65536; ++d) {
    fgfp8::FastDiv f(d);
    const uint32_t edge[] = {0u, 1u, d - 1, d, d + 1, 2 * d - 1, 2 * d, 0x7FFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFEu};
    for (uint32_t n : edge)
      if (f.div(n) != n / d) ++bad;
    for (int i = 0; i < 64; ++i) {
      uint32_t n = static_cast<uint32_t>(rng());
      if (f.div(n) != n / d) ++bad;
    }
  }
  std::printf("fastdiv mismatches: %ld\n", bad);
  if (bad) return 1;

  // ---- 2. FMA-based quotient vs IEEE division, exhaustive over bf16 pairs
  long pairs = 0, qbad = 0, below = 0;
  const float zero_limit = 0x1p-10f;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, qbad, below)
  for (int64_t ab = 1; ab <= 0x7F7F; ++ab) {               // every positive finite bf16 amax
    const float amax = bf16_bits_to_float(static_cast<uint32_t>(ab));
    const float amax_c = amax < 1e-4f ? 1e-4f : amax;
    const float s = amax_c / 448.0f;
    const float r = 1.0f / s;
    for (uint32_t h = 0; h <= static_cast<uint32_t>(ab); ++h) {   // every |x| <= amax
      const float a = bf16_bits_to_float(h);
      const float q0 = a * r;
      const float e = std::fmaf(-q0, s, a);
      const float q = std::fmaf(e, r, q0);
      const float ref = a / s;
      ++pairs;
      if (q <= zero_limit && ref <= zero_limit) {
        ++below;                                   // both encode to a zero code
      } else if (fbits(q) != fbits(ref)) {
        ++qbad;
      }
    }
  }
  std::printf("quotient pairs: %ld (of which %ld both <= 2^-10) mismatches: %ld\n", pairs, below, qbad);
  if (qbad) return 2;

  // ---- 3. amax / 448 by the same FMA-based division with the constant
  //         r448 = RN(1/448), against IEEE division, for every positive bf16
  //         amax (finite and infinite) and the 1e-4 floor
  const float r448 = 1.0f / 448.0f;
  long sbad = 0;
  for (uint32_t ab = 1; ab <= 0x7F80; ++ab) {
    const float amax = bf16_bits_to_float(ab);
    const float a = amax < 1e-4f ? 1e-4f : amax;
    const float q0 = a * r448;
    const float e = std::fmaf(-q0, 448.0f, a);
    const float q = std::fmaf(e, r448, q0);
    const float ref = a / 448.0f;
    if (fbits(q) != fbits(ref) && !(std::isinf(ref) && std::isnan(q))) ++sbad;
  }
  std::printf("scale divisions checked: %u mismatches: %ld\n", 0x7F80u, sbad);
  if (sbad) return 3;

  // ---- 4. the static quantizer's quotient |x| / s for a caller-given scale
  //         s > 0 (fgfp8::static_quotient, the kernel's own function, with the
  //         kernel's choice of form), against IEEE division, for every bf16
  //         magnitude (+inf included) and a sweep of scales: every binade from
  //         the smallest subnormal 2^-149 to 2^127 at fixed and random
  //         mantissas, the ends of the FMA window and their neighbours, FLT_MAX,
  //         +inf, and random scales inside the window.  The code depends on the
  //         quotient only through E4M3 rounding with saturation, so a pair also
  //         passes when both quotients are <= 2^-10 (zero code) or both >= 448
  //         (saturated code, infinity included).
  std::vector<float> scales;
  auto from_bits = [](uint32_t u) {
    float f;
    std::memcpy(&f, &u, 4);
    return f;
  };
  std::mt19937 srng(7);
  for (int b = 0; b < 255; ++b) {                       // biased exponent 0 (subnormals) .. 254
    const uint32_t fixed[] = {0u, 1u, 0x400000u, 0x7FFFFFu, 0x12345u, 0x7FFFFEu};
    for (uint32_t m : fixed)
      if (b > 0 || m > 0) scales.push_back(from_bits((static_cast<uint32_t>(b) << 23) | m));
    for (int i = 0; i < 10; ++i) scales.push_back(from_bits((static_cast<uint32_t>(b) << 23) | (srng() & 0x7FFFFFu)));
  }
  for (float edge : {0x1p-92f, 0x1p126f}) {
    const uint32_t u = fbits(edge);
    for (uint32_t d = 0; d < 4; ++d) {
      scales.push_back(from_bits(u + d));
      scales.push_back(from_bits(u - d));
    }
  }
  scales.push_back(from_bits(0x7F7FFFFFu));             // FLT_MAX
  scales.push_back(from_bits(0x7F800000u));             // +inf
  std::uniform_int_distribution<uint32_t> win(fbits(0x1p-92f), fbits(0x1p126f));
  for (int i = 0; i < 4000; ++i) scales.push_back(from_bits(win(srng)));

  long spairs = 0, sq_bad = 0, fast_scales = 0;
#pragma omp parallel for schedule(dynamic, 8) reduction(+ : spairs, sq_bad, fast_scales)
  for (int64_t i = 0; i < static_cast<int64_t>(scales.size()); ++i) {
    const float sc = scales[i];
    const bool fast = fgfp8::static_scale_fast(sc);
    const float r = 1.0f / sc;
    if (fast) ++fast_scales;
    for (uint32_t h = 0; h <= 0x7F80u; ++h) {
      const float a = bf16_bits_to_float(h);
      const float q = fast ? fgfp8::static_quotient<true>(a, sc, r) : fgfp8::static_quotient<false>(a, sc, r);
      const float ref = a / sc;
      ++spairs;
      const bool same = fbits(q) == fbits(ref) || (std::isnan(q) && std::isnan(ref));
      const bool zero = q <= zero_limit && ref <= zero_limit;
      const bool sat = q >= 448.0f && ref >= 448.0f;
      if (!(same || zero || sat)) ++sq_bad;
    }
  }
  std::printf("static quotient pairs: %ld over %zu scales (%ld in the FMA window) mismatches: %ld\n", spairs,
              scales.size(), fast_scales, sq_bad);
  return sq_bad ? 4 : 0;
}
