/*
 * Plain CPU oracle for fine-grained FP8 W8A8 linear layers.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * What it computes (sources are the pages "Fine-grained FP8" (Transformers
 * docs, Korean and Arabic copies) and "FP8 W8A8" (vLLM docs)):
 *   - OCP FP8 E4M3FN: 1 sign, 4 exponent, 3 mantissa bits, largest finite
 *     value 448, a NaN and no infinity ("FP8 W8A8", section "Two FP8
 *     representations").
 *   - weights quantized to 8 bits per 2-D block of 128x128, activations per
 *     token in groups of 128 along the input-channel axis, matching the weight
 *     block ("Fine-grained FP8", introduction).
 *   - dynamic activation scales ("Fine-grained FP8", "DeepGEMM fast path").
 *   - scales stored as float32 or as packed float8_e8m0fnu (UE8M0, value
 *     2^(e-127)) ("Fine-grained FP8", "UE8M0 scale format").
 *   - the block-scaled GEMM applies both scales per 128-wide K block.
 * Every step the pages leave open is fixed in the design notes; the choices
 * made here are: scale = amax/448 (one IEEE fp32 division), amax clamped
 * below at 1e-4, UE8M0 scale = the smallest power of two >= amax/448,
 * codes = round-to-nearest-even with saturation to +-448 of (x / scale).
 *
 * Arithmetic: decoding and the GEMM run in fp64.  The quantizer runs in
 * fp32 because the method fixes fp32 scales and an fp32 quotient.  Build
 * with -O2 -ffp-contract=off and without fast-math so every fp32 operation
 * is a single IEEE round-to-nearest operation.
 *
 * Parity pins for every function live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_GROUP 128          /* K group / block edge, "Fine-grained FP8" */
#define ORC_E4M3_MAX 448.0     /* "FP8 W8A8", "Two FP8 representations" */
#define ORC_AMAX_FLOOR 1e-4f   /* reading of the pages: all-zero groups */

enum { ORC_SCALE_F32 = 0, ORC_SCALE_UE8M0 = 1 };

/* ------------------------------------------------------------------ */
/* bf16 and E4M3 codecs                                                */
/* ------------------------------------------------------------------ */

/* bf16 is the top half of an fp32 bit pattern, so widening is exact. */
static float bf16_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Value of an E4M3FN code s.eeee.mmm.
 *   e == 0           : subnormal, (-1)^s * 2^-6 * m/8
 *   e == 15, m == 7  : NaN (no infinities in the fn variant)
 *   otherwise        : (-1)^s * 2^(e-7) * (1 + m/8)               */
double orc_e4m3_decode(uint8_t code) {
    int s = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Values of the non-negative finite codes 0x00..0x7E, in increasing order
 * (the E4M3 encoding is monotonic in its low 7 bits).  Filled at load time
 * from orc_e4m3_decode. */
static double pos_value[0x7F];

__attribute__((constructor)) static void fill_pos_value(void) {
    for (int c = 0; c < 0x7F; ++c) pos_value[c] = orc_e4m3_decode((uint8_t)c);
}

/* Nearest E4M3FN code to v: NaN -> 0x7F; |v| clamped to 448 (saturation);
 * otherwise round to the nearest representable value, ties to the code with
 * an even mantissa, subnormals kept (no flush to zero); the sign of v is kept,
 * so -0 and small negatives give 0x80.
 *
 * Method: bracket |v| between two consecutive codes of the sorted table by
 * binary search and compare the two distances exactly in fp64 (every E4M3
 * value and every fp32 input is exact in fp64, and so are their differences,
 * which are multiples of 2^-149 below 2^9). */
uint8_t orc_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= ORC_E4M3_MAX) return sign | 0x7E;
    /* largest code lo with pos_value[lo] <= a; pos_value[0] == 0 <= a */
    int lo = 0, hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (pos_value[mid] <= a) lo = mid;
        else hi = mid - 1;
    }
    if (lo == 0x7E) return sign | 0x7E;
    int up = lo + 1;
    double dlo = a - pos_value[lo];
    double dup = pos_value[up] - a;
    int pick;
    if (dlo < dup) pick = lo;
    else if (dup < dlo) pick = up;
    else pick = (lo % 2 == 0) ? lo : up;   /* tie: even mantissa LSB */
    return sign | (uint8_t)pick;
}

/* ------------------------------------------------------------------ */
/* Scales                                                              */
/* ------------------------------------------------------------------ */

/* amax over n bf16 values; a NaN anywhere makes the result NaN; the result is
 * raised to 1e-4 when smaller (keeps an all-zero group's scale finite). */
static float amax_clamped(const uint16_t* x, int64_t n, int64_t stride_rows,
                          int64_t rows) {
    float amax = 0.0f;
    int nan_seen = 0;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < n; ++i) {
            float a = fabsf(bf16_to_float(x[r * stride_rows + i]));
            if (isnan(a)) nan_seen = 1;
            else if (a > amax) amax = a;
        }
    if (nan_seen) return NAN;
    if (amax < ORC_AMAX_FLOOR) amax = ORC_AMAX_FLOOR;
    return amax;
}

/* fp32 scale: amax / 448 as one IEEE fp32 division. */
float orc_scale_f32(float amax_c) { return amax_c / 448.0f; }

/* UE8M0 scale byte: t = amax/448 (fp32), then the smallest power of two
 * 2^(e-127) with 2^(e-127) >= t.  frexpf gives t = f * 2^x with f in
 * [0.5, 1); t is a power of two exactly when f == 0.5, i.e. t = 2^(x-1).
 * A non-finite t gives 0xFF (the e8m0 NaN). */
uint8_t orc_scale_ue8m0(float amax_c) {
    float t = amax_c / 448.0f;
    if (!isfinite(t)) return 0xFF;
    int x;
    float f = frexpf(t, &x);
    int p = (f == 0.5f) ? x - 1 : x;      /* ceil(log2 t) */
    int e = p + 127;
    if (e < 0) e = 0;                     /* unreachable with the 1e-4 floor */
    if (e > 254) e = 254;
    return (uint8_t)e;
}

/* Value of a UE8M0 byte, 2^(e-127); 0xFF is NaN. */
double orc_ue8m0_decode(uint8_t e) {
    if (e == 0xFF) return NAN;
    return ldexp(1.0, (int)e - 127);
}

/* Quantize n values with the scale of their group: q = e4m3(x / s). */
static void quantize_run(const uint16_t* x, int64_t n, float s, uint8_t* q) {
    for (int64_t i = 0; i < n; ++i) q[i] = orc_e4m3_encode(bf16_to_float(x[i]) / s);
}

/* scale value used to divide: fp32 scale as is, UE8M0 as an exact power of
 * two in fp32 (2^(e-127) is a normal fp32 for 1 <= e <= 254). */
static float scale_value(float amax_c, int fmt, float* out_f32, uint8_t* out_e8) {
    if (fmt == ORC_SCALE_F32) {
        float s = orc_scale_f32(amax_c);
        *out_f32 = s;
        return s;
    }
    uint8_t e = orc_scale_ue8m0(amax_c);
    *out_e8 = e;
    if (e == 0xFF) return NAN;
    return ldexpf(1.0f, (int)e - 127);
}

/* ------------------------------------------------------------------ */
/* Activation quantization: per token, groups of 128 along K            */
/* X bf16 [M, K] (row stride ldx) -> Xq u8 [M, K] (row stride K)          */
/* scales MN-major: Xs[g * ld_s + m], g = k / 128                          */
/* ------------------------------------------------------------------ */
void orc_quant_act(const uint16_t* X, int64_t M, int64_t K, int64_t ldx,
                   uint8_t* Xq, void* Xs, int64_t ld_s, int fmt) {
    int64_t KB = K / ORC_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < KB; ++g) {
            const uint16_t* xg = X + m * ldx + g * ORC_GROUP;
            float amax_c = amax_clamped(xg, ORC_GROUP, 0, 1);
            float sf = 0.0f;
            uint8_t se = 0;
            float s = scale_value(amax_c, fmt, &sf, &se);
            if (fmt == ORC_SCALE_F32) ((float*)Xs)[g * ld_s + m] = sf;
            else ((uint8_t*)Xs)[g * ld_s + m] = se;
            quantize_run(xg, ORC_GROUP, s, Xq + m * K + g * ORC_GROUP);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Weight quantization: 128x128 blocks                                  */
/* W bf16 [N, K] (row stride ldw) -> Wq u8 [N, K] (row stride K)          */
/* scales Ws[nb * KB + kb] (row-major [N/128, K/128])                      */
/* ------------------------------------------------------------------ */
void orc_quant_weight(const uint16_t* W, int64_t N, int64_t K, int64_t ldw,
                      uint8_t* Wq, void* Ws, int fmt) {
    int64_t NB = N / ORC_GROUP, KB = K / ORC_GROUP;
#pragma omp parallel for schedule(static) collapse(2)
    for (int64_t nb = 0; nb < NB; ++nb) {
        for (int64_t kb = 0; kb < KB; ++kb) {
            const uint16_t* blk = W + nb * ORC_GROUP * ldw + kb * ORC_GROUP;
            float amax_c = amax_clamped(blk, ORC_GROUP, ldw, ORC_GROUP);
            float sf = 0.0f;
            uint8_t se = 0;
            float s = scale_value(amax_c, fmt, &sf, &se);
            if (fmt == ORC_SCALE_F32) ((float*)Ws)[nb * KB + kb] = sf;
            else ((uint8_t*)Ws)[nb * KB + kb] = se;
            for (int64_t r = 0; r < ORC_GROUP; ++r)
                quantize_run(blk + r * ldw, ORC_GROUP, s,
                             Wq + (nb * ORC_GROUP + r) * K + kb * ORC_GROUP);
        }
    }
}

static double scale_at(const void* S, int64_t idx, int fmt) {
    if (fmt == ORC_SCALE_F32) return (double)((const float*)S)[idx];
    return orc_ue8m0_decode(((const uint8_t*)S)[idx]);
}

/* ------------------------------------------------------------------ */
/* Dequantization (fp64): x_hat = decode(q) * scale                     */
/* ------------------------------------------------------------------ */
void orc_dequant_act(const uint8_t* Xq, const void* Xs, int64_t ld_s, int64_t M,
                     int64_t K, int fmt, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k)
            out[m * K + k] = orc_e4m3_decode(Xq[m * K + k]) *
                             scale_at(Xs, (k / ORC_GROUP) * ld_s + m, fmt);
}

void orc_dequant_weight(const uint8_t* Wq, const void* Ws, int64_t N, int64_t K,
                        int fmt, double* out) {
    int64_t KB = K / ORC_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = orc_e4m3_decode(Wq[n * K + k]) *
                             scale_at(Ws, (n / ORC_GROUP) * KB + k / ORC_GROUP, fmt);
}

/* ------------------------------------------------------------------ */
/* Block-scaled GEMM                                                    */
/*   P_kb[m,n] = sum_{k in block kb} e4m3(Xq[m,k]) * e4m3(Wq[n,k])  (exact) */
/*   Y[m,n]    = sum_kb Xs[m,kb] * Ws[n/128,kb] * P_kb[m,n]   (ascending kb) */
/*   S[m,n]    = sum_k |x_hat[m,k] * w_hat[n,k]|                           */
/* Each product of two E4M3 values is a multiple of 2^-18 below 2^18 and   */
/* has at most 8 significant bits, so a 128-term block sum needs at most   */
/* 44 bits: P_kb is exact in fp64 whatever the summation order.            */
/* rows: the output rows to compute (row indices into Xq), nrows of them;  */
/* Y and S are [nrows, N].                                                 */
/* ------------------------------------------------------------------ */
static void gemm_rows(const uint8_t* Xq, const void* Xs, int64_t ld_s,
                      const uint8_t* Wq, const void* Ws, int64_t N, int64_t K,
                      int fmt, const int64_t* rows, int64_t nrows, double* Y,
                      double* S, const int64_t* expert_of_row) {
    int64_t KB = K / ORC_GROUP, NB = N / ORC_GROUP;
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = orc_e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t m = rows[r];
        int64_t e = expert_of_row ? expert_of_row[r] : 0;
        const uint8_t* xr = Xq + m * K;
        const uint8_t* We = Wq + e * N * K;
        int64_t ws_off = e * NB * KB;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wr = We + n * K;
            double y = 0.0, sabs = 0.0;
            for (int64_t kb = 0; kb < KB; ++kb) {
                double p = 0.0, pabs = 0.0;
                for (int64_t k = kb * ORC_GROUP; k < (kb + 1) * ORC_GROUP; ++k) {
                    double prod = table[xr[k]] * table[wr[k]];
                    p += prod;
                    pabs += fabs(prod);
                }
                double sa = scale_at(Xs, kb * ld_s + m, fmt);
                double sw = scale_at(Ws, ws_off + (n / ORC_GROUP) * KB + kb, fmt);
                y += (sa * sw) * p;
                sabs += fabs(sa * sw) * pabs;
            }
            Y[r * N + n] = y;
            S[r * N + n] = sabs;
        }
    }
}

void orc_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s, const uint8_t* Wq,
              const void* Ws, int64_t N, int64_t K, int fmt, const int64_t* rows,
              int64_t nrows, double* Y, double* S) {
    gemm_rows(Xq, Xs, ld_s, Wq, Ws, N, K, fmt, rows, nrows, Y, S, 0);
}

/* M-grouped GEMM: row m belongs to expert e when offs[e] <= m < offs[e+1];
 * that row is multiplied by expert e's weights Wq[e] ([N, K]) with scales
 * Ws[e] ([N/128, K/128]).  Returns -1 for a requested row outside every
 * segment. */
int orc_grouped_gemm(const uint8_t* Xq, const void* Xs, int64_t ld_s,
                     const uint8_t* Wq, const void* Ws, const int32_t* offs,
                     int32_t E, int64_t N, int64_t K, int fmt, const int64_t* rows,
                     int64_t nrows, double* Y, double* S,
                     int64_t* expert_scratch) {
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t m = rows[r], e = -1;
        for (int32_t i = 0; i < E; ++i)
            if (offs[i] <= m && m < offs[i + 1]) { e = i; break; }
        if (e < 0) return -1;
        expert_scratch[r] = e;
    }
    gemm_rows(Xq, Xs, ld_s, Wq, Ws, N, K, fmt, rows, nrows, Y, S, expert_scratch);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Row and tensor scale granularity ("FP8 W8A8", "Applying quantization": */
/* the FP8_DYNAMIC scheme quantizes weights statically per output channel */
/* and activations dynamically per token; "Fine-grained FP8", "DeepGEMM   */
/* fast path", and the OwLite FP8 page's AbsMax per-tensor calibration:    */
/* static per-tensor scales).  Same scale and code rules as above, with   */
/* the group widened to a whole row of K, or to the whole tensor.         */
/* ------------------------------------------------------------------ */

/* One fp32 scale per row r of X [R, K]: s[r] = max(amax(row), 1e-4) / 448,
 * codes Xq[r, k] = e4m3(X[r, k] / s[r]). */
void orc_quant_rows(const uint16_t* X, int64_t R, int64_t K, int64_t ldx,
                    uint8_t* Xq, float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        const uint16_t* xr = X + r * ldx;
        float s = orc_scale_f32(amax_clamped(xr, K, 0, 1));
        scales[r] = s;
        quantize_run(xr, K, s, Xq + r * K);
    }
}

/* Per-tensor scale: max(amax over all R x K elements, 1e-4) / 448. */
float orc_tensor_scale(const uint16_t* X, int64_t R, int64_t K, int64_t ldx) {
    return orc_scale_f32(amax_clamped(X, K, ldx, R));
}

/* Static quantization with a given scale s: Xq = e4m3(X / s). */
void orc_quant_static(const uint16_t* X, int64_t R, int64_t K, int64_t ldx,
                      float s, uint8_t* Xq) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) quantize_run(X + r * ldx, K, s, Xq + r * K);
}

/* Row/column-scaled GEMM:
 *   Y[m,n] = sx[m] * sw[n] * sum_k e4m3(Xq[m,k]) * e4m3(Wq[n,k])
 * with sx[0] for every m when x_per_tensor, sw[0] for every n when
 * w_per_tensor.  The K sum is exact in fp64 for K < 2^17 (each product is a
 * multiple of 2^-18 below 2^18).  S[m,n] = sum_k |x_hat * w_hat|.  rows as
 * in orc_gemm. */
void orc_gemm_rowcol(const uint8_t* Xq, const float* sx, int x_per_tensor,
                     const uint8_t* Wq, const float* sw, int w_per_tensor,
                     int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                     double* Y, double* S) {
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = orc_e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t m = rows[r];
        const uint8_t* xr = Xq + m * K;
        double a = (double)sx[x_per_tensor ? 0 : m];
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wr = Wq + n * K;
            double p = 0.0, pabs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double prod = table[xr[k]] * table[wr[k]];
                p += prod;
                pabs += fabs(prod);
            }
            double c = a * (double)sw[w_per_tensor ? 0 : n];
            Y[r * N + n] = c * p;
            S[r * N + n] = fabs(c) * pabs;
        }
    }
}

/* bf16 round-to-nearest-even of an fp64 value, for reporting only. */
uint16_t orc_bf16_rne(double v) {
    if (isnan(v)) return 0x7FC0;
    /* value -> nearest fp32 (RNE), then fp32 -> nearest bf16 (RNE); doing it
     * in two steps can double-round, so round directly: scale into the bf16
     * grid of v's binade. */
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    int ex;
    frexp(a, &ex);                 /* a = f * 2^ex, f in [0.5,1) */
    int e = ex - 1;                /* a in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;        /* bf16 subnormal quantum 2^-133 */
    double quantum = ldexp(1.0, e - 7);
    double q = nearbyint(a / quantum) * quantum;  /* ties to even */
    float f = (float)q;            /* exact: q has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t h = (uint16_t)(u >> 16);   /* low half is zero (or overflowed to inf) */
    if (!isfinite(f)) h = 0x7F80;
    return (uint16_t)(h | (signbit(v) ? 0x8000 : 0));
}

/* ------------------------------------------------------------------ */
/* Array forms of the codecs (the same per-element functions, looped).  */
/* ------------------------------------------------------------------ */
void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_scale_f32_array(const float* amax_c, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_scale_f32(amax_c[i]);
}

void orc_scale_ue8m0_array(const float* amax_c, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_scale_ue8m0(amax_c[i]);
}

void orc_bf16_rne_array(const double* v, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_rne(v[i]);
}
