/*
 * lowbit_oracle.c -- the oracle for the low-bit-weight linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, scalar CPU statement of
 * what the GPU path computes: quantise -> pack -> unpack -> integer dot ->
 * rescale.  Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline
 * leg may load or call it.  It shares no code, header, table or constant with
 * the CUDA library; the two are written independently from the same pages:
 *
 *   [M8.8]   "M8.8 - Native Binary and Ternary Transformers"
 *            (transformer-system.numinens.com), sections 0x02C-0x02E, 0x05A-0x05D,
 *            0x06E, 0x09A-0x09C.
 *   [Atomic] "Atomic-1Bit" README, opening section (add/sub/skip rule) and the
 *            "Config presets" text (four ternary codes per byte).
 *   [T4NT]   "T4NT-0.5B" model card, "What is T4NT?" and the Architecture table
 *            (15 symmetric levels, tanh(w/3)*3 clipping).
 *   [Impeto] "Extreme DQT with an FP4 Optimizer", abstract and "Attention"
 *            (INT1 weights with INT8 activations).
 *
 * Floating point: built with -O2 -ffp-contract=off (no FMA contraction, no
 * fast-math).  Every float operation below is one IEEE-754 operation in the
 * stated precision, round-to-nearest-even, in the stated order.
 *
 * Parity status of each function (the pins live in tests/test_oracle_pins.py):
 *   orc_ternary_codes, orc_binary_codes, orc_int4_codes, orc_tanh,
 *   orc_act_quant_*, orc_int_dot, orc_rescale_*, orc_pack/unpack (binary),
 *   orc_binary_centred_codes, orc_fwht32, orc_act_prologue_*:
 *     pinned (closed forms, worked cases, library routines, brute force).
 *   orc_pack/orc_unpack for TERNARY2 and INT4: the pages fix "four codes per
 *     byte" and "two's complement" but not the order of codes inside a byte, so
 *     that order is "parity unpinned" (round-trip, alphabet, field encoding and
 *     reserved-pattern invariants pin the rest).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Status values.  The numbers are part of the library's documented contract
 * (include/lowbit.h states the same numbers); they are restated here, not
 * shared. */
enum {
    ORC_OK = 0,
    ORC_EINVAL = 1,
    ORC_EOVERFLOW = 4,
    ORC_ENONFINITE = 5,
    ORC_ERESERVED = 6,
};

enum { ORC_TERNARY2 = 0, ORC_BINARY1 = 1, ORC_INT4 = 2 };

/* ------------------------------------------------------------------------ */
/* Small helpers                                                             */
/* ------------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the high half of an fp32 bit pattern; widening is exact. */
float orc_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest even, from the IEEE bit definition: keep the
 * top 16 bits, add half of the dropped range, and break exact ties toward the
 * kept value whose lowest bit is 0.  NaN stays a quiet NaN with its sign. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u = bits_from_f32(f);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

static int finite_f32(float f) { return (bits_from_f32(f) & 0x7f800000u) != 0x7f800000u; }

/* ------------------------------------------------------------------------ */
/* tanh, written out for the 4-bit clipping 3*tanh(w/3) [T4NT]               */
/* ------------------------------------------------------------------------ */
/* The pages fix the clipping function but not how tanh is evaluated; a
 * last-bit difference in tanh can move a weight across a rounding boundary.
 * So the oracle evaluates tanh with its own fixed sequence of fp64 operations:
 *
 *   tanh(a) = e / (e + 2),  e = expm1(2a),  a >= 0, sign restored after;
 *   expm1(u): if u <= ln2/2, Taylor series sum_{n>=1} u^n/n! to n = 16,
 *             evaluated by Horner as u*(1 + u/2*(1 + u/3*(...)));
 *             else Cody-Waite reduction u = k*ln2 + r with ln2 split into a
 *             high part (21 trailing zero bits, so k*hi is exact) and a low
 *             part, expm1(u) = 2^k*(1 + expm1(r)) - 1;
 *   tanh(a) = 1 for a > 20 (1 - tanh(20) < 2^-55).
 *
 * Truncation after u^16/16! at |u| <= ln2/2 leaves < 2^-60 relative error. */
static const double ORC_LN2_HI = 0x1.62e42fee00000p-1;
static const double ORC_LN2_LO = 0x1.a39ef35793c76p-33;
static const double ORC_HALF_LN2 = 0x1.62e42fefa39efp-2; /* RN(ln 2) / 2 */

static double orc_expm1_series(double r)
{
    double p = 1.0;
    for (int n = 16; n >= 2; --n)
        p = 1.0 + (r * p) / (double)n;
    return r * p;
}

static double orc_expm1_nonneg(double u)
{
    if (u <= ORC_HALF_LN2)
        return orc_expm1_series(u);
    double k = rint(u / (ORC_LN2_HI + ORC_LN2_LO));
    double r = (u - k * ORC_LN2_HI) - k * ORC_LN2_LO;
    double p = orc_expm1_series(r);
    return ldexp(1.0 + p, (int)k) - 1.0;
}

double orc_tanh(double z)
{
    if (z != z) return z;
    double a = fabs(z);
    double t;
    if (a > 20.0) {
        t = 1.0;
    } else {
        double e = orc_expm1_nonneg(2.0 * a);
        t = e / (e + 2.0);
    }
    return z < 0 ? -t : t;
}

/* ------------------------------------------------------------------------ */
/* Weight quantisers                                                          */
/* ------------------------------------------------------------------------ */

/* Ternary absmean codes [M8.8 §0x05A, §0x05B]: gamma = mean|W| over the whole
 * tensor; Q = clip(round(W / (gamma + eps)), -1, 1), round = nearest-even; the
 * decode scale is gamma itself (scaled_ternary, §0x05B).
 * The sum is fp64, k ascending within a row, then rows ascending.  gamma is
 * the fp64 mean rounded once to fp32; the divide and round are fp32.
 * A zero denominator (all-zero tensor with eps = 0) gives all-zero codes. */
int orc_ternary_codes(const float *w, long N, long K, long ldw, float eps,
                      int8_t *codes, float *gamma_out)
{
    if (N <= 0 || K <= 0 || ldw < K || !(eps >= 0.0f) || !finite_f32(eps)) return ORC_EINVAL;
    double S = 0.0;
    for (long n = 0; n < N; ++n) {
        double r = 0.0;
        for (long k = 0; k < K; ++k) {
            float v = w[n * ldw + k];
            if (!finite_f32(v)) return ORC_ENONFINITE;
            r += fabs((double)v);
        }
        S += r;
    }
    float gamma = (float)(S / (double)(N * K));
    float d = gamma + eps;
    for (long n = 0; n < N; ++n)
        for (long k = 0; k < K; ++k) {
            int8_t c = 0;
            if (d != 0.0f) {
                float t = rintf(w[n * ldw + k] / d);
                c = (int8_t)(t > 1.0f ? 1 : (t < -1.0f ? -1 : (int)t));
            }
            codes[n * K + k] = c;
        }
    *gamma_out = gamma;
    return ORC_OK;
}

/* Binary sign codes with the total rule "+1 if w >= 0 else -1", so both signed
 * zeros give +1 [M8.8 §0x06E]; one scale per output row, s_w[n] = mean_k |W|
 * (the mean-absolute binary scale of §0x02B, taken per row).  fp64 sum, k
 * ascending, divided by K in fp64, rounded once to fp32. */
int orc_binary_codes(const float *w, long N, long K, long ldw, int8_t *codes, float *s_w)
{
    if (N <= 0 || K <= 0 || ldw < K) return ORC_EINVAL;
    for (long n = 0; n < N; ++n) {
        double r = 0.0;
        for (long k = 0; k < K; ++k) {
            float v = w[n * ldw + k];
            if (!finite_f32(v)) return ORC_ENONFINITE;
            r += fabs((double)v);
            codes[n * K + k] = (int8_t)(v >= 0.0f ? 1 : -1);
        }
        s_w[n] = (float)(r / (double)K);
    }
    return ORC_OK;
}

/* BitNet v1 centred binary codes [M8.8 §0x02B, §0x02E]: alpha = mean(W) over
 * the whole tensor, codes +1 where w - alpha > 0 and -1 otherwise (a weight
 * equal to the mean takes -1, the tie of the page's trace), and one scale per
 * tensor beta = mean|W|.  Both sums are fp64 in the ternary scale's fixed
 * order (k ascending within a row, then rows ascending), divided by N*K in
 * fp64 and rounded once to fp32.  The difference w - alpha of two fp32 values
 * is positive exactly when w > alpha, so the code is that comparison.
 * Writes alpha_out[0] and beta_out[0]. */
int orc_binary_centred_codes(const float *w, long N, long K, long ldw, int8_t *codes,
                             float *alpha_out, float *beta_out)
{
    if (N <= 0 || K <= 0 || ldw < K) return ORC_EINVAL;
    double S = 0.0, A = 0.0;
    for (long n = 0; n < N; ++n) {
        double r = 0.0, ra = 0.0;
        for (long k = 0; k < K; ++k) {
            float v = w[n * ldw + k];
            if (!finite_f32(v)) return ORC_ENONFINITE;
            r += (double)v;
            ra += fabs((double)v);
        }
        S += r;
        A += ra;
    }
    float alpha = (float)(S / (double)(N * K));
    float beta = (float)(A / (double)(N * K));
    for (long n = 0; n < N; ++n)
        for (long k = 0; k < K; ++k)
            codes[n * K + k] = (int8_t)(w[n * ldw + k] > alpha ? 1 : -1);
    *alpha_out = alpha;
    *beta_out = beta;
    return ORC_OK;
}

/* 4-bit symmetric codes [T4NT]: clip w_c = 3*tanh(w/3) (fp64, rounded once to
 * fp32), per row s_w[n] = max_k |w_c| / 7 (fp32), q = clip(round(w_c / s_w),
 * -7, 7) (fp32 divide, nearest-even), 15 levels.  A row whose scale is zero
 * gets zero codes. */
int orc_int4_codes(const float *w, long N, long K, long ldw, int8_t *codes, float *s_w)
{
    if (N <= 0 || K <= 0 || ldw < K) return ORC_EINVAL;
    float *wc = (float *)malloc(sizeof(float) * (size_t)K);
    if (!wc) return ORC_EINVAL;
    for (long n = 0; n < N; ++n) {
        float m = 0.0f;
        for (long k = 0; k < K; ++k) {
            float v = w[n * ldw + k];
            if (!finite_f32(v)) { free(wc); return ORC_ENONFINITE; }
            double z = (double)v / 3.0;
            wc[k] = (float)(3.0 * orc_tanh(z));
            float a = fabsf(wc[k]);
            if (a > m) m = a;
        }
        float s = m / 7.0f;
        s_w[n] = s;
        for (long k = 0; k < K; ++k) {
            int8_t c = 0;
            if (s != 0.0f) {
                float t = rintf(wc[k] / s);
                c = (int8_t)(t > 7.0f ? 7 : (t < -7.0f ? -7 : (int)t));
            }
            codes[n * K + k] = c;
        }
    }
    free(wc);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Packing                                                                    */
/* ------------------------------------------------------------------------ */
/* Row n of the artifact starts at byte n*ldp; bits past the logical extent of
 * a row are zero.
 *   BINARY1:  bit (k%8) of byte k/8 is (1 - c)/2, little-bit-first, i.e. bit 1
 *             means -1 [M8.8 §0x06E]; a row takes ceil(K/8) bytes.
 *   TERNARY2: four codes per byte [Atomic], as 2-bit two's-complement fields
 *             00 = 0, 01 = +1, 11 = -1, 10 reserved.  The pages do not fix the
 *             order of codes inside a byte; the layout here stores them plane by
 *             plane within each little-endian 32-bit word of 16 codes: code k
 *             lives in word k/16, byte (k%16)%4, field (k%16)/4, i.e. bits
 *             8*((k%16)%4) + 2*((k%16)/4) and the bit above.  A row takes
 *             4*ceil(K/16) bytes.
 *   INT4:     4-bit two's-complement fields, 1000 (-8) reserved (15 levels
 *             [T4NT]).  Same plane order: code k lives in word k/8, byte
 *             (k%8)%4, nibble (k%8)/4.  A row takes 4*ceil(K/8) bytes. */
static long code_bits(int fmt) { return fmt == ORC_TERNARY2 ? 2 : (fmt == ORC_BINARY1 ? 1 : 4); }

/* Bit position of code k inside its row. */
static long code_bit_pos(int fmt, long k)
{
    if (fmt == ORC_BINARY1) return k;
    long per_word = 32 / code_bits(fmt);
    long word = k / per_word, kk = k % per_word;
    return 32 * word + 8 * (kk % 4) + code_bits(fmt) * (kk / 4);
}

long orc_row_bytes(int fmt, long K)
{
    switch (fmt) {
    case ORC_TERNARY2: return 4 * ((K + 15) / 16);
    case ORC_BINARY1: return (K + 7) / 8;
    case ORC_INT4: return 4 * ((K + 7) / 8);
    default: return -1;
    }
}

int orc_pack(const int8_t *codes, long N, long K, int fmt, uint8_t *packed, long ldp)
{
    long rb = orc_row_bytes(fmt, K);
    if (N <= 0 || K <= 0 || rb < 0 || ldp < rb) return ORC_EINVAL;
    long cmax = (fmt == ORC_INT4) ? 7 : 1;
    uint32_t mask = (1u << code_bits(fmt)) - 1u;
    for (long n = 0; n < N; ++n) {
        uint8_t *row = packed + n * ldp;
        memset(row, 0, (size_t)ldp);
        for (long k = 0; k < K; ++k) {
            int c = codes[n * K + k];
            if (c < -cmax || c > cmax || (fmt == ORC_BINARY1 && c == 0)) return ORC_EINVAL;
            uint32_t field = (fmt == ORC_BINARY1) ? (uint32_t)((1 - c) / 2) : ((uint32_t)c & mask);
            long pos = code_bit_pos(fmt, k);
            row[pos / 8] |= (uint8_t)(field << (pos % 8));
        }
    }
    return ORC_OK;
}

/* Inverse of orc_pack.  Rejects a reserved pattern inside the logical extent
 * and any non-zero bit that no code owns [M8.8 §0x06E, §0x0BB "reserved
 * patterns reject"]. */
int orc_unpack(const uint8_t *packed, long ldp, long N, long K, int fmt, int8_t *codes)
{
    long rb = orc_row_bytes(fmt, K);
    if (N <= 0 || K <= 0 || rb < 0 || ldp < rb) return ORC_EINVAL;
    long b = code_bits(fmt);
    uint32_t mask = (1u << b) - 1u;
    uint8_t *owned = (uint8_t *)calloc((size_t)ldp * 8, 1);
    if (!owned) return ORC_EINVAL;
    int status = ORC_OK;
    for (long n = 0; n < N; ++n) {
        const uint8_t *row = packed + n * ldp;
        memset(owned, 0, (size_t)ldp * 8);
        for (long k = 0; k < K; ++k) {
            long pos = code_bit_pos(fmt, k);
            for (long j = 0; j < b; ++j) owned[pos + j] = 1;
            uint32_t f = (uint32_t)(row[pos / 8] >> (pos % 8)) & mask;
            int c;
            if (fmt == ORC_BINARY1) {
                c = f ? -1 : 1;
            } else if (f == (1u << (b - 1))) { /* 10 or 1000: reserved */
                status = ORC_ERESERVED;
                c = 0;
            } else {
                c = (f >= (1u << (b - 1))) ? (int)f - (int)(1u << b) : (int)f;
            }
            codes[n * K + k] = (int8_t)c;
        }
        for (long bit = 0; bit < ldp * 8; ++bit)
            if (!owned[bit] && ((row[bit / 8] >> (bit % 8)) & 1u)) status = ORC_ERESERVED;
    }
    free(owned);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Activation quantiser, per token absmax to int8 [M8.8 §0x05C]               */
/* ------------------------------------------------------------------------ */
/* gamma_t = max_k |x[t,k]| (fp32, exact in any order);
 * gamma_t == 0: q = 0, s_x = 0 (a zero row gives zero codes and scale);
 * else q = clip(round((x * 127) / (gamma_t + eps)), -128, 127) with an fp32
 * multiply, an fp32 divide and nearest-even rounding, and
 * s_x = gamma_t / 127 (the reconstruction scale leaves eps out, §0x05C).
 * A non-finite x, or an x*127 that overflows, returns ORC_ENONFINITE. */
static int act_quant_row(const float *x, long K, float eps, int8_t *q, float *s_x)
{
    float g = 0.0f;
    for (long k = 0; k < K; ++k) {
        if (!finite_f32(x[k]) || !finite_f32(x[k] * 127.0f)) return ORC_ENONFINITE;
        float a = fabsf(x[k]);
        if (a > g) g = a;
    }
    if (g == 0.0f) {
        for (long k = 0; k < K; ++k) q[k] = 0;
        *s_x = 0.0f;
        return ORC_OK;
    }
    float d = g + eps;
    for (long k = 0; k < K; ++k) {
        float t = rintf((x[k] * 127.0f) / d);
        q[k] = (int8_t)(t > 127.0f ? 127 : (t < -128.0f ? -128 : (int)t));
    }
    *s_x = g / 127.0f;
    return ORC_OK;
}

int orc_act_quant_f32(const float *x, long M, long K, long ldx, float eps,
                      int8_t *q, long ldq, float *s_x)
{
    if (M <= 0 || K <= 0 || ldx < K || ldq < K || !(eps >= 0.0f) || !finite_f32(eps))
        return ORC_EINVAL;
    int status = ORC_OK;
    for (long t = 0; t < M; ++t) {
        int st = act_quant_row(x + t * ldx, K, eps, q + t * ldq, s_x + t);
        if (st != ORC_OK) status = st;
    }
    return status;
}

int orc_act_quant_bf16(const uint16_t *x, long M, long K, long ldx, float eps,
                       int8_t *q, long ldq, float *s_x)
{
    if (M <= 0 || K <= 0 || ldx < K || ldq < K || !(eps >= 0.0f) || !finite_f32(eps))
        return ORC_EINVAL;
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    if (!row) return ORC_EINVAL;
    int status = ORC_OK;
    for (long t = 0; t < M; ++t) {
        for (long k = 0; k < K; ++k) row[k] = orc_bf16_to_f32(x[t * ldx + k]);
        int st = act_quant_row(row, K, eps, q + t * ldq, s_x + t);
        if (st != ORC_OK) status = st;
    }
    free(row);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Activation prologue: RMSNorm, gain, Hadamard rotation, per-token codes     */
/* ------------------------------------------------------------------------ */
/* Fast Walsh-Hadamard transform of one block of n = 2^p fp32 values, in place,
 * unnormalised: the radix-2 algorithm with stages h = 1, 2, 4, ..., n/2, each
 * replacing the pair (v[j], v[j+h]) of every 2h-block by (v[j] + v[j+h],
 * v[j] - v[j+h]) as two fp32 operations.  This is the O(n log n) transform the
 * BitNet v2 H-BitLinear applies online [M8.8 §0x07C]; its result is the
 * Sylvester-ordered Hadamard matrix H (H[i][j] = (-1)^popcount(i & j)) times
 * v, rounded by these fp32 steps. */
void orc_fwht32(float *v, long n)
{
    for (long h = 1; h < n; h *= 2)
        for (long i = 0; i < n; i += 2 * h)
            for (long j = i; j < i + h; ++j) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* The activation side of a BitLinear layer, row by row:
 *   1. RMSNorm with gain [M8.8 §0x02C-§0x02E and §0x03: normalise, then take the
 *      absmax codes; b1.58 and T4NT use RMSNorm]:  y = x * g / rms(x),
 *      rms(x) = sqrt(mean_k x_k^2 + eps_norm);  norm = 0 skips the division,
 *      so only the gain (the OneBit input value vector of §0x06A) applies;
 *   2. optionally the block Hadamard rotation of H-BitLinear [§0x07C]: blocks
 *      of hb consecutive features (hb a power of two dividing K), each
 *      multiplied by the normalised Walsh-Hadamard matrix H/sqrt(hb);
 *   3. per-token absmax int8 codes of the result [§0x05C], eps = 0.
 * The row factors 1/rms and 1/sqrt(hb) are positive and common to the whole
 * row, so they cancel in absmax codes: the codes are computed from
 *   u = FWHT(RN32(x_k * g_k)) (the fp32 transform above, or no transform),
 * by the per-token rule of act_quant_row, and the factors enter only the
 * scale, s_x = max|u| / sqrt(hb) / rms / 127, evaluated in fp64 (the sum of
 * squares k ascending) and rounded once to fp32.  g may be NULL (all ones).
 * A non-finite x or g, or a non-finite product or transform, returns
 * ORC_ENONFINITE. */
static int prologue_row(const float *xf, long K, const float *g, int norm, float eps_norm, long hb,
                        float *u, int8_t *q, float *s_x)
{
    for (long k = 0; k < K; ++k) {
        if (!finite_f32(xf[k]) || (g && !finite_f32(g[k]))) return ORC_ENONFINITE;
        u[k] = g ? xf[k] * g[k] : xf[k];
        if (!finite_f32(u[k])) return ORC_ENONFINITE;
    }
    if (hb > 0) {
        for (long b = 0; b < K; b += hb) orc_fwht32(u + b, hb);
        for (long k = 0; k < K; ++k)
            if (!finite_f32(u[k])) return ORC_ENONFINITE;
    }
    float s_unused;
    int st = act_quant_row(u, K, 0.0f, q, &s_unused);
    if (st != ORC_OK) return st;
    float gmax = 0.0f;
    for (long k = 0; k < K; ++k)
        if (fabsf(u[k]) > gmax) gmax = fabsf(u[k]);
    if (gmax == 0.0f) {
        *s_x = 0.0f;
        return ORC_OK;
    }
    double s = (double)gmax;
    if (hb > 0) s = s / sqrt((double)hb);
    if (norm) {
        double ss = 0.0;
        for (long k = 0; k < K; ++k) ss += (double)xf[k] * (double)xf[k];
        s = s / sqrt(ss / (double)K + (double)eps_norm);
    }
    *s_x = (float)(s / 127.0);
    return ORC_OK;
}

static int prologue_args_ok(long M, long K, long ldx, long ldq, int norm, float eps_norm, long hb)
{
    if (M <= 0 || K <= 0 || ldx < K || ldq < K || (norm != 0 && norm != 1)) return 0;
    if (!(eps_norm >= 0.0f) || !finite_f32(eps_norm)) return 0;
    if (hb < 0 || (hb > 0 && ((hb & (hb - 1)) != 0 || hb > K || K % hb != 0))) return 0;
    return 1;
}

int orc_act_prologue_f32(const float *x, long M, long K, long ldx, const float *g, int norm, float eps_norm,
                         long hb, int8_t *q, long ldq, float *s_x)
{
    if (!prologue_args_ok(M, K, ldx, ldq, norm, eps_norm, hb)) return ORC_EINVAL;
    float *u = (float *)malloc(sizeof(float) * (size_t)K);
    if (!u) return ORC_EINVAL;
    int status = ORC_OK;
    for (long t = 0; t < M; ++t) {
        int st = prologue_row(x + t * ldx, K, g, norm, eps_norm, hb, u, q + t * ldq, s_x + t);
        if (st != ORC_OK) status = st;
    }
    free(u);
    return status;
}

int orc_act_prologue_bf16(const uint16_t *x, long M, long K, long ldx, const float *g, int norm,
                          float eps_norm, long hb, int8_t *q, long ldq, float *s_x)
{
    if (!prologue_args_ok(M, K, ldx, ldq, norm, eps_norm, hb)) return ORC_EINVAL;
    float *row = (float *)malloc(sizeof(float) * (size_t)K);
    float *u = (float *)malloc(sizeof(float) * (size_t)K);
    if (!row || !u) { free(row); free(u); return ORC_EINVAL; }
    int status = ORC_OK;
    for (long t = 0; t < M; ++t) {
        for (long k = 0; k < K; ++k) row[k] = orc_bf16_to_f32(x[t * ldx + k]);
        int st = prologue_row(row, K, g, norm, eps_norm, hb, u, q + t * ldq, s_x + t);
        if (st != ORC_OK) status = st;
    }
    free(row);
    free(u);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Integer dot and rescale                                                    */
/* ------------------------------------------------------------------------ */
/* acc[t,n] = sum_k q[t,k] * c[n,k], in int64.  For ternary and binary codes it
 * is written as the add / subtract / skip rule [Atomic; M8.8 §0x05D]: c = +1
 * adds the activation, c = -1 subtracts it, c = 0 skips it.  4-bit codes
 * multiply.  The worst case |acc| <= 128 * cmax * K must fit int32
 * [M8.8 §0x09C]: K > INT32_MAX / (128 * cmax) returns ORC_EOVERFLOW.
 * Every (t, n) pair is independent; nthreads > 1 splits the pairs across
 * OpenMP threads without changing any result. */
int orc_int_dot(const int8_t *q, long ldq, const int8_t *codes, long M, long N, long K,
                int fmt, int64_t *acc, int nthreads)
{
    if (M <= 0 || N <= 0 || K <= 0 || ldq < K) return ORC_EINVAL;
    long cmax = (fmt == ORC_INT4) ? 7 : 1;
    if (K > 2147483647L / (128L * cmax)) return ORC_EOVERFLOW;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for collapse(2) schedule(static) num_threads(nthreads)
#endif
    for (long t = 0; t < M; ++t) {
        for (long n = 0; n < N; ++n) {
            const int8_t *qt = q + t * ldq;
            const int8_t *cn = codes + n * K;
            int64_t a = 0;
            if (fmt == ORC_INT4) {
                for (long k = 0; k < K; ++k) a += (int64_t)cn[k] * (int64_t)qt[k];
            } else {
                for (long k = 0; k < K; ++k) {
                    if (cn[k] == 1) a += qt[k];
                    else if (cn[k] == -1) a -= qt[k];
                }
            }
            acc[t * N + n] = a;
        }
    }
    return ORC_OK;
}

/* Rescale [M8.8 §0x02D, §0x09C]: y[t,n] = float(acc) * (s_w * s_x[t]), the two
 * scales multiplied first in fp32, then one fp32 multiply.  s_w has one entry
 * (sw_count == 1, per-tensor ternary scale) or one per output row. */
int orc_rescale_f32(const int64_t *acc, long M, long N, const float *s_w, long sw_count,
                    const float *s_x, float *y, long ldy)
{
    if (M <= 0 || N <= 0 || ldy < N || (sw_count != 1 && sw_count != N)) return ORC_EINVAL;
    for (long t = 0; t < M; ++t)
        for (long n = 0; n < N; ++n) {
            float sw = s_w[sw_count == 1 ? 0 : n];
            float sc = sw * s_x[t];
            y[t * ldy + n] = (float)acc[t * N + n] * sc;
        }
    return ORC_OK;
}

int orc_rescale_bf16(const int64_t *acc, long M, long N, const float *s_w, long sw_count,
                     const float *s_x, uint16_t *y, long ldy)
{
    if (M <= 0 || N <= 0 || ldy < N || (sw_count != 1 && sw_count != N)) return ORC_EINVAL;
    for (long t = 0; t < M; ++t)
        for (long n = 0; n < N; ++n) {
            float sw = s_w[sw_count == 1 ? 0 : n];
            float sc = sw * s_x[t];
            y[t * ldy + n] = orc_f32_to_bf16((float)acc[t * N + n] * sc);
        }
    return ORC_OK;
}

/* Number of threads OpenMP would use by default (reported beside timings). */
int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
