/*
 * CPU oracle for fine-grained FP8 quantization -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the bench's CPU-baseline leg
 * may load this library.  It shares no code, header, table or constant with
 * the CUDA path; it is written from the definitions below, plainly and slowly.
 *
 * Sources (cited by site and paragraph of the post):
 *   - the-good.kr wr_id=2169793, para 4: E4M3 on all tensors; the maximum
 *     absolute value is computed online for every 1x128 activation tile or
 *     128x128 weight block, the scale maps that maximum to the largest FP8
 *     value, and the tile is quantized with it.
 *   - why-be.co.kr wr_id=72410, para 1: scaling factors that are integral
 *     powers of two (option `pow2`).
 *   - E4M3 itself (sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 *     infinities, S.1111.111 is NaN, largest finite 448) is the OCP 8-bit
 *     floating point format "E4M3FN"; the pages only name "E4M3".
 *
 * Readings taken where the pages are silent (each listed in the design notes):
 *   - rounding of the cast: nearest, ties to even; saturate to +-448;
 *   - s = fl32(amax / 448) with IEEE fp32 division; amax == 0 gives s = 1;
 *   - pow2: s becomes the smallest power of two >= s (so amax/s <= 448);
 *   - q = E4M3(fl32(x / s)): the fp32 quotient first, then the cast;
 *   - the sign of a value that rounds to zero is kept (-0 -> 0x80);
 *   - NaN encodes to 0x7F and is ignored by the amax (outside the contract).
 *
 * Build: plain C99, no fast-math (IEEE division and no flush-to-zero are
 * part of the definition).  The outer loops run over independent tiles and
 * may be spread over host threads with OpenMP; that changes no result.
 * See oracle/build.py.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define E4M3_MAX 448.0

/* ---------------------------------------------------------------------- */
/* E4M3 codec                                                              */
/* ---------------------------------------------------------------------- */

/* Value of an E4M3 byte as a double (exact). NaN codes return NaN. */
double orc_e4m3_decode(uint8_t c) {
    int sgn = c >> 7;
    int e = (c >> 3) & 0xF;
    int m = c & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);           /* subnormal: m * 2^-9 */
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return sgn ? -v : v;
}

/* Byte of an E4M3 magnitude that is exactly representable (0 <= a <= 448). */
static uint8_t e4m3_bits_of_exact(double a) {
    int ex;
    if (a == 0.0) return 0;
    if (a < ldexp(1.0, -6)) /* subnormal */
        return (uint8_t)(a / ldexp(1.0, -9));
    frexp(a, &ex);          /* a = f * 2^ex, f in [0.5, 1) -> a in [2^(ex-1), 2^ex) */
    {
        int E = ex - 1;
        int mant = (int)((a / ldexp(1.0, E) - 1.0) * 8.0);
        return (uint8_t)(((E + 7) << 3) | mant);
    }
}

/* E4M3 encoding of an fp32 value: round to nearest, ties to even, then saturate. */
uint8_t orc_e4m3_encode(float v) {
    uint8_t sgn;
    double a, quantum, n, r, val;
    int ex, E;
    if (isnan(v)) return 0x7F;
    sgn = signbit(v) ? 0x80 : 0x00;
    a = fabs((double)v);
    if (a == 0.0) return sgn;
    frexp(a, &ex);
    E = ex - 1;              /* a in [2^E, 2^(E+1)) */
    if (E < -6) E = -6;      /* the subnormal range shares the spacing of the first binade */
    quantum = ldexp(1.0, E - 3);
    n = a / quantum;         /* exact: division by a power of two */
    r = nearbyint(n);        /* default rounding mode: nearest, ties to even */
    val = r * quantum;       /* may carry into the next binade; still exact */
    if (val > E4M3_MAX) val = E4M3_MAX;
    return (uint8_t)(sgn | e4m3_bits_of_exact(val));
}

/* ---------------------------------------------------------------------- */
/* scales                                                                  */
/* ---------------------------------------------------------------------- */

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Smallest power of two >= s (s > 0, finite). */
static float pow2_ceil(float s) {
    int ex;
    double f = frexp((double)s, &ex); /* s = f * 2^ex, f in [0.5, 1) */
    return (float)(f == 0.5 ? (double)s : ldexp(1.0, ex));
}

/* Scale of a tile with maximum magnitude `amax`. */
float orc_scale_from_amax(float amax, int pow2) {
    float s;
    if (amax == 0.0f) return 1.0f;
    s = amax / 448.0f;       /* IEEE fp32 division */
    if (pow2) s = pow2_ceil(s);
    return s;
}

static float amax_update(float acc, float x) {
    float a = fabsf(x);
    return (a > acc) ? a : acc; /* a NaN x never wins */
}

/* ---------------------------------------------------------------------- */
/* 1x128 activation tiles                                                  */
/* ---------------------------------------------------------------------- */

/*
 * x: bf16 bits [M, K] with row stride ldx.  q: E4M3 [M, K] with row stride ldq.
 * s: fp32 scales, group-major: scale of (row m, group g) at s[g * ld_s + m].
 * K must be a multiple of 128.
 */
void orc_quant_act_1x128(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                         uint8_t* q, int64_t ldq, float* s, int64_t ld_s, int pow2) {
    int64_t G = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t* xr = x + m * ldx + g * 128;
            float amax = 0.0f, sc;
            for (int k = 0; k < 128; ++k) amax = amax_update(amax, bf16_to_f32(xr[k]));
            sc = orc_scale_from_amax(amax, pow2);
            for (int k = 0; k < 128; ++k)
                q[m * ldq + g * 128 + k] = orc_e4m3_encode(bf16_to_f32(xr[k]) / sc);
            s[g * ld_s + m] = sc;
        }
    }
}

/* ---------------------------------------------------------------------- */
/* 128x128 weight blocks                                                   */
/* ---------------------------------------------------------------------- */

/*
 * w: bf16 bits [N, K] with row stride ldw.  q: E4M3 [N, K] with row stride ldq.
 * s: fp32 [N/128][K/128] row-major.  N and K must be multiples of 128.
 */
void orc_quant_weight_128x128(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                              uint8_t* q, int64_t ldq, float* s, int pow2) {
    int64_t NB = N / 128, G = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t nb = 0; nb < NB; ++nb) {
        for (int64_t g = 0; g < G; ++g) {
            float amax = 0.0f, sc;
            for (int r = 0; r < 128; ++r)
                for (int k = 0; k < 128; ++k)
                    amax = amax_update(amax, bf16_to_f32(w[(nb * 128 + r) * ldw + g * 128 + k]));
            sc = orc_scale_from_amax(amax, pow2);
            for (int r = 0; r < 128; ++r)
                for (int k = 0; k < 128; ++k) {
                    int64_t i = (nb * 128 + r);
                    q[i * ldq + g * 128 + k] = orc_e4m3_encode(bf16_to_f32(w[i * ldw + g * 128 + k]) / sc);
                }
            s[nb * G + g] = sc;
        }
    }
}

/* ---------------------------------------------------------------------- */
/* 1xK rows (one scale per row over all of K)                              */
/* ---------------------------------------------------------------------- */

/*
 * The per-tensor-row baseline of the accumulation study: a single scale per
 * row cannot be applied group by group, so the whole K is accumulated before
 * scaling.  Same scale rule as the tiles, with the amax over the full row.
 */
void orc_quant_rowwise(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                       uint8_t* q, int64_t ldq, float* s, int pow2) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f, sc;
        for (int64_t k = 0; k < K; ++k) amax = amax_update(amax, bf16_to_f32(x[m * ldx + k]));
        sc = orc_scale_from_amax(amax, pow2);
        for (int64_t k = 0; k < K; ++k)
            q[m * ldq + k] = orc_e4m3_encode(bf16_to_f32(x[m * ldx + k]) / sc);
        s[m] = sc;
    }
}

/* ---------------------------------------------------------------------- */
/* one scale for the whole tensor (the coarse baseline)                    */
/* ---------------------------------------------------------------------- */

/*
 * The per-tensor scaling that fine-grained quantization replaces.  the-good.kr
 * wr_id=2169793 para 4: the usual practice maps the maximum absolute value of the
 * whole input tensor to the largest FP8 value, which leaves low-precision training
 * very sensitive to activation outliers; pkd.ac.th webboard 78017 para 1 answers
 * with scaling at a finer grain.  Same scale rule as the tiles, with the amax over
 * all R x C elements; *s receives the single scale.
 */
void orc_quant_tensorwise(const uint16_t* x, int64_t R, int64_t C, int64_t ldx,
                          uint8_t* q, int64_t ldq, float* s, int pow2) {
    float amax = 0.0f, sc;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c) amax = amax_update(amax, bf16_to_f32(x[r * ldx + c]));
    sc = orc_scale_from_amax(amax, pow2);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c)
            q[r * ldq + c] = orc_e4m3_encode(bf16_to_f32(x[r * ldx + c]) / sc);
    *s = sc;
}

/* ---------------------------------------------------------------------- */
/* brute-force GEMM (tiny shapes)                                          */
/* ---------------------------------------------------------------------- */

/*
 * C[m, n] = sum_k (decode(qa[m,k]) * sa[m, k/128]) * (decode(qb[n,k]) * sb(n, k/128)),
 * T[m, n] = sum_k |same product|, accumulated in double in increasing k.
 *
 * sa is group-major (sa[g * ld_sa + m]).  b_rowwise == 0: sb is [N/128][K/128]
 * row-major (one scale per 128x128 block); b_rowwise == 1: sb is group-major
 * like sa (sb[g * ld_sb + n]).
 */
void orc_gemm_triple(const uint8_t* qa, const float* sa, int64_t ld_sa,
                     const uint8_t* qb, const float* sb, int64_t ld_sb, int b_rowwise,
                     int64_t M, int64_t N, int64_t K, double* C, double* T) {
    int64_t G = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double c = 0.0, t = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t g = k / 128;
                double a = orc_e4m3_decode(qa[m * K + k]) * (double)sa[g * ld_sa + m];
                double bs = b_rowwise ? (double)sb[g * ld_sb + n] : (double)sb[(n / 128) * G + g];
                double b = orc_e4m3_decode(qb[n * K + k]) * bs;
                c += a * b;
                t += fabs(a * b);
            }
            C[m * N + n] = c;
            T[m * N + n] = t;
        }
}
