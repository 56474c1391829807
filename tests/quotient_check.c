/*
 * Exhaustive host check of the quantizer kernels' quotient shortcut.
 *
 * The kernels compute x / s without a division for most tiles (see Quotient in
 * fp8_fine_grained_weight_b200/csrc/quant.cuh): a power-of-two s uses the exact
 * reciprocal; s >= 2^-92 uses a correctly rounded reciprocal plus one FMA residual
 * correction, with the residual taken as d = q0 s - x and the quotient as RN(q0 - d r)
 * so that x = -0 keeps its sign without a sign restore (the f32x2 path feeds the
 * negated input -x and -r, which gives the same values); smaller s divide.  This program replays
 * that sequence with IEEE
 * single-precision host arithmetic (the GPU's fmul/fma/rcp.rn are IEEE too) for
 * every positive finite bf16 amax, both scale modes, and every bf16 x with
 * |x| <= amax, and checks that it yields the same E4M3 input as RN(x / s):
 *   - the same fp32 quotient whenever |x / s| >= 2^-11, and
 *   - otherwise a quotient of the same sign with magnitude <= 2^-10 (E4M3 rounds
 *     both to a signed zero).
 * It also checks the kernels' power-of-two rounding of s (an exponent bit trick)
 * against the definition "smallest power of two >= s", and their amax / 448 (a
 * corrected reciprocal) against IEEE division for every positive bf16 amax.
 * Exit status 0 and "ok" on success.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t b_of(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

/* the kernels' power-of-two rounding (bit trick) */
static float kernel_pow2(float s) {
    uint32_t b = b_of(s), mant = b & 0x7FFFFFu, expo = b & 0x7F800000u;
    if (expo != 0) {
        if (mant != 0) b = expo + 0x00800000u;
    } else if ((mant & (mant - 1u)) != 0) {
        int lz = __builtin_clz(mant);
        b = 1u << (32 - lz);
    }
    return f_of(b);
}

/* the definition: smallest power of two >= s */
static float def_pow2(float s) {
    int ex;
    double f = frexp((double)s, &ex);
    return (float)(f == 0.5 ? (double)s : ldexp(1.0, ex));
}

/* the kernels' amax / 448: RN(1/448) and one FMA residual correction (tiny amax divide) */
static float kernel_div448(float amax) {
    if (amax < 0x1p-100f) return amax / 448.0f;
    const float r = 0x1.24924ap-9f;
    float q0 = amax * r;
    float e = fmaf(-q0, 448.0f, amax);
    return fmaf(e, r, q0);
}

int main(void) {
    long long bad = 0, checked = 0, bad_pow2 = 0, bad_div448 = 0;
    if (0x1.24924ap-9f != 1.0f / 448.0f) { printf("RN(1/448) constant is wrong\n"); return 1; }
    for (int ab = 1; ab < 0x7F80; ++ab) {      /* every positive finite bf16 amax */
        float amax = f_of((uint32_t)ab << 16);
        if (b_of(kernel_div448(amax)) != b_of(amax / 448.0f)) ++bad_div448;
    }
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad, checked, bad_pow2)
    for (int ab = 1; ab < 0x7F80; ++ab) {
        float amax = f_of((uint32_t)ab << 16);
        for (int mode_pow2 = 0; mode_pow2 < 2; ++mode_pow2) {
            float s = amax / 448.0f;
            if (mode_pow2) {
                float sk = kernel_pow2(s), sd = def_pow2(s);
                if (b_of(sk) != b_of(sd)) { ++bad_pow2; continue; }
                s = sk;
            }
            uint32_t sb = b_of(s);
            int mode;
            if ((sb & 0x7FFFFFu) == 0 && (sb & 0x7F800000u) != 0) mode = 0;
            else if (s >= 0x1p-92f) mode = 1;
            else mode = 2;
            if (mode == 2) continue;            /* IEEE division on both sides */
            float r = 1.0f / s;                 /* rcp.rn: correctly rounded */
            for (int xb = 0; xb <= ab; ++xb) {
                for (int sg = 0; sg < 2; ++sg) {
                    float x = f_of(((uint32_t)xb << 16) | (sg ? 0x80000000u : 0));
                    float ref = x / s;
                    float q;
                    const float nx = -x, nr = -r;   /* the corrected f32x2 path feeds -x, -r */
                    if (mode == 0) {
                        q = x * r;
                    } else {
                        float q0 = nx * nr;
                        float d = fmaf(q0, s, nx);
                        q = fmaf(d, nr, q0);
                    }
                    ++checked;
                    if (fabsf(ref) >= 0x1p-11f) {
                        if (b_of(q) != b_of(ref)) ++bad;
                    } else {
                        if (signbit(q) != signbit(ref) || fabsf(q) > 0x1p-10f) ++bad;
                    }
                }
            }
        }
    }
    printf("checked %lld quotients: %lld mismatches, %lld pow2 mismatches, %lld amax/448 mismatches\n",
           checked, bad, bad_pow2, bad_div448);
    if (bad == 0 && bad_pow2 == 0 && bad_div448 == 0) { printf("ok\n"); return 0; }
    return 1;
}
