/* Exhaustive host check of the division step of the INT4 quantizer's clip search.
 *
 * A code needs rint(w / s) for a bf16 weight w and the block's fp16 scale s. The kernel
 * forms the quotient from the scale's reciprocal r = RN(1/s) by one exact FMA correction
 * (Markstein, "Computation of elementary functions on the IBM RISC System/6000 processor",
 * 1990):
 *   q0 = w * r,  e = fma(q0, s, -w),  q = fma(-e, r, q0)      (all fp32, RN)
 * on blocks with max|w| * r < 2^126 and a finite scale (other blocks divide). This program
 * visits every finite positive fp16 s and every finite bf16 w with |w| * r < 2^126 and
 * counts the pairs where rint(q) differs from rint(w / s) (IEEE quotient), or where one of
 * the two is not finite and they differ. Only rint(w / s) reaches a code, a reconstruction
 * or a block error, so a count of zero makes the codes identical to a division.
 * Prints "<pairs> pairs, <bits> bit differences, <bad> code differences"; exit status 1 if
 * <bad> is not zero.
 * Build: cc -O2 -ffp-contract=off -fopenmp quantizer_division_check.c -lm */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* IEEE binary16 bits -> value (subnormals m * 2^-24, normals (1024 + m) * 2^(E - 25)) */
static float half_value(uint16_t h) {
    int E = (h >> 10) & 0x1F, m = h & 0x3FF;
    return (float)(E == 0 ? ldexp((double)m, -24) : ldexp(1024.0 + m, E - 25));
}

int main(void) {
    long long pairs = 0, bits = 0, bad = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : pairs, bits, bad)
    for (int sb = 1; sb < 0x7C00; ++sb) { /* every finite positive fp16 scale */
        const float s = half_value((uint16_t)sb);
        volatile float one = 1.0f;
        const float r = one / s;
        for (uint32_t wb = 0; wb < 0x10000; ++wb) {
            if ((wb & 0x7F80) == 0x7F80) continue; /* bf16 infinities and NaNs */
            const float w = f_of(wb << 16);
            if (!(fabsf(w) * r < 0x1p126f)) continue; /* such blocks divide */
            const float q = w / s;
            const float q0 = w * r;
            const float e = fmaf(q0, s, -w);
            const float q1 = fmaf(-e, r, q0);
            ++pairs;
            if (u_of(q1) == u_of(q)) continue;
            ++bits;
            if (!isfinite(q) || !isfinite(q1) || rintf(q1) != rintf(q)) ++bad;
        }
    }
    printf("%lld pairs, %lld bit differences, %lld code differences\n", pairs, bits, bad);
    return bad != 0;
}
