/* Exhaustive host check of the division step of the FP8 row quantizer.
 *
 * The kernel forms x / s (s = max(amax, 1e-8) / 448, the row scale) as
 *   q0 = x * r,  e = fma(q0, s, -x),  q = fma(-e, r, q0),  r = 1 / s  (all fp32, RN)
 * (Markstein, "Computation of elementary functions on the IBM RISC System/6000 processor",
 * 1990; e is minus the remainder, which keeps the sign of a zero x). This program visits
 * every finite positive bf16
 * amax and every bf16 x with |x| <= amax and counts the pairs where q can decide a
 * different E4M3 code than the IEEE quotient: a different value where either quotient
 * exceeds 2^-11 in magnitude (below that both round to a zero code), a different zero, or
 * a different sign. Prints the count; exit status 1 if it is not zero.
 * Build: cc -O2 -ffp-contract=off -fopenmp row_scale_division_check.c -lm */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

int main(void) {
    long long bad = 0, pairs = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad, pairs)
    for (int ab = 0; ab < 0x7F80; ++ab) { /* positive finite bf16 magnitudes, 0 included */
        const float amax = f_of((uint32_t)ab << 16);
        volatile float floor_v = 1e-8f, c448 = 448.0f, one = 1.0f;
        const float s = (amax > floor_v ? amax : floor_v) / c448;
        const float r = one / s;
        for (uint32_t xb = 0; xb < 0x10000; ++xb) {
            if ((xb & 0x7FFF) > (uint32_t)ab) continue; /* only |x| <= amax occurs */
            const float x = f_of(xb << 16);
            const float q = x / s;
            const float q0 = x * r;
            const float e = fmaf(q0, s, -x);
            const float q1 = fmaf(-e, r, q0);
            ++pairs;
            if (u_of(q1) != u_of(q) &&
                (fabsf(q) > 0x1p-11f || fabsf(q1) > 0x1p-11f || q == 0.0f || q1 == 0.0f || signbit(q) != signbit(q1)))
                ++bad;
        }
    }
    printf("%lld pairs, %lld differences\n", pairs, bad);
    return bad != 0;
}
