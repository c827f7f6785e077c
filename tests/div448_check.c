/* Exhaustive check of the scale division used by the append kernels:
 * for every positive finite float a from 2^-120 up, the product with
 * z = RN(1/448) corrected once by its FMA residual,
 *     q0 = RN(a z),  r = RN(a - q0*448) (exact, one FMA),  q1 = RN(r z + q0),
 * equals the IEEE round-to-nearest quotient RN(a / 448).  All three steps
 * are single IEEE operations, so the result is the same on any IEEE machine
 * with a fused multiply-add.  Prints "checked mismatches"; exit status 0 iff
 * there is no mismatch. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

int main(void)
{
    const float z = 1.0f / 448.0f;
    const long long lo = 0x03800000LL, hi = 0x7f800000LL;   /* 2^-120 .. +inf (excluded) */
    unsigned long long bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (long long u = lo; u < hi; ++u) {
        const uint32_t bits = (uint32_t)u;
        float a;
        memcpy(&a, &bits, 4);
        volatile float ref = a / 448.0f;
        const float q0 = a * z;
        const float r = fmaf(-q0, 448.0f, a);
        const float q1 = fmaf(r, z, q0);
        const float rr = ref;
        bad += memcmp(&rr, &q1, 4) != 0;
    }
    printf("%lld %llu\n", hi - lo, bad);
    return bad != 0;
}
