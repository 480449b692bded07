/* Checks the identity the fused producers rely on for their per-row divisions
 * (Markstein, IBM J. Res. Dev. 34(1), 1990): with y = RN(1/b), q0 = RN(a * y),
 * r = RN(a - b * q0) (one FMA) and q = RN(q0 + r * y) (one FMA), q equals the
 * correctly rounded quotient RN(a / b) in binary32.
 *
 * The reference quotient is (float)((double)a / (double)b): binary64 holds
 * more than 2 * 24 + 2 bits, so rounding the binary64 quotient to binary32 is
 * the correctly rounded binary32 quotient (double rounding is innocuous for
 * division at that precision). Built without FP contraction on a target whose
 * float operations round to binary32.
 *
 * Two sweeps, as the kernels use the identity:
 *   1. a = every positive finite FP16 value, b = n_div divisors with random
 *      significands (edge significands first) and exponents in [-40, 20]
 *      (the RMSNorm x / r);
 *   2. b = every positive finite FP16 value, a = n_num numerators per b with
 *      quotients in [-256, 256], half of them within 4 ulp of a half-integer
 *      quotient (the quantisation h / s).
 * Prints "mismatches <count> of <checked>" and exits 1 on any mismatch.
 * Built with -DPLANT_NO_CORRECTION it returns q0 itself, which the sweeps
 * must catch. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float fp16_value(uint32_t h) {
    const int e = (h >> 10) & 31, f = h & 1023;
    const float v = e == 0 ? ldexpf((float)f, -24) : ldexpf((float)(f | 1024), e - 25);
    return (h & 0x8000u) ? -v : v;
}

static uint64_t state = 0x9E3779B97F4A7C15ull;
static uint32_t next32(void) {   /* xorshift64 */
    state ^= state << 13;
    state ^= state >> 7;
    state ^= state << 17;
    return (uint32_t)(state >> 16);
}

static float quotient(float a, float b, float y) {
    const float q0 = a * y;
    const float r = fmaf(-q0, b, a);
#ifdef PLANT_NO_CORRECTION   /* a planted mistake: the uncorrected product */
    (void)r;
    return q0;
#else
    return fmaf(r, y, q0);
#endif
}

static long bad = 0, checked = 0;
static void check(float a, float b) {
    const float y = (float)(1.0 / (double)b);
    const float want = (float)((double)a / (double)b);
    const float got = quotient(a, b, y);
    ++checked;
    if (u_of(got) != u_of(want)) {
        if (bad < 5) printf("a=%a b=%a got %a want %a\n", a, b, got, want);
        ++bad;
    }
}

int main(int argc, char **argv) {
    const int n_div = argc > 1 ? atoi(argv[1]) : 2000;
    const int n_num = argc > 2 ? atoi(argv[2]) : 200;
    for (int i = 0; i < n_div; ++i) {
        const int ex = (int)(next32() % 61u) - 40;
        uint32_t sig = next32() & 0x7FFFFFu;
        if (i < 32) sig = (i & 1) ? 0x7FFFFFu - (uint32_t)(i >> 1) : (uint32_t)(i >> 1);
        const float b = f_of(((uint32_t)(ex + 127) << 23) | sig);
        for (uint32_t h = 1; h < 0x7C00u; ++h) check(fp16_value(h), b);
    }
    for (uint32_t hs = 1; hs < 0x7C00u; ++hs) {
        const float b = fp16_value(hs);
        for (int k = 0; k < n_num; ++k) {
            float a;
            if (k & 1) {
                const int q = (int)(next32() % 513u) - 256;
                a = f_of(u_of(((float)q + 0.5f) * b) + (uint32_t)((int)(next32() % 9u) - 4));
            } else {
                a = ((float)(next32() & 0xFFFFFFu) / 16777216.0f - 0.5f) * 512.0f * b;
            }
            if (isfinite(a)) check(a, b);
        }
    }
    printf("mismatches %ld of %ld\n", bad, checked);
    return bad != 0;
}
