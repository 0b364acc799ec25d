/*
 * Exhaustive CPU replay of the dual-level kernel's division step (CUDA
 * dl_div): for every finite bf16 level-0 amax a0 > 0, s0 = fl32(a0 / 6) and
 * r = fl32(1 / s0), and for every bf16 x with |x| <= a0 (both signs), the
 * corrected reciprocal product
 *     q = fl(x r),  e = fma(-q, s0, x),  y = fma(e, r, q)
 * is compared with the IEEE quotient fl32(x / s0) wherever the kernel uses it
 * (|x| >= 2^-102 and |q| >= 2^-124); zeros and the remaining elements take
 * other routes there (+0, IEEE division). Prints "pairs N fast F bad B".
 *
 * Also checks the kernel's table for s0 and r: for every bf16 a0 >= 2^-65
 * (exponent field >= 62), fl32(a0 / 6) and fl32(1 / s0) equal the entries
 * computed for a0's significand at exponent 0, shifted by a0's exponent.
 * Prints "table T table_bad B".
 * Built with -ffp-contract=off so that every product and fma is the one
 * written.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t u)
{
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int main(void)
{
    long long pairs = 0, fast = 0, bad = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, fast, bad)
#endif
    for (uint32_t ab = 1; ab < 0x7F80u; ++ab) {
        const float a0 = f_of(ab << 16);
        float s0 = a0 / 6.0f;
        if (s0 == 0.0f)
            s0 = 1.0f;
        const float r = 1.0f / s0;
        for (uint32_t xb = 1; xb <= ab; ++xb) {
            for (int neg = 0; neg < 2; ++neg) {
                const float x = f_of((xb | (neg ? 0x8000u : 0u)) << 16);
                const float q = x * r;
                ++pairs;
                if (!(fabsf(x) >= 0x1p-102f && fabsf(q) >= 0x1p-124f))
                    continue;
                ++fast;
                const float e = fmaf(-q, s0, x);
                const float y = fmaf(e, r, q);
                const float t = x / s0;
                if (memcmp(&y, &t, 4) != 0)
                    ++bad;
            }
        }
    }
    printf("pairs %lld fast %lld bad %lld\n", pairs, fast, bad);

    long long table = 0, table_bad = 0;
    for (uint32_t ab = 62u << 7; ab < 0x7F80u; ++ab) {
        const float a0 = f_of(ab << 16);
        const float s0 = a0 / 6.0f, r = 1.0f / s0;
        const float t_s0 = f_of((0x3F80u + (ab & 0x7Fu)) << 16) / 6.0f;
        const float t_r = 1.0f / t_s0;
        const int e = (int)(ab >> 7) - 127;
        uint32_t us0, ur, uts0, utr;
        memcpy(&us0, &s0, 4);
        memcpy(&ur, &r, 4);
        memcpy(&uts0, &t_s0, 4);
        memcpy(&utr, &t_r, 4);
        ++table;
        if (us0 != uts0 + ((uint32_t)e << 23) || ur != utr - ((uint32_t)e << 23))
            ++table_bad;
    }
    printf("table %lld table_bad %lld\n", table, table_bad);
    return 0;
}
