/* Exhaustive check of the activation quantiser's quotient on the host, in
 * IEEE binary32 (no fast-math, no contraction; fmaf is one rounding).
 *
 * The quantiser divides each BF16 value x of a 1x128 group by the group's
 * scale s = RN(amax / 448), |x| <= amax.  The GPU forms the quotient without
 * a divide: y = RN(1/s), q = RN(x*y), r = RN(s*q - x), d = RN(q - r*y), then
 * copies the sign of x onto d.  For every finite positive BF16 amax whose
 * scale is at least 2^-100 and every BF16 x with |x| <= amax (both signs),
 * this program compares d with the IEEE quotient RN(x/s) and counts the
 * pairs whose E4M3 codes could differ: d != RN(x/s) unless both lie below
 * 2^-11 in magnitude with the same sign (E4M3 encodes every magnitude below
 * 2^-10 to a signed zero).  The group scale itself is formed the same way,
 * with y = RN(1/448); for every finite non-negative BF16 amax the program
 * compares it with RN(amax/448) bit for bit.  It prints "pairs=<n>
 * code_mismatch=<m> float_mismatch=<f> scales=<s> scale_mismatch=<z>" and
 * exits 0. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float bf16(uint32_t b)
{
    uint32_t u = b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint32_t bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

int main(void)
{
    long long pairs = 0, code_bad = 0, float_bad = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, code_bad, float_bad)
    for (int ai = 1; ai < 0x7F80; ++ai) {
        const float amax = bf16((uint32_t)ai);
        volatile float sv = amax / 448.0f;
        const float s = sv;
        if (!(s >= 0x1p-100f)) continue;
        volatile float yv = 1.0f / s;
        const float y = yv;
        for (int xi = 0; xi <= ai; ++xi) {
            for (int sg = 0; sg < 2; ++sg) {
                const float x = bf16((uint32_t)xi | (sg ? 0x8000u : 0u));
                volatile float div = x / s;
                volatile float q = x * y;
                volatile float r = fmaf(s, q, -x);
                volatile float d = copysignf(fmaf(-r, y, q), x);
                const float a = div, b = d;
                ++pairs;
                if (bits(a) == bits(b)) continue;
                ++float_bad;
                if (fabsf(a) >= 0x1p-11f || fabsf(b) >= 0x1p-11f || signbit(a) != signbit(b)) ++code_bad;
            }
        }
    }
    long long scales = 0, scale_bad = 0;
    volatile float inv448v = 1.0f / 448.0f;
    const float inv448 = inv448v;
    for (int ai = 0; ai < 0x7F80; ++ai) {
        const float amax = bf16((uint32_t)ai);
        volatile float div = amax / 448.0f;
        volatile float q = amax * inv448;
        volatile float r = fmaf(448.0f, q, -amax);
        volatile float d = fmaf(-r, inv448, q);
        ++scales;
        if (bits(div) != bits(d)) ++scale_bad;
    }
    printf("pairs=%lld code_mismatch=%lld float_mismatch=%lld scales=%lld scale_mismatch=%lld\n", pairs, code_bad,
           float_bad, scales, scale_bad);
    return 0;
}
