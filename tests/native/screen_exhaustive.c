/*
 * Exhaustive check of the E4M3 conversion screen used by the CUDA quantizer (test
 * infrastructure; the device code in quant_e4m3.cuh is restated here in C).
 *
 * The quantizer forms y = x * RN(1/s) instead of t = RN(x / s); y is within 3 FP32
 * ulps of t.  It keeps y's E4M3 code unless one of two screens fires:
 *   normal:    ((bits(y) + 0x80006) & 0xFFFFF) <= 12
 *   subnormal: rr = RN(1024 y + 1.5 * 2^23), n = rr - 1.5 * 2^23,
 *              d = RN(1024 y - n), fires when |d| <= 2^-18 and bits(rr) is odd.
 * Claim: whenever neither fires, every FP32 value within 3 ulps of y (on y's side
 * of zero) has y's E4M3 code, so y and t give the same code.  E4M3 rounding is
 * monotone, so it is enough to compare the codes 3 ulps below and above.  Checked
 * here for every FP32 y with |y| <= 464 (x / s never exceeds 448 (1 + 2^-22)).
 * Prints the number of counterexamples and the first few.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

/* round-to-nearest-even on the FP32 bits: 3 mantissa bits in the normal range,
   quantum 2^-9 below 2^-6, saturation at 448, sign of zero kept */
static uint8_t ref_encode(uint32_t u)
{
    uint8_t sign = (uint8_t)((u >> 31) << 7);
    uint32_t mag = u & 0x7FFFFFFFu;
    float a;
    memcpy(&a, &mag, 4);
    if (a > 448.0f) return sign | 0x7E;
    if (a < 0x1p-6f) return sign | (uint8_t)rintf(a * 512.0f);
    int32_t e = (int32_t)((mag >> 23) & 0xFF) - 127;
    uint32_t m3 = (mag >> 20) & 7u, rem = mag & 0xFFFFFu;
    if (rem > 0x80000u || (rem == 0x80000u && (m3 & 1u))) ++m3;
    if (m3 == 8u) { m3 = 0; ++e; }
    return sign | (uint8_t)(((uint32_t)(e + 7) << 3) | m3);
}

static int screen_fires(uint32_t u)
{
    float y, rr, n, d;
    memcpy(&y, &u, 4);
    if (((u + 0x80006u) & 0xFFFFFu) <= 12u) return 1;
    rr = fmaf(y, 1024.0f, 0x1.8p23f);
    n = rr - 0x1.8p23f;
    d = fmaf(y, 1024.0f, -n);
    uint32_t rb;
    memcpy(&rb, &rr, 4);
    return fabsf(d) <= 0x1p-18f && (rb & 1u);
}

int main(void)
{
    const uint32_t max_mag = 0x43E80000u; /* 464.0f */
    long long bad = 0, fired = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad, fired)
    for (long long i = 0; i <= 2LL * max_mag + 1; ++i) {
        uint32_t mag = (uint32_t)(i >> 1), sign = (uint32_t)(i & 1) << 31;
        uint32_t u = sign | mag;
        if (screen_fires(u)) {
            ++fired;
            continue;
        }
        uint32_t lo = mag >= 3u ? mag - 3u : 0u, hi = mag + 3u;
        uint8_t c = ref_encode(u);
        if (ref_encode(sign | lo) != c || ref_encode(sign | hi) != c) {
            ++bad;
            if (bad <= 5) {
#pragma omp critical
                printf("counterexample 0x%08x\n", u);
            }
        }
    }
    printf("fired %lld of %lld\n", fired, 2LL * max_mag + 2);
    printf("counterexamples %lld\n", bad);
    return bad != 0;
}
