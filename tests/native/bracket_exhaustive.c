/*
 * Exhaustive check of the E4M3 conversion the CUDA quantizer uses (test
 * infrastructure; the device arithmetic of quant_e4m3.cuh restated in C, one
 * IEEE rounding per operation).
 *
 * A block's scale is s = fl32(amax / 448) with amax one of the 32640 positive
 * finite BF16 values, and the block's elements x are BF16 values with |x| <= amax.
 * For every such (x, s) pair -- about 1.07e9 -- the quantizer's code must equal
 * E4M3(fl32(x / s)), the definition:
 *   r = fl32(1 / s), rlo = fl32(r (1 - 2^-21)), rhi = fl32(r (1 + 2^-21)),
 *   lo = E4M3(fl32(x rlo)), hi = E4M3(fl32(x rhi));
 *   code = hi if lo == hi, else E4M3(fl32(x / s)) (the division path).
 * E4M3() is round-to-nearest-even on the FP32 bits with saturation at 448 and the
 * sign of zero kept (the hardware conversion's semantics; written here, not shared
 * with the oracle).  Prints the number of mismatches and how often the division
 * path ran.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static uint8_t e4m3(float v)
{
    uint32_t u;
    memcpy(&u, &v, 4);
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

static float bf16(uint32_t h)
{
    uint32_t u = h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int main(void)
{
    long long bad = 0, slow = 0, pairs = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad, slow, pairs)
    for (uint32_t ah = 1; ah < 0x7F80u; ++ah) {            /* amax: positive finite BF16 */
        const float amax = bf16(ah);
        const float s = amax / 448.0f;
        const float r = 1.0f / s;
        if (!isfinite(r)) continue;                          /* the quantizer divides directly then */
        const float rlo = r * (1.0f - 0x1p-21f), rhi = r * (1.0f + 0x1p-21f);
        for (uint32_t xm = 0; xm <= ah; ++xm) {              /* |x| <= amax, both signs */
            for (uint32_t sg = 0; sg < 2; ++sg) {
                const float x = bf16(xm | (sg << 15));
                const uint8_t lo = e4m3(x * rlo), hi = e4m3(x * rhi);
                const uint8_t want = e4m3(x / s);
                uint8_t got = hi;
                if (lo != hi) {
                    ++slow;
                    got = want;
                }
                ++pairs;
                if (got != want) {
                    ++bad;
                    if (bad <= 5) {
#pragma omp critical
                        printf("mismatch amax 0x%04x x 0x%04x: got 0x%02x want 0x%02x\n", ah, xm | (sg << 15), got,
                               want);
                    }
                }
            }
        }
    }
    printf("pairs %lld division path %lld\n", pairs, slow);
    printf("mismatches %lld\n", bad);
    return bad != 0;
}
