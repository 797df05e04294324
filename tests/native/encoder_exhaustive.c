/*
 * Exhaustive check of the oracle's E4M3 encoder (test infrastructure).
 *
 * For every FP32 bit pattern that is not NaN or infinite, the oracle's encoder
 * (nearest E4M3 value by table search, ties to the even code, saturation at 448)
 * must agree with an encoder written here another way: round-to-nearest-even on
 * the FP32 bits themselves -- three mantissa bits kept in the normal range
 * (|v| >= 2^-6), the quantum 2^-9 below it, |v| > 448 saturating to 448, and the
 * sign of zero kept.  Prints the number of mismatches and the first few.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

uint8_t dgo_e4m3_encode(float v); /* the oracle (linked) */
void dgo_init(void);

static uint8_t ref_encode(uint32_t u)
{
    uint8_t sign = (uint8_t)((u >> 31) << 7);
    uint32_t mag = u & 0x7FFFFFFFu;
    float a;
    memcpy(&a, &mag, 4);
    if (a > 448.0f) return sign | 0x7E;                /* saturate */
    if (a < 0x1p-6f) {                                   /* subnormal quantum 2^-9 */
        float q = rintf(a * 512.0f);                     /* exact scaling; rint = ties to even */
        return sign | (uint8_t)q;                        /* q == 8 is the code of 2^-6 */
    }
    int32_t e = (int32_t)((mag >> 23) & 0xFF) - 127;     /* -6 .. 8 */
    uint32_t m3 = (mag >> 20) & 7u, rem = mag & 0xFFFFFu;
    if (rem > 0x80000u || (rem == 0x80000u && (m3 & 1u))) ++m3;
    if (m3 == 8u) { m3 = 0; ++e; }
    return sign | (uint8_t)(((uint32_t)(e + 7) << 3) | m3);
}

int main(void)
{
    dgo_init();
    long long bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
    for (long long i = 0; i < (1LL << 32); ++i) {
        uint32_t u = (uint32_t)i;
        if (((u >> 23) & 0xFF) == 0xFF) continue;        /* NaN and infinity: not in the contract */
        float v;
        memcpy(&v, &u, 4);
        uint8_t got = dgo_e4m3_encode(v), want = ref_encode(u);
        if (got != want) {
            ++bad;
            if (bad <= 5) {
#pragma omp critical
                printf("mismatch 0x%08x: oracle 0x%02x, reference 0x%02x\n", u, got, want);
            }
        }
    }
    printf("mismatches %lld\n", bad);
    return bad != 0;
}
