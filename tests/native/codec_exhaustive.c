/*
 * Exhaustive check of the oracle's binary16 codec against the x86 F16C
 * conversion instructions (VCVTPS2PH with round-to-nearest-even, VCVTPH2PS):
 * all 2^32 binary32 inputs of the narrowing conversion, all 2^16 inputs of
 * the widening one.  NaN inputs must give a NaN with the same sign; every
 * other input must give the identical bit pattern.  Test harness only.
 */
#include <immintrin.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "oracle.h"

static int is_nan16(uint16_t h) { return (h & 0x7c00u) == 0x7c00u && (h & 0x3ffu); }

int main(void)
{
    unsigned long long narrow_bad = 0, nan_bad = 0, widen_bad = 0;

#pragma omp parallel for reduction(+ : narrow_bad, nan_bad) schedule(static)
    for (long long hi = 0; hi < 65536; ++hi) {
        for (uint32_t lo = 0; lo < 65536u; ++lo) {
            uint32_t u = ((uint32_t)hi << 16) | lo;
            float x;
            memcpy(&x, &u, sizeof x);
            uint16_t ref = (uint16_t)_cvtss_sh(x, _MM_FROUND_TO_NEAREST_INT);
            uint16_t got = orc_rne16(x);
            if (x != x) {
                if (!is_nan16(got) || (got & 0x8000u) != (ref & 0x8000u))
                    ++nan_bad;
            } else if (ref != got) {
                ++narrow_bad;
            }
        }
    }
    for (uint32_t h = 0; h < 65536u; ++h) {
        float ref = _cvtsh_ss((unsigned short)h);
        float got = orc_widen16((uint16_t)h);
        uint32_t a, b;
        memcpy(&a, &ref, 4);
        memcpy(&b, &got, 4);
        if (is_nan16((uint16_t)h) ? (got == got || (a >> 31) != (b >> 31)) : a != b)
            ++widen_bad;
    }
    printf("narrow_mismatch %llu nan_mismatch %llu widen_mismatch %llu\n",
           narrow_bad, nan_bad, widen_bad);
    return (narrow_bad || nan_bad || widen_bad) ? 1 : 0;
}
