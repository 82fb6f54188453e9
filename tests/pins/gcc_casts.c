/* Independent pin for the oracle's float32 -> 16-bit conversion: GCC's own
 * IEEE casts to _Float16 and __bf16 (round to nearest even; NaN quieted with
 * the payload's top bits kept). Compiled by the test that uses it. */
#include <stdint.h>
#include <string.h>

static uint16_t cast_f16(uint32_t b)
{
    float f;
    memcpy(&f, &b, 4);
    _Float16 h = (_Float16)f;
    uint16_t r;
    memcpy(&r, &h, 2);
    return r;
}

static uint16_t cast_bf16(uint32_t b)
{
    float f;
    memcpy(&f, &b, 4);
    __bf16 h = (__bf16)f;
    uint16_t r;
    memcpy(&r, &h, 2);
    return r;
}

/* Compares got[i] (the oracle's result for pattern start+i) with GCC's cast.
 * Returns the number of mismatches; the first one's index goes to *first. */
int64_t pin_compare_range(uint64_t start, uint64_t count, int dtype, const uint16_t *got, int64_t *first)
{
    int64_t bad = 0, f = -1;
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) {
        uint32_t b = (uint32_t)(start + (uint64_t)i);
        uint16_t want = dtype == 1 ? cast_f16(b) : cast_bf16(b);
        if (want != got[i]) {
            bad += 1;
#pragma omp critical
            if (f < 0 || i < f) f = i;
        }
    }
    *first = f;
    return bad;
}

uint16_t pin_cast(uint32_t b, int dtype) { return dtype == 1 ? cast_f16(b) : cast_bf16(b); }
