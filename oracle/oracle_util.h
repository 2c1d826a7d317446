/*
 * oracle_util.h -- the one helper every oracle file uses: exact widening of a
 * stored element (fp32, or bf16 held as a uint16 bit pattern) to double.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 */
#ifndef DFLASH2_ORACLE_UTIL_H
#define DFLASH2_ORACLE_UTIL_H

#include <stdint.h>
#include <string.h>

#include "oracle.h"

/* A bf16 value is the upper 16 bits of the fp32 value with the same sign,
 * exponent and leading mantissa bits, so widening is a 16-bit shift. */
static inline double orc_load(const void* base, int dtype, int64_t i) {
    if (dtype == ORC_F32) {
        return (double)((const float*)base)[i];
    }
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static inline int orc_dtype_ok(int dtype) { return dtype == ORC_F32 || dtype == ORC_BF16; }

#endif
