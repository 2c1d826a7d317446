/*
 * philox.cpp -- Philox4x32-10, written from its definition in Salmon, Moraes,
 * Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11),
 * section 5, and the uniform the verify step draws from it.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * One round maps the counter (c0, c1, c2, c3) under the round key (k0, k1) to
 *   (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0))
 * where hi/lo are the upper and lower 32 bits of the 64-bit product.  The key
 * advances by the Weyl increments (W0, W1) between rounds; ten rounds make
 * Philox4x32-10.  M0, M1, W0 and W1 are the constants the paper gives for
 * this member of the family (W0 from the golden ratio, W1 from sqrt(3) - 1).
 *
 * The uniform: counter = (step, seq_id, position, purpose), key = (seed low
 * 32 bits, seed high 32 bits), u = (word0 >> 8) * 2^-24, so u is one of the
 * 2^24 values k/2^24 in [0, 1) and is exactly representable in fp32.
 * Purposes: 0 = accept test, 1 = residual / bonus draw, 2 = a test-only draw
 * of the drafted token from q.
 */
#include "oracle.h"

static const uint32_t PHILOX_M0 = 0xD2511F53u;
static const uint32_t PHILOX_M1 = 0xCD9E8D57u;
static const uint32_t PHILOX_W0 = 0x9E3779B9u;
static const uint32_t PHILOX_W1 = 0xBB67AE85u;

extern "C" void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

extern "C" double orc_uniform(uint64_t seed, uint32_t step, uint32_t seq_id, uint32_t pos,
                              uint32_t purpose) {
    uint32_t ctr[4] = {step, seq_id, pos, purpose};
    uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    return (double)(out[0] >> 8) / 16777216.0;
}

extern "C" void orc_uniforms(uint64_t seed, uint32_t step, const uint32_t* seq_id, int64_t n,
                             uint32_t pos, uint32_t purpose, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_uniform(seed, step, seq_id[i], pos, purpose);
}
