// torch_philox.cpp -- Philox4x32-10 words from PyTorch's own engine
// (ATen/core/PhiloxRNGEngine.h, at::Philox4_32), called as a library on the
// host.  TEST REFERENCE ONLY: an implementation written by a third party,
// used to pin the oracle's Philox stream; neither the oracle nor the CUDA
// library uses it.
//
// at::Philox4_32(seed, subsequence, offset) starts at the 128-bit counter
// (offset low 32, offset high 32, subsequence low 32, subsequence high 32)
// with key (seed low 32, seed high 32); its first four calls return the four
// output words of that counter, in order.
#include <ATen/core/PhiloxRNGEngine.h>
#include <stdint.h>

extern "C" void torch_philox_words(const uint32_t* ctr, const uint32_t* key, int64_t n,
                                   uint32_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        const uint32_t* c = ctr + 4 * i;
        const uint64_t seed = (uint64_t)key[2 * i] | ((uint64_t)key[2 * i + 1] << 32);
        const uint64_t offset = (uint64_t)c[0] | ((uint64_t)c[1] << 32);
        const uint64_t subsequence = (uint64_t)c[2] | ((uint64_t)c[3] << 32);
        at::Philox4_32 eng(seed, subsequence, offset);
        for (int j = 0; j < 4; ++j) out[4 * i + j] = eng();
    }
}
