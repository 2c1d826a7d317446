// curand_philox.cu -- Philox4x32-10 words from cuRAND's device API
// (curand_kernel.h, curandStatePhilox4_32_10_t), called as a library on the
// GPU.  TEST REFERENCE ONLY: a third party's implementation, used to pin the
// oracle's Philox stream; neither the oracle nor the CUDA library uses it.
//
// curand_init(seed, subsequence, offset, &s) places the generator at the
// 128-bit counter (offset / 4 as a 64-bit number in words 0-1, subsequence in
// words 2-3) with key (seed low 32, seed high 32); with offset a multiple of
// 4, curand4 returns the four output words of that counter.  The same words
// are also taken from curand_Philox4x32_10(counter, key) directly.
#include <cuda_runtime.h>
#include <curand_kernel.h>
#include <stdint.h>

__global__ void curand_philox_kernel(const uint4* ctr, const uint2* key, int n, uint4* via_state,
                                     uint4* direct) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const uint4 c = ctr[i];
    const uint2 k = key[i];
    const unsigned long long seed = (unsigned long long)k.x | ((unsigned long long)k.y << 32);
    const unsigned long long subsequence = (unsigned long long)c.z | ((unsigned long long)c.w << 32);
    const unsigned long long block = (unsigned long long)c.x | ((unsigned long long)c.y << 32);
    curandStatePhilox4_32_10_t s;
    curand_init(seed, subsequence, 4ull * block, &s);
    via_state[i] = curand4(&s);
    direct[i] = curand_Philox4x32_10(c, k);
}

// ctr [n][4], key [n][2] host arrays; via_state, direct [n][4] host outputs.
// counter word 1 must be below 2^30 (offset = 4 * block fits 64 bits).
// Returns 0 on success, else the CUDA error code.
extern "C" int curand_philox_words(const uint32_t* ctr, const uint32_t* key, int n,
                                   uint32_t* via_state, uint32_t* direct) {
    if (n <= 0) return 0;
    uint4 *dc = nullptr, *dv = nullptr, *dd = nullptr;
    uint2* dk = nullptr;
    cudaError_t e = cudaMalloc(&dc, sizeof(uint4) * n);
    if (e == cudaSuccess) e = cudaMalloc(&dk, sizeof(uint2) * n);
    if (e == cudaSuccess) e = cudaMalloc(&dv, sizeof(uint4) * n);
    if (e == cudaSuccess) e = cudaMalloc(&dd, sizeof(uint4) * n);
    if (e == cudaSuccess) e = cudaMemcpy(dc, ctr, sizeof(uint4) * n, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(dk, key, sizeof(uint2) * n, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
        curand_philox_kernel<<<(n + 127) / 128, 128>>>(dc, dk, n, dv, dd);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpy(via_state, dv, sizeof(uint4) * n, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(direct, dd, sizeof(uint4) * n, cudaMemcpyDeviceToHost);
    cudaFree(dc);
    cudaFree(dk);
    cudaFree(dv);
    cudaFree(dd);
    return (int)e;
}
