// Test support only: cuRAND's Philox4_32_10 (an implementation independent of
// this repository's oracle and library) evaluated at given counters, used to
// pin the oracle's Philox4x32-10 stream.  curand_init(seed, subsequence,
// offset) sets key = (seed lo, seed hi) and counter = (offset/4 lo, offset/4
// hi, subsequence lo, subsequence hi); the first curand4() returns the block
// function of that counter.
#include <cuda_runtime.h>
#include <curand_kernel.h>
#include <stdint.h>

__global__ void philox_blocks(uint64_t seed, uint64_t subsequence, const uint64_t *g, int n,
                              uint4 *out) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    curandStatePhilox4_32_10_t st;
    curand_init(seed, subsequence, 4ull * g[i], &st);
    out[i] = curand4(&st);
}

extern "C" int curand_philox_blocks(uint64_t seed, uint64_t subsequence, const uint64_t *g_host,
                                    int n, uint32_t *out_host) {
    uint64_t *g = nullptr;
    uint4 *out = nullptr;
    if (cudaMalloc(&g, sizeof(uint64_t) * n) != cudaSuccess) return 1;
    if (cudaMalloc(&out, sizeof(uint4) * n) != cudaSuccess) return 2;
    cudaMemcpy(g, g_host, sizeof(uint64_t) * n, cudaMemcpyHostToDevice);
    philox_blocks<<<(n + 127) / 128, 128>>>(seed, subsequence, g, n, out);
    cudaError_t e = cudaMemcpy(out_host, out, sizeof(uint4) * n, cudaMemcpyDeviceToHost);
    cudaFree(g);
    cudaFree(out);
    return e == cudaSuccess ? 0 : 3;
}
