// Test helper (not part of the library): runs curand's Philox4_32_10 device
// generator so the oracle's counter/key layout can be checked against it.
// For each (seed, j): curand_init(seed, 0, 4 j) then curand4() -- the block at
// counter j of key seed.
#include <cuda_runtime.h>
#include <curand_kernel.h>

#include <cstdint>

__global__ void probe(const unsigned long long* seeds, const unsigned long long* js, int count, uint32_t* out) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    curandStatePhilox4_32_10_t st;
    curand_init(seeds[i], 0ull, 4ull * js[i], &st);
    const uint4 r = curand4(&st);
    out[4 * i + 0] = r.x;
    out[4 * i + 1] = r.y;
    out[4 * i + 2] = r.z;
    out[4 * i + 3] = r.w;
}

extern "C" int philox_curand_probe(const unsigned long long* d_seeds, const unsigned long long* d_js, int count,
                                   uint32_t* d_out) {
    if (count <= 0) return 0;
    probe<<<(count + 127) / 128, 128>>>(d_seeds, d_js, count, d_out);
    if (cudaGetLastError() != cudaSuccess) return 1;
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 1;
}
