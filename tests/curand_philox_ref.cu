// Test helper (not part of the library): cuRAND's device-side Philox4_32_10,
// used as an independent library implementation of the generator that the
// CPU oracle writes out by hand.  With subsequence 0 and offset 4 * block, the
// first curand4() of a state returns the generator's output for the counter
// (block, 0, 0, 0) and key (low, high word of the seed).
#include <curand_kernel.h>
#include <stdint.h>

__global__ void philox_blocks(uint64_t seed, const unsigned long long *blocks, int count, uint4 *out)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count)
        return;
    curandStatePhilox4_32_10_t state;
    curand_init(seed, 0ull, 4ull * blocks[i], &state);
    out[i] = curand4(&state);
}

extern "C" int curand_philox_blocks(uint64_t seed, const unsigned long long *blocks, int count,
                                    uint4 *out)
{
    philox_blocks<<<(count + 127) / 128, 128>>>(seed, blocks, count, out);
    return (int)cudaDeviceSynchronize();
}
