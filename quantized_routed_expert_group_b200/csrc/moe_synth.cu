// moe_synth.cu -- device copy of the seeded synthetic-input generator.
//
// Holds no arithmetic of the MoE method.  SplitMix64 (Steele, Lea and Flood,
// OOPSLA 2014) used counter-style: output n of a stream seeded with s is
// mix(s + (n+1) * GAMMA).  key(seed, tid) is output tid of the stream seeded
// with `seed`; element i of tensor tid sums the twelve 16-bit fields of
// outputs 3i, 3i+1, 3i+2 of the stream seeded with key (Irwin-Hall), centres
// and scales them: value = ((S - 393210) / 65536) * sigma, one fp32 multiply.
// Bit-identical to the host generator of the package's synth module.
#include "moe_internal.h"

namespace moe {

__host__ __device__ __forceinline__ uint64_t sm_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

__global__ void k_synth_normal(uint64_t key, int64_t offset, int64_t n, float sigma, float* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t e = (uint64_t)(offset + i);
        int64_t s = 0;
#pragma unroll
        for (int w = 0; w < 3; ++w) {
            const uint64_t r = sm_mix(key + (3 * e + (uint64_t)w + 1) * kGamma);
            s += (int64_t)(r & 0xFFFF) + (int64_t)((r >> 16) & 0xFFFF) + (int64_t)((r >> 32) & 0xFFFF) +
                 (int64_t)(r >> 48);
        }
        const float z = __fdiv_rn((float)(s - 393210), 65536.0f);
        out[i] = __fmul_rn(z, sigma);
    }
}

cudaError_t launch_synth_normal(uint64_t seed, uint64_t tid, int64_t offset, int64_t n, float sigma, float* out,
                                cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const uint64_t key = sm_mix(seed + (tid + 1) * kGamma);
    const int64_t grid = (n + 255) / 256;
    const int g = (int)(grid < (int64_t)device_info().sm_count * 32 ? grid : (int64_t)device_info().sm_count * 32);
    k_synth_normal<<<g, 256, 0, s>>>(key, offset, n, sigma, out);
    return cudaGetLastError();
}

}  // namespace moe
