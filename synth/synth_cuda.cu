// Seeded synthetic input generator, device side (input generation only; none of the method's
// arithmetic). It draws exactly the counter-based SplitMix64 streams of synth.c and applies the
// same Box-Muller transform, but with the device's double-precision sqrt/log/cos, whose last bits
// may differ from the host library's: a value can then round to a neighbouring bf16. Workloads
// that need byte-exact inputs on both sides (parity cases) regenerate those units on the host.
#include <cuda_runtime.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

__device__ __forceinline__ double normal_at(uint64_t key, uint64_t n) {
    const uint64_t z = mix64(key + (n + 1) * GAMMA);
    const double u1 = ((double)(z >> 32) + 1.0) * (1.0 / 4294967296.0);
    const double u2 = (double)(z & 0xFFFFFFFFULL) * (1.0 / 4294967296.0);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    const uint32_t b = __float_as_uint(f);
    return (uint16_t)((b + (((b >> 16) & 1u) + 0x7FFFu)) >> 16);
}

// out[r][c] = bf16(f32(mu[j][c] + sigma[j] * normal(key, r * d + c))), j = min(r / L, nb - 1)
__global__ void block_rows_bf16_kernel(uint64_t key, const float* mu, const float* sigma, int64_t nb, int64_t T,
                                       int64_t d, int64_t L, uint16_t* out) {
    const int64_t total = T * d;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / d, c = e % d;
        int64_t j = r / L;
        if (j >= nb) j = nb - 1;
        const double v = (double)mu[j * d + c] + (double)sigma[j] * normal_at(key, (uint64_t)e);
        out[e] = f32_to_bf16_bits((float)v);
    }
}

// Anisotropic blocks: row r of block j = mu_j + sum_{i < R} s_{j,i} z_{r,i} U_j[:, i] + 0.1 sigma_j eps_r,
// with U_j[c][i] = normal(ku, (j d + c) R + i) / sqrt(d), z_{r,i} = normal(key, r (R + d) + i),
// eps_{r,c} = normal(key, r (R + d) + R + c) and s_{j,i} = sigma_j sqrt(d 2^-i / sum_i' 2^-i'): the
// block's spread concentrated on R directions with geometrically decaying variances.
__global__ void aniso_rows_bf16_kernel(uint64_t key, uint64_t ku, const float* mu, const float* sigma, int64_t nb,
                                       int64_t T, int64_t d, int64_t L, int R, uint16_t* out) {
    const int64_t total = T * d;
    double wsum = 0.0;
    for (int i = 0; i < R; ++i) wsum += ldexp(1.0, -i);
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / d, c = e % d;
        int64_t j = r / L;
        if (j >= nb) j = nb - 1;
        const double sj = (double)sigma[j];
        double v = (double)mu[j * d + c] + 0.1 * sj * normal_at(key, (uint64_t)(r * (R + d) + R + c));
        for (int i = 0; i < R; ++i) {
            const double s = sj * sqrt((double)d * ldexp(1.0, -i) / wsum);
            const double u = normal_at(ku, (uint64_t)((j * d + c) * R + i)) * inv_sqrt_d;
            v += s * normal_at(key, (uint64_t)(r * (R + d) + i)) * u;
        }
        out[e] = f32_to_bf16_bits((float)v);
    }
}

extern "C" int synth_gpu_aniso_rows_bf16(uint64_t key, uint64_t ku, const float* mu, const float* sigma, int64_t nb,
                                         int64_t T, int64_t d, int64_t L, int R, uint16_t* out, void* stream) {
    aniso_rows_bf16_kernel<<<8 * 148, 256, 0, (cudaStream_t)stream>>>(key, ku, mu, sigma, nb, T, d, L, R, out);
    return (int)cudaGetLastError();
}

extern "C" int synth_gpu_block_rows_bf16(uint64_t key, const float* mu, const float* sigma, int64_t nb, int64_t T,
                                         int64_t d, int64_t L, uint16_t* out, void* stream) {
    block_rows_bf16_kernel<<<4 * 148, 256, 0, (cudaStream_t)stream>>>(key, mu, sigma, nb, T, d, L, out);
    return (int)cudaGetLastError();
}
