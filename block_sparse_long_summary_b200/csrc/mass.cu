// Exact attention mass per key block, for evaluating a selector against the oracle sparse
// attention (OSA) of COBS (gist.science explainer) §2.1: the mass of block b for head h is
// m_{h,b} = sum_{r in b} exp(q_h . k_r / sqrt(d)), and OSA keeps the blocks of largest mass.
// This is an evaluation kernel: the decode and prefill paths never call it.
//
// grid (ceil(nB / kWarps), B * Hkv), kWarps warps. Warp w takes one block of 64 keys; lane l
// holds keys l and l + 32 of it and computes their logits against the G heads of the group
// (float32 fused multiply-adds, ascending channels), then the warp forms
// ln m = max + ln(sum exp(s - max)) for each head with shuffles.
#include <float.h>

#include "common.cuh"
#include "dims.h"

namespace cobs {
namespace {

constexpr int kMassWarps = 4;
constexpr int kMaxG = 16;
constexpr unsigned kFullMask = 0xffffffffu;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&x)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kMassWarps * 32) block_log_mass_kernel(const T* __restrict__ Q,
                                                                         const T* __restrict__ K,
                                                                         float* __restrict__ out, int Tctx,
                                                                         int Hkv, int G, int nB, int L, float isd) {
    __shared__ float qs[kMaxG][D];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int unit = blockIdx.y;
    const int b = unit / Hkv, g = unit % Hkv;
    // the group's query heads are rows unit * G .. unit * G + G - 1 of Q [B, Hq, d]
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) qs[e / D][e % D] = Elem<T>::load(Q + (size_t)unit * G * D + e);
    __syncthreads();
    const int blk = blockIdx.x * kMassWarps + warp;
    if (blk >= nB) return;  // warp-uniform
    const T* rows = K + ((size_t)unit * Tctx + (size_t)blk * L) * D;
    float s[2][kMaxG];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) s[j][h] = 0.0f;
        const T* row = rows + (size_t)(lane + 32 * j) * D;
        for (int c8 = 0; c8 < D / 8; ++c8) {
            float x[8];
            load8<T>(row + 8 * c8, x);
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h < G) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) s[j][h] = __fmaf_rn(qs[h][8 * c8 + i], x[i], s[j][h]);
                }
            }
        }
    }
    float* o = out + ((size_t)b * Hkv * G + (size_t)g * G) * nB + blk;
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        if (h < G) {
            const float a0 = s[0][h] * isd, a1 = s[1][h] * isd;
            float mx = fmaxf(a0, a1);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
            float sum = expf(a0 - mx) + expf(a1 - mx);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFullMask, sum, off);
            if (lane == 0) o[(size_t)h * nB] = mx + logf(sum);
        }
    }
}

template <typename T, int D>
cudaError_t launch_t(const Dims& m, const void* Q, const void* K, float* out, cudaStream_t s) {
    if (m.nB == 0) return cudaSuccess;
    const float isd = (float)(1.0 / sqrt((double)m.d));
    count_launch();
    block_log_mass_kernel<T, D><<<dim3((m.nB + kMassWarps - 1) / kMassWarps, m.units()), kMassWarps * 32, 0, s>>>(
        static_cast<const T*>(Q), static_cast<const T*>(K), out, m.T, m.Hkv, m.G, m.nB, m.L, isd);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_log_mass(const Dims& m, const void* Q, const void* K, float* out, cudaStream_t s) {
    if (m.G > kMaxG) return cudaErrorNotSupported;
    if (m.dtype == COBS_BF16)
        return m.d == 128 ? launch_t<__nv_bfloat16, 128>(m, Q, K, out, s) : launch_t<__nv_bfloat16, 64>(m, Q, K, out, s);
    return m.d == 128 ? launch_t<float, 128>(m, Q, K, out, s) : launch_t<float, 64>(m, Q, K, out, s);
}

}  // namespace cobs
