// Block summaries (key mean and per-channel key variance) and compressed tokens.
//
// COBS: Cumulant Order Block Sparse Attention (gist.science explainer), §2.2-2.3: the
// block selector keeps, per key block, the mean key (first cumulant) and a compressed
// second-order statistic — here the per-channel variance, the diagonal of the block
// covariance. NSA compression path (Janus issue #181): compressed tokens aggregate
// cmp_block rows every cmp_stride rows; the aggregation is mean-pooling followed by a
// fixed d x d linear map.
//
// Summaries are float32 in a fixed order (rows ascending, one thread per channel),
// so the selector downstream is reproducible bit for bit.
#include "common.cuh"
#include "dims.h"

namespace cobs {
namespace {

constexpr int kBlock = 64;  // selection block size (validated by the API)

// grid (blocks to build, units), block d threads (one per channel).
template <typename T>
__global__ void __launch_bounds__(128) summaries_kernel(const T* __restrict__ K, int Tctx, int d, int nG,
                                                        int j_begin, float* __restrict__ summ) {
    const int c = threadIdx.x;
    const int unit = blockIdx.y;
    const int j = j_begin + blockIdx.x;
    const T* rows = K + ((size_t)unit * Tctx + (size_t)j * kBlock) * d + c;
    float x[kBlock];
#pragma unroll
    for (int r = 0; r < kBlock; ++r) x[r] = Elem<T>::load(rows + (size_t)r * d);
    float s = 0.0f;
#pragma unroll
    for (int r = 0; r < kBlock; ++r) s = __fadd_rn(s, x[r]);
    const float mu = __fmul_rn(s, 1.0f / kBlock);
    float a = 0.0f;
#pragma unroll
    for (int r = 0; r < kBlock; ++r) {
        const float t = __fsub_rn(x[r], mu);
        a = __fmaf_rn(t, t, a);
    }
    const float var = __fmul_rn(a, 1.0f / kBlock);
    float* base = summ + (size_t)unit * nG * 2 * d * 32;
    const int g = j >> 5, lane = j & 31;
    const size_t o_mu = ((size_t)(g * 2 + 0) * (d / 4) + c / 4) * 128 + lane * 4 + (c & 3);
    const size_t o_var = ((size_t)(g * 2 + 1) * (d / 4) + c / 4) * 128 + lane * 4 + (c & 3);
    base[o_mu] = mu;
    base[o_var] = var;
}

// grid (tokens to build, units, 2 = {K, V}), block d threads. out_i = P @ mean(rows).
template <typename T>
__global__ void __launch_bounds__(128) compress_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                       const float* __restrict__ Pk,
                                                       const float* __restrict__ Pv, int Tctx, int d,
                                                       int lc, int sc, int nC, int i_begin,
                                                       T* __restrict__ Kc, T* __restrict__ Vc) {
    __shared__ float pooled[128];
    const int c = threadIdx.x;
    const int unit = blockIdx.y;
    const int i = i_begin + blockIdx.x;
    const bool isv = blockIdx.z == 1;
    const T* X = isv ? V : K;
    const float* P = isv ? Pv : Pk;
    T* out = isv ? Vc : Kc;
    const T* rows = X + ((size_t)unit * Tctx + (size_t)sc * i) * d + c;
    float s = 0.0f;
    for (int r = 0; r < lc; ++r) s += Elem<T>::load(rows + (size_t)r * d);
    const float m = s / (float)lc;
    pooled[c] = m;
    __syncthreads();
    float y = m;
    if (P != nullptr) {
        y = 0.0f;
        const float* prow = P + (size_t)c * d;
        for (int cc = 0; cc < d; ++cc) y = fmaf(__ldg(prow + cc), pooled[cc], y);
    }
    Elem<T>::store(out + ((size_t)unit * nC + i) * d + c, y);
}

template <typename T>
cudaError_t launch_summaries_t(const Dims& m, const T* K, const T* V, const float* Pk, const float* Pv,
                               int t_begin, float* summ, T* Kc, T* Vc, cudaStream_t s) {
    const int units = m.units();
    // blocks whose last row (j+1)L-1 >= t_begin
    const int j_begin = t_begin <= 0 ? 0 : (t_begin + 1 + m.L - 1) / m.L - 1;
    const int nbuild = m.nB - (j_begin < 0 ? 0 : j_begin);
    if (nbuild > 0) {
        count_launch();
        summaries_kernel<T><<<dim3(nbuild, units), m.d, 0, s>>>(K, m.T, m.d, m.nG, j_begin, summ);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // compressed tokens whose last row sc*i + lc - 1 >= t_begin
    int i_begin = 0;
    if (t_begin > 0) {
        const int num = t_begin - m.lc + 1;  // need sc*i >= num
        i_begin = num <= 0 ? 0 : (num + m.sc - 1) / m.sc;
    }
    const int ncomp = m.nC - i_begin;
    if (ncomp > 0) {
        count_launch();
        compress_kernel<T><<<dim3(ncomp, units, 2), m.d, 0, s>>>(K, V, Pk, Pv, m.T, m.d, m.lc, m.sc, m.nC,
                                                                 i_begin, Kc, Vc);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_summaries(const Dims& m, const void* K, const void* V, const float* Pk, const float* Pv,
                             int t_begin, float* summ, void* Kc, void* Vc, cudaStream_t s) {
    if (m.dtype == COBS_BF16)
        return launch_summaries_t<__nv_bfloat16>(m, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, Pk, Pv,
                                                 t_begin, summ, (__nv_bfloat16*)Kc, (__nv_bfloat16*)Vc, s);
    return launch_summaries_t<float>(m, (const float*)K, (const float*)V, Pk, Pv, t_begin, summ, (float*)Kc,
                                     (float*)Vc, s);
}

}  // namespace cobs
