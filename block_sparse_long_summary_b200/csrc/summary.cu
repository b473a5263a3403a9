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
#include <algorithm>

#include "common.cuh"
#include "dims.h"
#include "tma.h"

namespace cobs {
namespace {

constexpr int kBlock = 64;  // selection block size (validated by the API)

// Offsets inside a unit's summaries of block j, channel c: the mean, the per-channel variance
// (channel layout), the block's variance scalar (isotropic layout).
__host__ __device__ __forceinline__ size_t summ_mu_at(int j, int c, int d, int iso) {
    const size_t gf = iso ? (size_t)(d + 1) * 32 : (size_t)2 * d * 32;
    return (size_t)(j >> 5) * gf + ((size_t)(c / 4) * 32 + (j & 31)) * 4 + (c & 3);
}
__host__ __device__ __forceinline__ size_t summ_var_at(int j, int c, int d) {
    return summ_mu_at(j, c, d, 0) + (size_t)d * 32;
}
__host__ __device__ __forceinline__ size_t summ_iso_at(int j, int d) {
    return (size_t)(j >> 5) * (size_t)(d + 1) * 32 + (size_t)d * 32 + (j & 31);
}

// The isotropic scalar of a block from its per-channel variances v[0..d): adds in ascending
// channel order from +0, then the exact scaling by 1/d (d a power of two).
__device__ __forceinline__ float iso_scalar(const float* v, int d) {
    float s = 0.0f;
    for (int c = 0; c < d; ++c) s = __fadd_rn(s, v[c]);
    return __fmul_rn(s, 1.0f / (float)d);
}

// grid (blocks to build, units), block d threads (one per channel).
template <typename T>
__global__ void __launch_bounds__(128) summaries_kernel(const T* __restrict__ K, int Tctx, int d, int nG,
                                                        int j_begin, int iso, float* __restrict__ summ) {
    __shared__ float vsm[128];
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
    const size_t gf = iso ? (size_t)(d + 1) * 32 : (size_t)2 * d * 32;
    float* base = summ + (size_t)unit * nG * gf;
    base[summ_mu_at(j, c, d, iso)] = mu;
    if (!iso) {
        base[summ_var_at(j, c, d)] = var;
        return;
    }
    vsm[c] = var;
    __syncthreads();
    if (c == 0) base[summ_iso_at(j, d)] = iso_scalar(vsm, d);
}

// ---------------------------------------------------------------- low-rank summaries
// The block mean and the R leading eigenpairs of the block covariance (COBS explainer §2.2/§2.3:
// the covariance kept in low-rank form), by a fixed float32 subspace iteration whose every
// operation is fixed (the same steps as the oracle's solver):
//   Y = rows - mu; V = V0 (+-1 by a bit of a hash of (c, j));
//   kLrIters times: T = Y V (four-chain sums over channels), W = Y^T T (four-chain sums over
//   rows), modified Gram-Schmidt over the columns of W with "32-lane" dot products (lane l sums
//   channels l, l + 32, ... with fma, then a five-level xor butterfly of adds), V = W;
//   then T = Y V and lambda_j = (four-chain sum of T[., j]^2) / L, pairs ordered by lambda
//   descending (ties: lower j).
// grid (blocks to build, units), NT threads (kLrThreadsWide for a few blocks, where the latency of
// one block is the cost; kLrThreadsNarrow for many, where several CTAs share an SM): thread c < D
// owns channel c for the mean and
// the outputs; in the products T = Y V and W = Y^T T a thread takes one chain of one row of Y
// (or column of Y) against all R columns, the four chains in four neighbouring lanes, combined
// by two shuffles in the canonical order (s0 + s1) + (s2 + s3); one warp orthonormalises.
constexpr int kLrIters = 24;
constexpr int kLrMaxR = 8;
constexpr int kLrThreadsWide = 512;
constexpr int kLrThreadsNarrow = 128;
constexpr int kLrPitch = 4;  // Y rows padded by 4 floats: T = Y V reads distinct banks, W = Yt T two lanes a bank

// Chain q of the four-chain dots of one row x (stride sx) against the R columns of a
// row-major [n][kLrMaxR] matrix y (16-byte aligned rows): s[jj] = fma over the terms i = q,
// q + 4, ... below n in ascending order, from +0. Then the chains of the four neighbouring
// lanes q = 0..3 are combined as (s0 + s1) + (s2 + s3): every lane of the quad ends with the
// same values as lr_dot4(x, y + jj, n, sx, kLrMaxR).
__device__ __forceinline__ void lr_quad_dots(const float* x, const float* y, int n, int sx, int q, int R,
                                             float (&s)[kLrMaxR]) {
#pragma unroll
    for (int jj = 0; jj < kLrMaxR; ++jj) s[jj] = 0.0f;
    if (R <= 4) {
#pragma unroll 4
        for (int i = q; i < n; i += 4) {
            const float xv = x[i * sx];
            const float4 a = *reinterpret_cast<const float4*>(y + i * kLrMaxR);
            s[0] = __fmaf_rn(xv, a.x, s[0]);
            s[1] = __fmaf_rn(xv, a.y, s[1]);
            s[2] = __fmaf_rn(xv, a.z, s[2]);
            s[3] = __fmaf_rn(xv, a.w, s[3]);
        }
    } else {
#pragma unroll 4
        for (int i = q; i < n; i += 4) {
            const float xv = x[i * sx];
            const float4 a = *reinterpret_cast<const float4*>(y + i * kLrMaxR);
            const float4 b = *reinterpret_cast<const float4*>(y + i * kLrMaxR + 4);
            s[0] = __fmaf_rn(xv, a.x, s[0]);
            s[1] = __fmaf_rn(xv, a.y, s[1]);
            s[2] = __fmaf_rn(xv, a.z, s[2]);
            s[3] = __fmaf_rn(xv, a.w, s[3]);
            s[4] = __fmaf_rn(xv, b.x, s[4]);
            s[5] = __fmaf_rn(xv, b.y, s[5]);
            s[6] = __fmaf_rn(xv, b.z, s[6]);
            s[7] = __fmaf_rn(xv, b.w, s[7]);
        }
    }
#pragma unroll
    for (int jj = 0; jj < kLrMaxR; ++jj) {
        const float v = __fadd_rn(s[jj], __shfl_xor_sync(0xffffffffu, s[jj], 1));  // s0 + s1, s2 + s3
        s[jj] = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 2));                 // (s0 + s1) + (s2 + s3)
    }
}

__device__ __forceinline__ float lr_v0(int c, int j) {
    const uint32_t h = (uint32_t)c * 2654435761u + (uint32_t)(j + 1) * 40503u;
    return ((h >> 11) & 1u) ? 1.0f : -1.0f;
}

// Four-chain dot over n terms (n a multiple of 4) with strides, (s0 + s1) + (s2 + s3).
__device__ __forceinline__ float lr_dot4(const float* x, const float* y, int n, int sx, int sy) {
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    for (int i = 0; i < n; i += 4) {
        s0 = __fmaf_rn(x[(i + 0) * sx], y[(i + 0) * sy], s0);
        s1 = __fmaf_rn(x[(i + 1) * sx], y[(i + 1) * sy], s1);
        s2 = __fmaf_rn(x[(i + 2) * sx], y[(i + 2) * sy], s2);
        s3 = __fmaf_rn(x[(i + 3) * sx], y[(i + 3) * sy], s3);
    }
    return __fadd_rn(__fadd_rn(s0, s1), __fadd_rn(s2, s3));
}

// E2M1 (FP4) code of x: the nearest of the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (ties to the even
// magnitude index), saturating above 6; the sign in bit 3 (a zero magnitude has code 0).
__device__ __forceinline__ int e2m1_code(float x) {
    const float mags[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    const float a = fabsf(x);
    int best = 0;
    float bd = a;
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        const float dist = fabsf(__fsub_rn(a, mags[i]));
        if (dist < bd || (dist == bd && (i & 1) == 0)) {
            best = i;
            bd = dist;
        }
    }
    if (a > 6.0f) best = 7;
    return best == 0 ? 0 : ((x < 0.0f ? 8 : 0) | best);
}

// Modified Gram-Schmidt of the R columns of W[D][kLrMaxR + 1] into V[D][kLrMaxR], by one warp holding every
// column in registers (lane l: channels l, l + 32, ...). Each "32-lane" dot sums its lane's
// channels in ascending order with fma, then adds across lanes by a five-level xor butterfly;
// column i is normalised (sqrt, divide; zero if its norm is zero) once the projections on the
// columns before it are removed, and then its projection is removed from every later column.
// Every column sees the same operations in the same order as in the column-by-column form
// (projections on columns 0, 1, ... in turn, then the normalisation), so the result is the
// same bit for bit; the dots of the later columns against column i are independent, so their
// butterflies run side by side.
template <int D, int R>
__device__ __forceinline__ void lr_orthonormalize_r(const float (*W)[kLrMaxR + 1], float (*V)[kLrMaxR], int lane) {
    constexpr int kPer = D / 32;
    float w[R][kPer];
#pragma unroll
    for (int jj = 0; jj < R; ++jj)
#pragma unroll
        for (int q = 0; q < kPer; ++q) w[jj][q] = W[lane + 32 * q][jj];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        float nn = 0.0f;
#pragma unroll
        for (int q = 0; q < kPer; ++q) nn = __fmaf_rn(w[i][q], w[i][q], nn);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) nn = __fadd_rn(nn, __shfl_xor_sync(0xffffffffu, nn, o));
        const float n = __fsqrt_rn(nn);
#pragma unroll
        for (int q = 0; q < kPer; ++q) w[i][q] = n > 0.0f ? __fdiv_rn(w[i][q], n) : 0.0f;
        float p[R];
#pragma unroll
        for (int jj = i + 1; jj < R; ++jj) {
            p[jj] = 0.0f;
#pragma unroll
            for (int q = 0; q < kPer; ++q) p[jj] = __fmaf_rn(w[i][q], w[jj][q], p[jj]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int jj = i + 1; jj < R; ++jj) p[jj] = __fadd_rn(p[jj], __shfl_xor_sync(0xffffffffu, p[jj], o));
#pragma unroll
        for (int jj = i + 1; jj < R; ++jj)
#pragma unroll
            for (int q = 0; q < kPer; ++q) w[jj][q] = __fmaf_rn(-p[jj], w[i][q], w[jj][q]);
    }
#pragma unroll
    for (int jj = 0; jj < R; ++jj)
#pragma unroll
        for (int q = 0; q < kPer; ++q) V[lane + 32 * q][jj] = w[jj][q];
}

// The rank is a launch argument (1..kLrMaxR); each rank gets its own fully unrolled routine, so
// that no dot, shuffle or update is spent on columns past R.
template <int D>
__device__ __forceinline__ void lr_orthonormalize(const float (*W)[kLrMaxR + 1], float (*V)[kLrMaxR], int R,
                                                  int lane) {
    switch (R) {
        case 1: lr_orthonormalize_r<D, 1>(W, V, lane); break;
        case 2: lr_orthonormalize_r<D, 2>(W, V, lane); break;
        case 3: lr_orthonormalize_r<D, 3>(W, V, lane); break;
        case 4: lr_orthonormalize_r<D, 4>(W, V, lane); break;
        case 5: lr_orthonormalize_r<D, 5>(W, V, lane); break;
        case 6: lr_orthonormalize_r<D, 6>(W, V, lane); break;
        case 7: lr_orthonormalize_r<D, 7>(W, V, lane); break;
        default: lr_orthonormalize_r<D, kLrMaxR>(W, V, lane); break;
    }
}

template <typename T, int D, int NT>
__global__ void __launch_bounds__(NT, 1) lowrank_kernel(const T* __restrict__ K, int Tctx, int nG, int j_begin, int R,
                                                    int fp4, const float* __restrict__ Pb, int S,
                                                    float* __restrict__ summ) {
    __shared__ float Y[kBlock][D + kLrPitch];
    // W: rows of kLrMaxR + 1 floats (lane l's row starts on bank 9 l mod 32: the orthonormalising
    // warp reads it free of bank conflicts); V and T: 16-byte aligned rows of kLrMaxR floats,
    // read a row at a time by the products
    __shared__ float W[D][kLrMaxR + 1];
    __shared__ __align__(16) float V[D][kLrMaxR];
    __shared__ __align__(16) float Tm[kBlock][kLrMaxR];
    __shared__ int ord_sh[kLrMaxR];
    __shared__ float lam_sh[kLrMaxR];
    __shared__ float red[D];
    __shared__ int code_sh[D];
    const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
    const bool ch = c < D;  // this thread owns channel c
    const int unit = blockIdx.y;
    const int j = j_begin + blockIdx.x;
    float mu_c = 0.0f;
    // the block's rows (as float) staged in Y by every thread, coalesced
    {
        const T* rows = K + ((size_t)unit * Tctx + (size_t)j * kBlock) * D;
        for (int e = c; e < kBlock * D; e += NT) Y[e / D][e % D] = Elem<T>::load(rows + e);
    }
    __syncthreads();
    // canonical mean of channel c (rows ascending), then the centred rows
    if (ch) {
        float sum = 0.0f;
#pragma unroll 16
        for (int r = 0; r < kBlock; ++r) sum = __fadd_rn(sum, Y[r][c]);
        const float mu = __fmul_rn(sum, 1.0f / kBlock);
#pragma unroll 16
        for (int r = 0; r < kBlock; ++r) Y[r][c] = __fsub_rn(Y[r][c], mu);
        mu_c = mu;
        for (int jj = 0; jj < R; ++jj) V[c][jj] = lr_v0(c, jj);
    }
    __syncthreads();
    for (int it = 0; it <= kLrIters; ++it) {
        // T[r][.] = four-chain dots over the channels of row r of Y and the columns of V (tasks
        // 4 r + q; NT and 4 L are multiples of 32, so whole warps take whole quads)
        for (int t = c; t < 4 * kBlock; t += NT) {
            float sv[kLrMaxR];
            lr_quad_dots(&Y[t >> 2][0], &V[0][0], D, 1, t & 3, R, sv);
            if ((t & 3) == 0)
#pragma unroll
                for (int jj = 0; jj < kLrMaxR; ++jj)
                    if (jj < R) Tm[t >> 2][jj] = sv[jj];
        }
        __syncthreads();
        if (it == kLrIters) break;
        // W[cc][.] = four-chain dots over the rows of column cc of Y and the columns of T
        // (tasks 4 cc + q)
        for (int t = c; t < 4 * D; t += NT) {
            float sw[kLrMaxR];
            lr_quad_dots(&Y[0][t >> 2], &Tm[0][0], kBlock, D + kLrPitch, t & 3, R, sw);
            if ((t & 3) == 0)
#pragma unroll
                for (int jj = 0; jj < kLrMaxR; ++jj)
                    if (jj < R) W[t >> 2][jj] = sw[jj];
        }
        __syncthreads();
        if (warp == 0) lr_orthonormalize<D>(W, V, R, lane);
        __syncthreads();
    }
    if (c < R) lam_sh[c] = __fmul_rn(lr_dot4(&Tm[0][c], &Tm[0][c], kBlock, kLrMaxR, kLrMaxR), 1.0f / kBlock);
    __syncthreads();
    if (c == 0) {
        int ord[kLrMaxR];
        for (int a = 0; a < R; ++a) ord[a] = a;
        for (int a = 0; a < R; ++a)
            for (int z = a + 1; z < R; ++z)
                if (lam_sh[ord[z]] > lam_sh[ord[a]] || (lam_sh[ord[z]] == lam_sh[ord[a]] && ord[z] < ord[a])) {
                    const int t = ord[a];
                    ord[a] = ord[z];
                    ord[z] = t;
                }
        for (int a = 0; a < R; ++a) ord_sh[a] = ord[a];
    }
    __syncthreads();
    const int ln = j & 31;
    if (S > 0 && !fp4) {
        // query-subspace form: eigenvector jj kept as u~_i = four-chain sum over c of P[c][i] u_c
        // (i < S), in the [S/4][32][4] interleaving
        const size_t gf = (size_t)32 * (D + R * S + R);
        float* base = summ + ((size_t)unit * nG + (size_t)(j >> 5)) * gf;
        if (ch) base[((size_t)(c / 4) * 32 + ln) * 4 + (c & 3)] = mu_c;
        for (int o = c; o < R * S; o += NT) {
            const int jj = o / S, i = o % S;
            base[(size_t)32 * D + (size_t)jj * S * 32 + ((size_t)(i / 4) * 32 + ln) * 4 + (i & 3)] =
                lr_dot4(Pb + i, &V[0][ord_sh[jj]], D, S, kLrMaxR);
        }
        if (c < R) base[(size_t)32 * (D + R * S) + (size_t)c * 32 + ln] = lam_sh[ord_sh[c]];
        return;
    }
    if (!fp4) {
        const size_t gf = (size_t)32 * (D + R * D + R);
        float* base = summ + (size_t)unit * nG * gf + (size_t)(j >> 5) * gf;
        if (!ch) return;
        base[((size_t)(c / 4) * 32 + ln) * 4 + (c & 3)] = mu_c;
        for (int jj = 0; jj < R; ++jj)
            base[(size_t)(1 + jj) * D * 32 + ((size_t)(c / 4) * 32 + ln) * 4 + (c & 3)] = V[c][ord_sh[jj]];
        if (c < R) base[(size_t)(1 + R) * D * 32 + (size_t)c * 32 + ln] = lam_sh[ord_sh[c]];
        return;
    }
    // FP4 layout (bytes): bf16 means [D/8][32][8], E2M1 codes of vector jj [CW/32][32][16]
    // (entry 2i in the low nibble of byte i), scales [R][32] f32, eigenvalues [R][32] f32. The
    // vector is the eigenvector (CW = D), or its S coordinates in the query subspace (the
    // projection of the float32 form above; CW = S rounded up to 32, the codes past S zero).
    const int CW = S > 0 ? (S + 31) / 32 * 32 : D;
    const size_t gbytes = (size_t)32 * (2 * D + R * CW / 2 + 8 * R);
    unsigned char* g8 = reinterpret_cast<unsigned char*>(summ) + ((size_t)unit * nG + (size_t)(j >> 5)) * gbytes;
    if (ch) {
        const __nv_bfloat16 mb = __float2bfloat16_rn(mu_c);
        *reinterpret_cast<__nv_bfloat16*>(g8 + ((size_t)(c / 8) * 32 + ln) * 16 + (c % 8) * 2) = mb;
    }
    float* scl = reinterpret_cast<float*>(g8 + (size_t)64 * D + (size_t)R * 16 * CW);
    float* lamo = scl + R * 32;
    const bool live = ch && (S == 0 || c < S);  // thread c holds an entry of the vector
    for (int jj = 0; jj < R; ++jj) {
        const float x = !live ? 0.0f
                        : S == 0 ? V[c][ord_sh[jj]] : lr_dot4(Pb + c, &V[0][ord_sh[jj]], D, S, kLrMaxR);
        if (ch) red[c] = fabsf(x);
        __syncthreads();
        for (int o = D / 2; o > 0; o >>= 1) {  // max is exact in any order
            if (c < o) red[c] = fmaxf(red[c], red[c + o]);
            __syncthreads();
        }
        const float sc = __fdiv_rn(red[0], 6.0f);
        if (ch) code_sh[c] = live && sc > 0.0f ? e2m1_code(__fdiv_rn(x, sc)) : 0;
        __syncthreads();
        if ((c & 1) == 0 && c < CW)
            g8[(size_t)64 * D + (size_t)jj * 16 * CW + ((size_t)(c / 32) * 32 + ln) * 16 + (c % 32) / 2] =
                (unsigned char)(code_sh[c] | (code_sh[c + 1] << 4));
        if (c == 0) {
            scl[jj * 32 + ln] = sc;
            lamo[jj * 32 + ln] = lam_sh[ord_sh[jj]];
        }
        __syncthreads();
    }
}

// grid (tokens to build, units, 2 = {K, V}), block d threads. out_i = P @ mean(rows).
template <typename T>
__global__ void __launch_bounds__(128) compress_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                       const float* __restrict__ Pk,
                                                       const float* __restrict__ Pv, int Tctx, int d,
                                                       int lc, int sc, int nC, int i_begin,
                                                       T* __restrict__ Kc, T* __restrict__ Vc) {
    __shared__ __align__(16) float pooled[128];
    const int c = threadIdx.x;
    const int unit = blockIdx.y;
    const int i = i_begin + blockIdx.x;
    const bool isv = blockIdx.z == 1;
    const T* X = isv ? V : K;
    const float* P = isv ? Pv : Pk;
    T* out = isv ? Vc : Kc;
    const T* rows = X + ((size_t)unit * Tctx + (size_t)sc * i) * d + c;
    float s = 0.0f;
#pragma unroll 16
    for (int r = 0; r < lc; ++r) s += Elem<T>::load(rows + (size_t)r * d);  // 16 loads in flight
    const float m = s / (float)lc;
    pooled[c] = m;
    __syncthreads();
    T* orow = out + ((size_t)unit * nC + i) * d;
    if (P == nullptr) {
        Elem<T>::store(orow + c, m);
        return;
    }
    // out[j] = P[j, :] . pooled: a warp per output row, lanes over 4-channel slices of the
    // row (coalesced 512-byte reads of P), shuffle reduction.
    const int lane = c & 31, warp = c >> 5, nwarps = blockDim.x >> 5;
    const float4* p4 = reinterpret_cast<const float4*>(P);
    const float4 q = lane * 4 < d ? reinterpret_cast<const float4*>(pooled)[lane] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int j = warp; j < d; j += nwarps) {
        float acc = 0.0f;
        if (lane * 4 < d) {
            const float4 pv = __ldg(p4 + (size_t)j * (d / 4) + lane);
            acc = pv.x * q.x + pv.y * q.y + pv.z * q.z + pv.w * q.w;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) Elem<T>::store(orow + j, acc);
    }
}

// ---------------------------------------------------------------- fused bf16 build
// One pass over K and V for bf16, block 64, compression 32 / 16 and a projection. A work item
// is 2 selection blocks (128 rows) of one unit plus the 16 following rows: it yields the
// summaries of its 2 blocks and its 8 compressed tokens (token i covers rows 16 i .. 16 i + 31,
// i.e. 16-row chunks i and i + 1). Persistent CTAs of 8 warps walk the items with a 2-stage
// bulk-copy ring. Per item:
//   * threads (block, channel) form the float32 summaries in row order (the canonical order)
//     and the 16-row chunk sums of K and V;
//   * the 8 pooled tokens (chunk pair sums / 32) are split into bf16 hi + lo;
//   * warps 0-3 (K) and 4-7 (V) project them on tensor cores: out = P pooled with P held in
//     registers as bf16 hi + lo and three products (Phi*hi + Phi*lo + Plo*hi), float32 sums.
constexpr int kFRows = 144;     // 128 rows + 16 halo rows
constexpr int kFThreads = 256;

template <int D>
struct FusedSmem {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kStage = 2 * kFRows * kRowBytes;  // K rows then V rows
    static constexpr int kPooledStride = D + 8;            // bf16 elements per pooled row (bank spread)
};

template <int D>
__global__ void __launch_bounds__(kFThreads, 1) summary_fused_kernel(
    const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V, const float* __restrict__ Pk,
    const float* __restrict__ Pv, int Tctx, int nB, int nG, int nC, int j_begin, int i_begin, int m_begin,
    int m_count, int units, int iso, float* __restrict__ summ, __nv_bfloat16* __restrict__ Kc,
    __nv_bfloat16* __restrict__ Vc, int* err) {
    using S = FusedSmem<D>;
    __shared__ float vsm[2][D];  // per-channel variances of the item's two blocks (isotropic layout)
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* ring = smem_raw;                                             // 2 stages
    float* cs = reinterpret_cast<float*>(ring + 2 * S::kStage);                 // [2][9][D] chunk sums
    __nv_bfloat16* pooled = reinterpret_cast<__nv_bfloat16*>(cs + 2 * 9 * D);   // [2 side][2 hi/lo][8][D+8]
    __nv_bfloat16* outst = pooled + 2 * 2 * 8 * S::kPooledStride;              // [2 side][8][D]
    __shared__ __align__(8) uint64_t bar[2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long n_items = (long long)units * m_count;

    // projection rows of this warp as A fragments (bf16 hi and lo): side = warp / 4,
    // output channels [(warp % 4) * D/4, +D/4) = D/64 m16 tiles
    constexpr int MT = D / 64, KS = D / 16;
    const int side = warp >> 2;
    const float* P = side ? Pv : Pk;
    uint32_t ahi[MT][KS][4], alo[MT][KS][4];
    {
        const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int r0 = (warp & 3) * (D / 4) + mt * 16 + gid, r1 = r0 + 8;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int c = ks * 16 + 2 * tig;
                const float v[4][2] = {{P[r0 * D + c], P[r0 * D + c + 1]},
                                       {P[r1 * D + c], P[r1 * D + c + 1]},
                                       {P[r0 * D + c + 8], P[r0 * D + c + 9]},
                                       {P[r1 * D + c + 8], P[r1 * D + c + 9]}};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const __nv_bfloat16 h0 = __float2bfloat16_rn(v[q][0]), h1 = __float2bfloat16_rn(v[q][1]);
                    const float l0 = v[q][0] - __bfloat162float(h0), l1 = v[q][1] - __bfloat162float(h1);
                    __nv_bfloat162 hh; hh.x = h0; hh.y = h1;
                    ahi[mt][ks][q] = *reinterpret_cast<uint32_t*>(&hh);
                    alo[mt][ks][q] = pack_bf16(l0, l1);
                }
            }
        }
    }

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_barrier_init();
    }
    __syncthreads();

    auto rows_of = [&](long long item, int& unit, int& m, int& r0, int& nrows) {
        unit = (int)(item / m_count);
        m = m_begin + (int)(item % m_count);
        r0 = m * 128;
        nrows = max(0, min(kFRows, Tctx - r0));
    };
    auto issue = [&](long long item, int st) {  // tid 0
        int unit, m, r0, nrows;
        rows_of(item, unit, m, r0, nrows);
        if (nrows == 0) return;
        const uint32_t bytes = (uint32_t)nrows * S::kRowBytes;
        unsigned char* dst = ring + st * S::kStage;
        mbar_arrive_expect_tx(&bar[st], 2 * bytes);
        bulk_g2s(dst, K + ((size_t)unit * Tctx + r0) * D, bytes, &bar[st]);
        bulk_g2s(dst + kFRows * S::kRowBytes, V + ((size_t)unit * Tctx + r0) * D, bytes, &bar[st]);
    };
    const long long first = blockIdx.x, stride = gridDim.x;
    if (tid == 0) {
        if (first < n_items) issue(first, 0);
        if (first + stride < n_items) issue(first + stride, 1);
    }
    uint32_t phase = 0;
    bool ok = true;
    int it = 0;
    for (long long item = first; item < n_items; item += stride, ++it) {
        const int st = it & 1;
        int unit, m, r0, nrows;
        rows_of(item, unit, m, r0, nrows);
        if (nrows > 0 && ok && !mbar_wait(&bar[st], (phase >> st) & 1u, err)) ok = false;
        ok = __syncthreads_and(ok) != 0;
        if (nrows > 0) phase ^= 1u << st;
        const __nv_bfloat16* sK = reinterpret_cast<const __nv_bfloat16*>(ring + st * S::kStage);
        const __nv_bfloat16* sV = sK + kFRows * D;
        // ---- summaries and chunk sums (thread = (block, channel))
        if (tid < 2 * D && ok) {
            const int blk = tid / D, c = tid % D;
            const int j = 2 * m + blk;
            const int rb = blk * 64;
            const bool have = (rb + 64) <= nrows;
            float ksum[4] = {0.f, 0.f, 0.f, 0.f};
            if (have) {
                float s = 0.0f;
#pragma unroll 16
                for (int r = 0; r < 64; ++r) {
                    const float x = __bfloat162float(sK[(rb + r) * D + c]);
                    s = __fadd_rn(s, x);
                    ksum[r >> 4] += x;
                }
                const float mu = __fmul_rn(s, 1.0f / 64.0f);
                float a2 = 0.0f;
#pragma unroll 16
                for (int r = 0; r < 64; ++r) {
                    const float tt = __fsub_rn(__bfloat162float(sK[(rb + r) * D + c]), mu);
                    a2 = __fmaf_rn(tt, tt, a2);
                }
                if (j < nB && j >= j_begin) {
                    float* base = summ + (size_t)unit * nG * (iso ? (D + 1) * 32 : 2 * D * 32);
                    base[summ_mu_at(j, c, D, iso)] = mu;
                    if (iso)
                        vsm[blk][c] = __fmul_rn(a2, 1.0f / 64.0f);
                    else
                        base[summ_var_at(j, c, D)] = __fmul_rn(a2, 1.0f / 64.0f);
                }
            } else {
                for (int q = 0; q < 4; ++q) {
                    float x = 0.0f;
                    for (int r = rb + 16 * q; r < min(rb + 16 * q + 16, nrows); ++r) x += __bfloat162float(sK[r * D + c]);
                    ksum[q] = x;
                }
            }
            for (int q = 0; q < 4; ++q) cs[(0 * 9 + blk * 4 + q) * D + c] = ksum[q];
            // halo chunk of K (rows 128..143) by block-0 threads; V chunks 0-4 / 5-8
            if (blk == 0) {
                float x = 0.0f;
                for (int r = 128; r < min(144, nrows); ++r) x += __bfloat162float(sK[r * D + c]);
                cs[(0 * 9 + 8) * D + c] = x;
            }
            const int q0 = blk == 0 ? 0 : 5, q1 = blk == 0 ? 5 : 9;
            for (int q = q0; q < q1; ++q) {
                float x = 0.0f;
                const int ra = 16 * q, rz = min(16 * q + 16, nrows);
#pragma unroll 16
                for (int r = ra; r < rz; ++r) x += __bfloat162float(sV[r * D + c]);
                cs[(1 * 9 + q) * D + c] = x;
            }
        }
        __syncthreads();
        // ---- isotropic scalars of the item's two blocks (one thread each, channels ascending)
        if (iso && ok && tid < 2) {
            const int j = 2 * m + tid;
            if ((tid * 64 + 64) <= nrows && j < nB && j >= j_begin)
                summ[(size_t)unit * nG * (D + 1) * 32 + summ_iso_at(j, D)] = iso_scalar(vsm[tid], D);
        }
        // ---- pooled tokens, split into bf16 hi + lo
        for (int e = tid; e < 2 * 8 * D; e += kFThreads) {
            const int sd = e / (8 * D), rem = e % (8 * D), p = rem / D, c = rem % D;
            const float x = (cs[(sd * 9 + p) * D + c] + cs[(sd * 9 + p + 1) * D + c]) * (1.0f / 32.0f);
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
            pooled[((sd * 2 + 0) * 8 + p) * S::kPooledStride + c] = hi;
            pooled[((sd * 2 + 1) * 8 + p) * S::kPooledStride + c] = lo;
        }
        __syncthreads();
        // the stage is free: prefetch the item after next into it
        if (tid == 0 && ok && item + 2 * stride < n_items) {
            fence_proxy_async();
            issue(item + 2 * stride, st);
        }
        // ---- projection on tensor cores: out[channel][token] for this warp's channels
        {
            const int gid = lane >> 2, tig = lane & 3;
            const __nv_bfloat16* ph = pooled + (side * 2 + 0) * 8 * S::kPooledStride;
            const __nv_bfloat16* pl = pooled + (side * 2 + 1) * 8 * S::kPooledStride;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const int c = ks * 16 + 2 * tig;
                    const uint32_t bh0 = *reinterpret_cast<const uint32_t*>(ph + gid * S::kPooledStride + c);
                    const uint32_t bh1 = *reinterpret_cast<const uint32_t*>(ph + gid * S::kPooledStride + c + 8);
                    const uint32_t bl0 = *reinterpret_cast<const uint32_t*>(pl + gid * S::kPooledStride + c);
                    const uint32_t bl1 = *reinterpret_cast<const uint32_t*>(pl + gid * S::kPooledStride + c + 8);
                    mma_bf16_16816(c4, ahi[mt][ks], bh0, bh1);
                    mma_bf16_16816(c4, ahi[mt][ks], bl0, bl1);
                    mma_bf16_16816(c4, alo[mt][ks], bh0, bh1);
                }
                const int ch = (warp & 3) * (D / 4) + mt * 16 + gid;
                __nv_bfloat16* o = outst + side * 8 * D;
                o[(2 * tig) * D + ch] = __float2bfloat16_rn(c4[0]);
                o[(2 * tig + 1) * D + ch] = __float2bfloat16_rn(c4[1]);
                o[(2 * tig) * D + ch + 8] = __float2bfloat16_rn(c4[2]);
                o[(2 * tig + 1) * D + ch + 8] = __float2bfloat16_rn(c4[3]);
            }
        }
        __syncthreads();
        // ---- compressed tokens out (16-byte stores)
        for (int e = tid; e < 2 * 8 * (D / 8); e += kFThreads) {
            const int sd = e / (8 * (D / 8)), rem = e % (8 * (D / 8)), p = rem / (D / 8), c8 = rem % (D / 8);
            const int i = 8 * m + p;
            if (ok && i < nC && i >= i_begin) {
                __nv_bfloat16* dst = (sd ? Vc : Kc) + ((size_t)unit * nC + i) * D + c8 * 8;
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(outst + sd * 8 * D + p * D + c8 * 8);
            }
        }
        __syncthreads();
    }
}

template <int D>
cudaError_t launch_fused(const Dims& m, const __nv_bfloat16* K, const __nv_bfloat16* V, const float* Pk,
                         const float* Pv, int t_begin, float* summ, __nv_bfloat16* Kc, __nv_bfloat16* Vc,
                         cudaStream_t s, int* err) {
    const int j_begin = t_begin <= 0 ? 0 : (t_begin + 1 + m.L - 1) / m.L - 1;
    int i_begin = 0;
    if (t_begin > 0) {
        const int num = t_begin - m.lc + 1;
        i_begin = num <= 0 ? 0 : (num + m.sc - 1) / m.sc;
    }
    const int m_end = std::max((m.nB + 1) / 2, (m.nC + 7) / 8);
    const int m_begin = std::min(j_begin / 2, i_begin / 8);
    const int m_count = m_end - m_begin;
    if (m_count <= 0) return cudaSuccess;
    using S = FusedSmem<D>;
    const size_t smem = 2 * (size_t)S::kStage + 2 * 9 * D * 4 + 2 * 2 * 8 * S::kPooledStride * 2 + 2 * 8 * D * 2;
    cudaError_t e = cudaFuncSetAttribute(summary_fused_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long items = (long long)m.units() * m_count;
    const int grid = (int)std::min<long long>(items, sm_count());
    count_launch();
    summary_fused_kernel<D><<<grid, kFThreads, smem, s>>>(K, V, Pk, Pv, m.T, m.nB, m.nG, m.nC, j_begin, i_begin,
                                                          m_begin, m_count, m.units(), m.iso, summ, Kc, Vc, err);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- decode-step append
// The update after appending one token: at most one newly complete block (its summary) and one
// newly complete compressed token (K and V) per unit. Grid (units, 4) of 256 threads: CTA y
// summarises channels [32 y, 32 y + 32) of the block and projects output rows
// [y d / 4, (y + 1) d / 4) of both compressed tokens, each warp d / 16 rows at once
// (out_j = P[j, :] . pooled, coalesced rows of P, interleaved shuffle reductions); every CTA
// pools the 32 rows itself (all row loads in flight at once).
template <typename T>
__global__ void __launch_bounds__(256) append_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                     const float* __restrict__ Pk, const float* __restrict__ Pv,
                                                     int Tctx, int d, int nG, int nC, int lc, int sc, int jb, int ic,
                                                     int iso, float* __restrict__ summ, T* __restrict__ Kc,
                                                     T* __restrict__ Vc) {
    __shared__ __align__(16) float pooled[2][128];
    __shared__ float vsm[128];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int unit = blockIdx.x, quarter = blockIdx.y;
    // this warp's rows of the projection (d / 16 <= 8 rows, one 16-byte chunk per lane), loaded
    // first so that their latency overlaps the row loads below
    const int ws = warp >> 2;  // warps 0-3: K, 4-7: V
    const float* P = ws ? Pv : Pk;
    const int per_warp = d / 16;
    const int j0 = quarter * (d / 4) + (warp & 3) * per_warp;
    float4 pv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
        pv[u] = (ic >= 0 && P != nullptr && u < per_warp && lane * 4 < d)
                    ? __ldg(reinterpret_cast<const float4*>(P + (size_t)(j0 + u) * d) + lane)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    // block summary (channels 32 quarter + tid; the isotropic layout needs every channel in
    // one CTA: quarter 0, thread = channel): the canonical row-order sums
    const bool sum_here = jb >= 0 && (iso ? (quarter == 0 && tid < d) : (tid < 32 && quarter * 32 + tid < d));
    if (sum_here) {
        const int c = iso ? tid : quarter * 32 + tid;
        const T* rows = K + ((size_t)unit * Tctx + (size_t)jb * kBlock) * d + c;
        float x[kBlock];
#pragma unroll
        for (int r = 0; r < kBlock; ++r) x[r] = Elem<T>::load(rows + (size_t)r * d);
        float sum = 0.0f;
#pragma unroll
        for (int r = 0; r < kBlock; ++r) sum = __fadd_rn(sum, x[r]);
        const float mu = __fmul_rn(sum, 1.0f / kBlock);
        float a2 = 0.0f;
#pragma unroll
        for (int r = 0; r < kBlock; ++r) {
            const float t = __fsub_rn(x[r], mu);
            a2 = __fmaf_rn(t, t, a2);
        }
        float* base = summ + (size_t)unit * nG * (iso ? (size_t)(d + 1) * 32 : (size_t)2 * d * 32);
        base[summ_mu_at(jb, c, d, iso)] = mu;
        if (iso)
            vsm[c] = __fmul_rn(a2, 1.0f / kBlock);
        else
            base[summ_var_at(jb, c, d)] = __fmul_rn(a2, 1.0f / kBlock);
    }
    if (iso) {
        __syncthreads();
        if (jb >= 0 && quarter == 0 && tid == 0)
            summ[(size_t)unit * nG * (d + 1) * 32 + summ_iso_at(jb, d)] = iso_scalar(vsm, d);
    }
    if (ic < 0) return;
    // pooled compressed token: threads [0, d) for K, [128, 128 + d) for V
    const int side = tid >> 7, c = tid & 127;
    if (c < d) {
        const T* rows = (side ? V : K) + ((size_t)unit * Tctx + (size_t)sc * ic) * d + c;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 32
        for (int r = 0; r < lc; ++r) acc[r & 3] += Elem<T>::load(rows + (size_t)r * d);
        pooled[side][c] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) / (float)lc;
    }
    __syncthreads();
    T* orow = (ws ? Vc : Kc) + ((size_t)unit * nC + ic) * d;
    if (P == nullptr) {
        const int cc = tid & 127;
        if (cc < d && cc / (d / 4) == quarter) Elem<T>::store(orow + cc, pooled[ws][cc]);
        return;
    }
    const float4 q = lane * 4 < d ? reinterpret_cast<const float4*>(pooled[ws])[lane] : make_float4(0.f, 0.f, 0.f, 0.f);
    float part[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) part[u] = pv[u].x * q.x + pv[u].y * q.y + pv[u].z * q.z + pv[u].w * q.w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int u = 0; u < 8; ++u) part[u] += __shfl_xor_sync(0xffffffffu, part[u], off);
    if (lane < per_warp) {
        float v = part[0];
#pragma unroll
        for (int u = 1; u < 8; ++u) v = lane == u ? part[u] : v;
        Elem<T>::store(orow + j0 + lane, v);
    }
}

// The low-rank summaries of blocks [j_begin, j_begin + nbuild) of every unit: wide CTAs while the
// grid leaves SMs idle (the decode step's one block per unit), narrow ones, several per SM, else.
template <typename T>
void launch_lowrank(const Dims& m, const T* K, int nbuild, int j_begin, float* summ, cudaStream_t s) {
    const dim3 grid(nbuild, m.units());
    const bool wide = (long long)nbuild * m.units() < (long long)sm_count();
    if (m.d == 128) {
        if (wide)
            lowrank_kernel<T, 128, kLrThreadsWide><<<grid, kLrThreadsWide, 0, s>>>(K, m.T, m.nG, j_begin, m.lr, m.fp4,
                                                                                m.basis, m.sub, summ);
        else
            lowrank_kernel<T, 128, kLrThreadsNarrow><<<grid, kLrThreadsNarrow, 0, s>>>(K, m.T, m.nG, j_begin, m.lr,
                                                                                    m.fp4, m.basis, m.sub, summ);
    } else {
        if (wide)
            lowrank_kernel<T, 64, kLrThreadsWide><<<grid, kLrThreadsWide, 0, s>>>(K, m.T, m.nG, j_begin, m.lr, m.fp4,
                                                                               m.basis, m.sub, summ);
        else
            lowrank_kernel<T, 64, kLrThreadsNarrow><<<grid, kLrThreadsNarrow, 0, s>>>(K, m.T, m.nG, j_begin, m.lr,
                                                                                   m.fp4, m.basis, m.sub, summ);
    }
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
        if (m.lr) {
            launch_lowrank(m, K, nbuild, j_begin, summ, s);
        } else {
            summaries_kernel<T><<<dim3(nbuild, units), m.d, 0, s>>>(K, m.T, m.d, m.nG, j_begin, m.iso, summ);
        }
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

template <typename T>
bool try_append(const Dims& m, const T* K, const T* V, const float* Pk, const float* Pv, int t_begin, float* summ,
                T* Kc, T* Vc, cudaStream_t s, cudaError_t* e) {
    if (t_begin <= 0 || m.L != kBlock || m.d > 128) return false;
    const int j_begin = (t_begin + 1 + m.L - 1) / m.L - 1;
    const int num = t_begin - m.lc + 1;
    const int i_begin = num <= 0 ? 0 : (num + m.sc - 1) / m.sc;
    const int nj = m.nB - j_begin, ni = m.nC - i_begin;
    if (nj > 1 || ni > 1) return false;
    *e = cudaSuccess;
    // low-rank summaries: the block goes to the eigen-solver, the token to the append kernel
    const bool block_here = nj > 0 && !m.lr;
    if (block_here || ni > 0) {
        count_launch();
        append_kernel<T><<<dim3(m.units(), 4), 256, 0, s>>>(K, V, Pk, Pv, m.T, m.d, m.nG, m.nC, m.lc, m.sc,
                                                            block_here ? j_begin : -1, ni > 0 ? i_begin : -1, m.iso,
                                                            summ, Kc, Vc);
        *e = cudaGetLastError();
        if (*e != cudaSuccess) return true;
    }
    if (nj > 0 && m.lr) {
        count_launch();
        launch_lowrank(m, K, 1, j_begin, summ, s);
        *e = cudaGetLastError();
    }
    return true;
}

cudaError_t launch_summaries(const Dims& m, const void* K, const void* V, const float* Pk, const float* Pv,
                             int t_begin, float* summ, void* Kc, void* Vc, cudaStream_t s, int* err) {
    // the decode-step update (one block, one compressed token): a small dedicated kernel
    cudaError_t ea = cudaSuccess;
    if ((m.dtype == COBS_BF16
                      ? try_append<__nv_bfloat16>(m, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, Pk, Pv, t_begin,
                                                  summ, (__nv_bfloat16*)Kc, (__nv_bfloat16*)Vc, s, &ea)
                      : try_append<float>(m, (const float*)K, (const float*)V, Pk, Pv, t_begin, summ, (float*)Kc,
                                          (float*)Vc, s, &ea)))
        return ea;
    // fused one-pass kernel for the bf16 layout it is written for; plain kernels otherwise
    if (!m.lr && m.dtype == COBS_BF16 && m.L == 64 && m.lc == 32 && m.sc == 16 && Pk != nullptr && Pv != nullptr &&
        (m.d == 128 || m.d == 64) && m.nC > 0) {
        if (m.d == 128)
            return launch_fused<128>(m, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, Pk, Pv, t_begin, summ,
                                     (__nv_bfloat16*)Kc, (__nv_bfloat16*)Vc, s, err);
        return launch_fused<64>(m, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, Pk, Pv, t_begin, summ,
                                (__nv_bfloat16*)Kc, (__nv_bfloat16*)Vc, s, err);
    }
    if (m.dtype == COBS_BF16)
        return launch_summaries_t<__nv_bfloat16>(m, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, Pk, Pv,
                                                 t_begin, summ, (__nv_bfloat16*)Kc, (__nv_bfloat16*)Vc, s);
    return launch_summaries_t<float>(m, (const float*)K, (const float*)V, Pk, Pv, t_begin, summ, (float*)Kc,
                                     (float*)Vc, s);
}

}  // namespace cobs
