// The query subspace of the subspace summaries, estimated from a sample of queries: the top
// eigenvectors of the queries' second moment (gist.science explainer §2.3: the eigenvectors are
// kept as coordinates in the subspace spanned by the leading eigenvectors of the query second
// moment).
//
//   moment_partial_kernel  each CTA sums q q^T over a contiguous range of rows (float32 FMAs,
//                          every thread an (D/16) x (D/16) tile of the D x D matrix, rows staged
//                          in shared memory 32 at a time)
//   moment_reduce_kernel   M = (1/n) sum of the partials, in partial order (deterministic)
//   jacobi_kernel          one CTA: cyclic Jacobi on M in shared memory, the D/2 rotations of a
//                          round in parallel (round-robin pairing), rows then columns; sweeps
//                          until the off-diagonal mass is below 1e-12 of the total or stops
//                          falling (the float32 rounding floor: after the quadratic phase a sweep
//                          that removes less than three quarters of it), at most kMaxSweeps; then
//                          the s largest eigenvalues in descending order, their eigenvectors as
//                          unit columns with the largest-magnitude entry positive.
#include <algorithm>

#include "common.cuh"
#include "dims.h"
#include "tma.h"  // sm_count

namespace cobs {
namespace {

constexpr int kMomThreads = 256;
constexpr int kMomRows = 32;       // rows staged per pass
constexpr int kJacThreads = 1024;
constexpr int kMaxSweeps = 30;

template <typename T>
__device__ __forceinline__ float to_float(T x);
template <>
__device__ __forceinline__ float to_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// grid (parts), 256 threads; out: [parts][D][D] float32 partial sums of q q^T.
template <typename T, int D>
__global__ void __launch_bounds__(kMomThreads) moment_partial_kernel(const T* __restrict__ Q, long long n, int parts,
                                                                     float* __restrict__ out) {
    constexpr int TL = D / 16;  // tile edge: 16 x 16 threads cover D x D
    __shared__ float rows[kMomRows][D];
    const int tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
    const long long r0 = (long long)blockIdx.x * n / parts, r1 = (long long)(blockIdx.x + 1) * n / parts;
    float acc[TL][TL];
#pragma unroll
    for (int i = 0; i < TL; ++i)
#pragma unroll
        for (int j = 0; j < TL; ++j) acc[i][j] = 0.0f;
    for (long long base = r0; base < r1; base += kMomRows) {
        const int nr = (int)min((long long)kMomRows, r1 - base);
        for (int e = tid; e < kMomRows * D; e += kMomThreads) {
            const int r = e / D, c = e % D;
            rows[r][c] = r < nr ? to_float<T>(Q[(base + r) * D + c]) : 0.0f;
        }
        __syncthreads();
        for (int r = 0; r < nr; ++r) {
            float a[TL], b[TL];
#pragma unroll
            for (int i = 0; i < TL; ++i) {
                a[i] = rows[r][ti * TL + i];
                b[i] = rows[r][tj * TL + i];
            }
#pragma unroll
            for (int i = 0; i < TL; ++i)
#pragma unroll
                for (int j = 0; j < TL; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* o = out + (size_t)blockIdx.x * D * D;
#pragma unroll
    for (int i = 0; i < TL; ++i)
#pragma unroll
        for (int j = 0; j < TL; ++j) o[(ti * TL + i) * D + tj * TL + j] = acc[i][j];
}

// M[e] = (1/n) sum over parts (ascending) of the partials; grid D*D/256.
template <int D>
__global__ void __launch_bounds__(256) moment_reduce_kernel(const float* __restrict__ part, int parts, long long n,
                                                            float* __restrict__ M) {
    const int e = blockIdx.x * 256 + threadIdx.x;
    if (e >= D * D) return;
    double s = 0.0;
    for (int c = 0; c < parts; ++c) s += part[(size_t)c * D * D + e];
    M[e] = (float)(s / (double)n);
}

// One CTA of 1024 threads; dynamic shared memory: A [D][D + 1], V [D][D + 1] float32.
template <int D>
__global__ void __launch_bounds__(kJacThreads) jacobi_kernel(const float* __restrict__ M, int S,
                                                             float* __restrict__ basis, float* __restrict__ evals) {
    constexpr int LD = D + 1;  // row pitch (bank spread of the column updates)
    constexpr int NP = D / 2;  // pairs per round
    extern __shared__ __align__(16) float sm[];
    float* A = sm;
    float* V = sm + D * LD;
    __shared__ float cs[NP], sn[NP];
    __shared__ int top[NP], bot[NP];
    __shared__ int order[D];
    __shared__ float red[kJacThreads / 32];
    __shared__ float off_sh, tot_sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < D * D; e += kJacThreads) {
        const int i = e / D, j = e % D;
        A[i * LD + j] = 0.5f * (M[i * D + j] + M[j * D + i]);  // exactly symmetric
        V[i * LD + j] = i == j ? 1.0f : 0.0f;
    }
    if (tid < NP) {
        top[tid] = 2 * tid;
        bot[tid] = 2 * tid + 1;
    }
    __syncthreads();
    // off-diagonal and total squared mass (block reduction)
    auto masses = [&]() {
        float o = 0.0f, t = 0.0f;
        for (int e = tid; e < D * D; e += kJacThreads) {
            const int i = e / D, j = e % D;
            const float x = A[i * LD + j];
            t = fmaf(x, x, t);
            if (i != j) o = fmaf(x, x, o);
        }
        for (int k = 16; k > 0; k >>= 1) {
            o += __shfl_xor_sync(0xffffffffu, o, k);
            t += __shfl_xor_sync(0xffffffffu, t, k);
        }
        if (lane == 0) red[warp] = o;
        __syncthreads();
        if (tid == 0) {
            float s = 0.0f;
            for (int w = 0; w < kJacThreads / 32; ++w) s += red[w];
            off_sh = s;
        }
        __syncthreads();
        if (lane == 0) red[warp] = t;
        __syncthreads();
        if (tid == 0) {
            float s = 0.0f;
            for (int w = 0; w < kJacThreads / 32; ++w) s += red[w];
            tot_sh = s;
        }
        __syncthreads();
    };
    float prev_off = INFINITY;
    for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
        masses();
        const float off = off_sh;
        if (!(off > 1e-12f * tot_sh)) break;               // also ends on a zero matrix
        if (sweep >= 4 && off > 0.25f * prev_off) break;   // at the rounding floor
        prev_off = off;
        for (int round = 0; round < D - 1; ++round) {
            // rotation of each pair: zero A[p][q] (symmetric Schur decomposition of the 2 x 2 block)
            if (tid < NP) {
                const int p = min(top[tid], bot[tid]), q = max(top[tid], bot[tid]);
                const float apq = A[p * LD + q];
                float c = 1.0f, s = 0.0f;
                if (apq != 0.0f) {
                    const float tau = (A[q * LD + q] - A[p * LD + p]) / (2.0f * apq);
                    const float t = (tau >= 0.0f ? 1.0f : -1.0f) / (fabsf(tau) + sqrtf(1.0f + tau * tau));
                    c = rsqrtf(1.0f + t * t);
                    s = t * c;
                }
                cs[tid] = c;
                sn[tid] = s;
            }
            __syncthreads();
            // rows p, q <- J^T: (c row_p - s row_q, s row_p + c row_q)
            for (int e = tid; e < NP * D; e += kJacThreads) {
                const int k = e / D, j = e % D;
                const int p = min(top[k], bot[k]), q = max(top[k], bot[k]);
                const float c = cs[k], s = sn[k];
                const float ap = A[p * LD + j], aq = A[q * LD + j];
                A[p * LD + j] = c * ap - s * aq;
                A[q * LD + j] = s * ap + c * aq;
            }
            __syncthreads();
            // columns p, q of A and V <- J
            for (int e = tid; e < NP * D; e += kJacThreads) {
                const int k = e / D, i = e % D;
                const int p = min(top[k], bot[k]), q = max(top[k], bot[k]);
                const float c = cs[k], s = sn[k];
                const float ap = A[i * LD + p], aq = A[i * LD + q];
                A[i * LD + p] = c * ap - s * aq;
                A[i * LD + q] = s * ap + c * aq;
                const float vp = V[i * LD + p], vq = V[i * LD + q];
                V[i * LD + p] = c * vp - s * vq;
                V[i * LD + q] = s * vp + c * vq;
            }
            __syncthreads();
            // next pairing (round-robin: player 0 stays, the others rotate)
            if (tid == 0) {
                const int last_top = top[NP - 1];
                for (int k = NP - 1; k > 1; --k) top[k] = top[k - 1];
                if (NP > 1) top[1] = bot[0];
                for (int k = 0; k < NP - 1; ++k) bot[k] = bot[k + 1];
                bot[NP - 1] = last_top;
            }
            __syncthreads();
        }
    }
    // descending order of the eigenvalues (ties: lower index first); the identity first, so that
    // every entry is a valid column even if a non-finite input made two ranks coincide
    if (tid < D) order[tid] = tid;
    __syncthreads();
    if (tid < D) {
        const float li = A[tid * LD + tid];
        int rank = 0;
        for (int j = 0; j < D; ++j) {
            const float lj = A[j * LD + j];
            rank += (lj > li || (lj == li && j < tid)) ? 1 : 0;
        }
        order[rank] = tid;
    }
    __syncthreads();
    // columns k < S: one warp per column, sign from the largest-magnitude entry (first on ties)
    for (int k = warp; k < S; k += kJacThreads / 32) {
        const int col = order[k];
        float best = -1.0f;
        int bi = 0;  // a valid row even when every entry is NaN
        for (int i = lane; i < D; i += 32) {
            const float a = fabsf(V[i * LD + col]);
            if (a > best) {
                best = a;
                bi = i;
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ob > best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
            }
        }
        // the rotations' rounding leaves the columns orthogonal to about 1e-7 but lets their
        // lengths drift (about 1e-7 per rotation of the column): divide by the length
        float ss = 0.0f;
        for (int i = lane; i < D; i += 32) ss = fmaf(V[i * LD + col], V[i * LD + col], ss);
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float scale = (V[bi * LD + col] < 0.0f ? -1.0f : 1.0f) * (ss > 0.0f ? rsqrtf(ss) : 1.0f);
        for (int i = lane; i < D; i += 32) basis[(size_t)i * S + k] = scale * V[i * LD + col];
        if (lane == 0 && evals != nullptr) evals[k] = A[col * LD + col];
    }
}

template <int D>
size_t jacobi_smem() { return (size_t)2 * D * (D + 1) * sizeof(float); }

int moment_parts(long long n) {
    return (int)std::max<long long>(1, std::min<long long>((n + 255) / 256, 2LL * sm_count()));
}

template <typename T, int D>
cudaError_t launch_basis_t(const Dims& m, const T* Q, long long n, float* basis, float* evals, void* ws,
                           cudaStream_t s) {
    const int parts = moment_parts(n);
    float* part = static_cast<float*>(ws);
    float* M = part + (size_t)parts * D * D;
    count_launch();
    moment_partial_kernel<T, D><<<parts, kMomThreads, 0, s>>>(Q, n, parts, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    moment_reduce_kernel<D><<<(D * D + 255) / 256, 256, 0, s>>>(part, parts, n, M);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem = jacobi_smem<D>();
    e = cudaFuncSetAttribute(jacobi_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    jacobi_kernel<D><<<1, kJacThreads, smem, s>>>(M, m.sub, basis, evals);
    return cudaGetLastError();
}

}  // namespace

size_t basis_workspace_bytes(const Dims& m) {
    return ((size_t)2 * sm_count() + 1) * m.d * m.d * sizeof(float);
}

cudaError_t launch_query_basis(const Dims& m, const void* Q, long long n, float* basis, float* evals, void* ws,
                               cudaStream_t s) {
    if (m.dtype == COBS_BF16) {
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
        return m.d == 128 ? launch_basis_t<__nv_bfloat16, 128>(m, q, n, basis, evals, ws, s)
                          : launch_basis_t<__nv_bfloat16, 64>(m, q, n, basis, evals, ws, s);
    }
    const float* q = static_cast<const float*>(Q);
    return m.d == 128 ? launch_basis_t<float, 128>(m, q, n, basis, evals, ws, s)
                      : launch_basis_t<float, 64>(m, q, n, basis, evals, ws, s);
}

}  // namespace cobs
