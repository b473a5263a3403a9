// Cumulant-order block selection: score every candidate block against a GQA group's
// queries and keep the top-k, without writing scores to global memory.
//
// COBS (gist.science explainer) §2.3 "Second-Order Scoring": score_b = q.mean_b +
// 1/2 q^T Sigma_b q, here with the attention logit scale and the per-channel variance
// (diagonal Sigma_b); skill card "Implementation steps" 3: score = first-order term +
// alpha * cumulant term, keep the top-k blocks. One selection per GQA group: the group
// score is the sum of its heads' scores,
//   S_{g,b} = (sum_c Qsum_c mu_{b,c}) * isd + c2 * (sum_c Q2_c var_{b,c}),
// with Qsum = sum_h q_h and Q2 = sum_h q_h^2, isd = RN(1/sqrt(d)), c2 = RN(alpha/(2d)).
//
// Arithmetic is float32 in a fixed order (ascending heads, ascending channels, one
// correctly rounded FMA per term, never contracted further), so the selected indices
// are reproducible bit for bit. Ties go to the lower block index.
#include <float.h>

#include "common.cuh"
#include "dims.h"

namespace cobs {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kInvalid = 0x7fffffff;
constexpr int kGroupBlocks = 32;

__device__ __forceinline__ bool better(float s1, int i1, float s2, int i2) {
    return s1 > s2 || (s1 == s2 && i1 < i2);
}

// Warp-wide top-k list: lane j < k holds the j-th best (score desc, index asc);
// lanes >= k hold (-inf, kInvalid).
struct TopK {
    float s;
    int i;
    float ts;  // threshold = entry k-1
    int ti;
    __device__ void init() {
        s = -INFINITY;
        i = kInvalid;
        ts = -INFINITY;
        ti = kInvalid;
    }
    // Offer one candidate per lane (valid lanes only). Deterministic: the resulting set
    // is the top-k of the union under a strict total order, independent of lane order.
    __device__ void offer(float cs, int ci, bool valid, int k, int lane) {
        unsigned done = 0;
        unsigned mask = __ballot_sync(kFull, valid && better(cs, ci, ts, ti));
        while (mask) {
            const int src = __ffs(mask) - 1;
            const float ns = __shfl_sync(kFull, cs, src);
            const int ni = __shfl_sync(kFull, ci, src);
            const int p = __popc(__ballot_sync(kFull, lane < k && better(s, i, ns, ni)));
            const float us = __shfl_up_sync(kFull, s, 1);
            const int ui = __shfl_up_sync(kFull, i, 1);
            if (lane == p) {
                s = ns;
                i = ni;
            } else if (lane > p && lane < k) {
                s = us;
                i = ui;
            }
            ts = __shfl_sync(kFull, s, k - 1);
            ti = __shfl_sync(kFull, i, k - 1);
            done |= 1u << src;
            mask = __ballot_sync(kFull, valid && better(cs, ci, ts, ti)) & ~done;
        }
    }
};

// Ascending bitonic sort of one int key per lane.
__device__ __forceinline__ int warp_sort_asc(int key, int lane) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const int other = __shfl_xor_sync(kFull, key, stride);
            const bool up = (lane & size) == 0;
            const bool low = (lane & stride) == 0;
            key = (low == up) ? min(key, other) : max(key, other);
        }
    }
    return key;
}

// Write the list (lanes < k) in ascending block order, -1 for empty slots.
__device__ __forceinline__ void emit_sorted(const TopK& tk, int k, int lane, int32_t* out) {
    const int key = warp_sort_asc(lane < k ? tk.i : kInvalid, lane);
    if (lane < k) out[lane] = key == kInvalid ? -1 : key;
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Canonical group query: Qsum_c = sum_h q_{h,c}, Q2_c = fma-sum of q_{h,c}^2, ascending h.
template <typename T>
__device__ __forceinline__ void group_query(const T* q, int G, int d, int c, float& qs, float& q2) {
    float s = 0.0f, s2 = 0.0f;
    for (int h = 0; h < G; ++h) {
        const float x = to_f(q[(size_t)h * d + c]);
        s = __fadd_rn(s, x);
        s2 = __fmaf_rn(x, x, s2);
    }
    qs = s;
    q2 = s2;
}

// Canonical score of the block held by this lane (channel-interleaved group tile in smem).
template <int D>
__device__ __forceinline__ float block_score(const float* tile, const float* qs, const float* q2, int lane,
                                             float isd, float c2) {
    const float4* mu4 = reinterpret_cast<const float4*>(tile) + lane;
    const float4* var4 = reinterpret_cast<const float4*>(tile + D * 32) + lane;
    float a = 0.0f, v = 0.0f;
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 m = mu4[c4 * 32];
        a = __fmaf_rn(qs[4 * c4 + 0], m.x, a);
        a = __fmaf_rn(qs[4 * c4 + 1], m.y, a);
        a = __fmaf_rn(qs[4 * c4 + 2], m.z, a);
        a = __fmaf_rn(qs[4 * c4 + 3], m.w, a);
    }
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 s = var4[c4 * 32];
        v = __fmaf_rn(q2[4 * c4 + 0], s.x, v);
        v = __fmaf_rn(q2[4 * c4 + 1], s.y, v);
        v = __fmaf_rn(q2[4 * c4 + 2], s.z, v);
        v = __fmaf_rn(q2[4 * c4 + 3], s.w, v);
    }
    return __fmaf_rn(c2, v, __fmul_rn(a, isd));
}

// ---------------------------------------------------------------------------- decode
// grid (nsplit, units); one warp; the CTA scores groups [split*gpc, ...) of its unit with
// a 2-stage bulk-copy pipeline, keeps a top-k list, then either writes the answer (one
// split) or deposits its list and, if it is the last split of the unit to finish
// (atomic ticket, no waiting), merges all lists.
template <typename T, int D>
__global__ void __launch_bounds__(32) select_decode_kernel(const T* __restrict__ Q, const float* __restrict__ summ,
                                                           int32_t* __restrict__ idx, float* __restrict__ ws_s,
                                                           int* __restrict__ ws_i, unsigned* __restrict__ ws_ctr,
                                                           int G, int nG, int ncand, int k, int gpc, int nsplit,
                                                           float isd, float c2, int* err) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float* tiles = reinterpret_cast<float*>(smem_raw);  // [2][2*D*32]
    __shared__ float qs[D], q2[D];
    __shared__ __align__(8) uint64_t bar[2];
    const int lane = threadIdx.x;
    const int unit = blockIdx.y;
    const int split = blockIdx.x;
    const int nGc = (ncand + kGroupBlocks - 1) / kGroupBlocks;
    const int g0 = split * gpc;
    const int g1 = min(nGc, g0 + gpc);
    const float* usum = summ + (size_t)unit * nG * 2 * D * 32;
    constexpr uint32_t kTileBytes = 2 * D * 32 * 4;

    if (lane == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_barrier_init();
    }
    __syncwarp();
    // prologue: first two tiles in flight
    if (lane == 0) {
        for (int st = 0; st < 2 && g0 + st < g1; ++st) {
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * 2 * D * 32, usum + (size_t)(g0 + st) * 2 * D * 32, kTileBytes, &bar[st]);
        }
    }
    // group query (all lanes), overlapped with the copies
    {
        // unit = b * Hkv + g and Hq = Hkv * G, so the group's first head row is unit * G
        const T* qg = Q + (size_t)unit * G * D;
        for (int c = lane; c < D; c += 32) group_query(qg, G, D, c, qs[c], q2[c]);
    }
    __syncwarp();

    TopK tk;
    tk.init();
    bool ok = true;
    for (int g = g0, it = 0; g < g1; ++g, ++it) {
        const int st = it & 1;
        const uint32_t parity = (it >> 1) & 1;
        if (ok) ok = mbar_wait(&bar[st], parity, err);
        ok = __all_sync(kFull, ok);
        const int b = g * kGroupBlocks + lane;
        float sc = -INFINITY;
        if (ok) sc = block_score<D>(tiles + st * 2 * D * 32, qs, q2, lane, isd, c2);
        __syncwarp();
        // refill this stage with group g + 2
        if (lane == 0 && ok && g + 2 < g1) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * 2 * D * 32, usum + (size_t)(g + 2) * 2 * D * 32, kTileBytes, &bar[st]);
        }
        tk.offer(sc, b, ok && b < ncand, k, lane);
    }

    if (nsplit == 1) {
        emit_sorted(tk, k, lane, idx + (size_t)unit * k);
        return;
    }
    float* my_s = ws_s + ((size_t)unit * nsplit + split) * k;
    int* my_i = ws_i + ((size_t)unit * nsplit + split) * k;
    if (lane < k) {
        my_s[lane] = tk.s;
        my_i[lane] = tk.i;
    }
    __threadfence();
    __syncwarp();
    unsigned ticket = 0;
    if (lane == 0) ticket = atomicInc(ws_ctr + unit, (unsigned)(nsplit - 1));
    ticket = __shfl_sync(kFull, ticket, 0);
    if (ticket != (unsigned)(nsplit - 1)) return;
    __threadfence();
    TopK all;
    all.init();
    for (int sp = 0; sp < nsplit; ++sp) {
        const float* ps = ws_s + ((size_t)unit * nsplit + sp) * k;
        const int* pi = ws_i + ((size_t)unit * nsplit + sp) * k;
        float cs = -INFINITY;
        int ci = kInvalid;
        if (lane < k) {
            cs = __ldcg(ps + lane);
            ci = __ldcg(pi + lane);
        }
        all.offer(cs, ci, lane < k && ci != kInvalid, k, lane);
    }
    emit_sorted(all, k, lane, idx + (size_t)unit * k);
}

// ---------------------------------------------------------------------------- prefill
// grid (ceil(T / 32), B * Hkv); 4 warps x 8 positions = a tile of 32 consecutive positions.
// Candidates at position t are blocks b < (t+1)/L. Each warp keeps one top-k list per
// position (lanes = list slots) and scores 32 blocks per smem tile (lane = block).
constexpr int kPfPos = 32;
constexpr int kPfWarps = 4;
constexpr int kPfPerWarp = kPfPos / kPfWarps;

template <typename T, int D>
__global__ void __launch_bounds__(128) select_prefill_kernel(const T* __restrict__ Q, const float* __restrict__ summ,
                                                             int32_t* __restrict__ idx, int Tctx, int Hq, int Hkv,
                                                             int G, int nG, int L, int k, float isd, float c2,
                                                             int* err) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float* tiles = reinterpret_cast<float*>(smem_raw);           // [2][2*D*32]
    float* sq = tiles + 2 * 2 * D * 32;                            // [kPfPos][2][D]: Qsum, Q2
    __shared__ __align__(8) uint64_t bar[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int unit = blockIdx.y;
    const int b = unit / Hkv, g = unit % Hkv;
    const int t0 = blockIdx.x * kPfPos;
    const int tlast = min(Tctx - 1, t0 + kPfPos - 1);
    const int ncand_max = (tlast + 1) / L;
    const int ngroups = (ncand_max + kGroupBlocks - 1) / kGroupBlocks;
    const float* usum = summ + (size_t)unit * nG * 2 * D * 32;
    constexpr uint32_t kTileBytes = 2 * D * 32 * 4;

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int st = 0; st < 2 && st < ngroups; ++st) {
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * 2 * D * 32, usum + (size_t)st * 2 * D * 32, kTileBytes, &bar[st]);
        }
    }
    // group queries of the tile's positions
    for (int e = tid; e < kPfPos * D; e += blockDim.x) {
        const int p = e / D, c = e % D;
        const int t = t0 + p;
        float a = 0.0f, a2 = 0.0f;
        if (t < Tctx) group_query(Q + (((size_t)b * Tctx + t) * Hq + (size_t)g * G) * D, G, D, c, a, a2);
        sq[(p * 2 + 0) * D + c] = a;
        sq[(p * 2 + 1) * D + c] = a2;
    }
    __syncthreads();

    TopK tk[kPfPerWarp];
#pragma unroll
    for (int j = 0; j < kPfPerWarp; ++j) tk[j].init();
    bool ok = true;
    for (int gi = 0; gi < ngroups; ++gi) {
        const int st = gi & 1;
        const uint32_t parity = (gi >> 1) & 1;
        if (ok) ok = mbar_wait(&bar[st], parity, err);
        ok = __syncthreads_and(ok) != 0;
        const float* tile = tiles + st * 2 * D * 32;
        const int blk = gi * kGroupBlocks + lane;
#pragma unroll
        for (int j = 0; j < kPfPerWarp; ++j) {
            const int p = warp * kPfPerWarp + j;
            const int t = t0 + p;
            const int nc = (t + 1) / L;
            float sc = -INFINITY;
            const bool valid = ok && t < Tctx && blk < nc;
            if (__any_sync(kFull, valid)) {
                sc = block_score<D>(tile, sq + (p * 2 + 0) * D, sq + (p * 2 + 1) * D, lane, isd, c2);
                tk[j].offer(sc, blk, valid, k, lane);
            }
        }
        __syncthreads();  // every warp is done with this stage
        if (tid == 0 && ok && gi + 2 < ngroups) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * 2 * D * 32, usum + (size_t)(gi + 2) * 2 * D * 32, kTileBytes, &bar[st]);
        }
    }
#pragma unroll
    for (int j = 0; j < kPfPerWarp; ++j) {
        const int t = t0 + warp * kPfPerWarp + j;
        if (t < Tctx) emit_sorted(tk[j], k, lane, idx + (((size_t)b * Tctx + t) * Hkv + g) * k);
    }
}

template <typename T, int D>
cudaError_t launch_select_t(const Dims& m, const T* Q, const float* summ, int prefill, int32_t* idx, void* ws,
                            cudaStream_t s, int* err) {
    float isd, c2;
    score_constants(m.d, m.alpha, &isd, &c2);
    const size_t tile_bytes = (size_t)2 * D * 32 * 4;
    if (!prefill) {
        const int ncand = m.T / m.L;
        const int nGc = (ncand + 31) / 32;
        int gpc = 1;
        while ((nGc + gpc - 1) / gpc > 64) gpc *= 2;  // at most 64 lists to merge per unit
        const int nsplit = nGc == 0 ? 1 : (nGc + gpc - 1) / gpc;
        float* ws_s = nullptr;
        int* ws_i = nullptr;
        unsigned* ws_ctr = nullptr;
        if (nsplit > 1) {
            unsigned char* w = static_cast<unsigned char*>(ws);
            ws_ctr = reinterpret_cast<unsigned*>(w);
            size_t off = ((size_t)m.units() * sizeof(unsigned) + 255) & ~(size_t)255;
            ws_s = reinterpret_cast<float*>(w + off);
            off += (size_t)m.units() * nsplit * m.k * sizeof(float);
            ws_i = reinterpret_cast<int*>(w + off);
        }
        const size_t smem = tile_bytes * (gpc > 1 ? 2 : 1);
        auto kern = select_decode_kernel<T, D>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        count_launch();
        count_launch();
        kern<<<dim3(nsplit, m.units()), 32, smem, s>>>(Q, summ, idx, ws_s, ws_i, ws_ctr, m.G, m.nG, ncand, m.k,
                                                     gpc, nsplit, isd, c2, err);
        return cudaGetLastError();
    }
    const size_t smem = tile_bytes * 2 + (size_t)kPfPos * 2 * D * 4;
    auto kern = select_prefill_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    count_launch();
    kern<<<dim3((m.T + kPfPos - 1) / kPfPos, m.units()), 128, smem, s>>>(Q, summ, idx, m.T, m.Hq, m.Hkv, m.G,
                                                                        m.nG, m.L, m.k, isd, c2, err);
    return cudaGetLastError();
}

}  // namespace

size_t select_workspace_bytes(const Dims& m, int prefill) {
    if (prefill) return 0;
    const int ncand = m.T / m.L;
    const int nGc = (ncand + 31) / 32;
    int gpc = 1;
    while ((nGc + gpc - 1) / gpc > 64) gpc *= 2;
    const int nsplit = nGc == 0 ? 1 : (nGc + gpc - 1) / gpc;
    if (nsplit <= 1) return 0;
    size_t off = ((size_t)m.units() * sizeof(unsigned) + 255) & ~(size_t)255;
    return off + (size_t)m.units() * nsplit * m.k * (sizeof(float) + sizeof(int));
}

cudaError_t launch_select(const Dims& m, const void* Q, const float* summ, int prefill, int32_t* idx, void* ws,
                          cudaStream_t s, int* err) {
    if (m.dtype == COBS_BF16) {
        if (m.d == 128)
            return launch_select_t<__nv_bfloat16, 128>(m, (const __nv_bfloat16*)Q, summ, prefill, idx, ws, s, err);
        return launch_select_t<__nv_bfloat16, 64>(m, (const __nv_bfloat16*)Q, summ, prefill, idx, ws, s, err);
    }
    if (m.d == 128) return launch_select_t<float, 128>(m, (const float*)Q, summ, prefill, idx, ws, s, err);
    return launch_select_t<float, 64>(m, (const float*)Q, summ, prefill, idx, ws, s, err);
}

}  // namespace cobs
