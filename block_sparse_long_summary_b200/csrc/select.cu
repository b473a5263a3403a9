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

#include <algorithm>

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

// Same canonical score, with the group query held in registers: lane l keeps channels
// 4l .. 4l + 3 of Qsum and Q2 and the other lanes read them by shuffle (keeps shared memory for
// the summary tile alone).
template <int D>
__device__ __forceinline__ float block_score_regq(const float* tile, float4 qs4, float4 q24, int lane, float isd,
                                                  float c2) {
    const float4* mu4 = reinterpret_cast<const float4*>(tile) + lane;
    const float4* var4 = reinterpret_cast<const float4*>(tile + D * 32) + lane;
    float a = 0.0f, v = 0.0f;
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 m = mu4[c4 * 32];
        const float4 s = var4[c4 * 32];
        const float qa = __shfl_sync(kFull, qs4.x, c4), qb = __shfl_sync(kFull, qs4.y, c4);
        const float qc = __shfl_sync(kFull, qs4.z, c4), qd = __shfl_sync(kFull, qs4.w, c4);
        const float ra = __shfl_sync(kFull, q24.x, c4), rb = __shfl_sync(kFull, q24.y, c4);
        const float rc = __shfl_sync(kFull, q24.z, c4), rd = __shfl_sync(kFull, q24.w, c4);
        a = __fmaf_rn(qa, m.x, a);
        a = __fmaf_rn(qb, m.y, a);
        a = __fmaf_rn(qc, m.z, a);
        a = __fmaf_rn(qd, m.w, a);
        v = __fmaf_rn(ra, s.x, v);
        v = __fmaf_rn(rb, s.y, v);
        v = __fmaf_rn(rc, s.z, v);
        v = __fmaf_rn(rd, s.w, v);
    }
    return __fmaf_rn(c2, v, __fmul_rn(a, isd));
}

// ---------------------------------------------------------------------------- decode
// Warp-wide sorted list helpers: one (score, index) entry per lane, best first.
__device__ __forceinline__ void cmp_swap(float& s, int& i, int j, bool up, int lane) {
    const float os = __shfl_xor_sync(kFull, s, j);
    const int oi = __shfl_xor_sync(kFull, i, j);
    const bool low = (lane & j) == 0;
    const bool ob = better(os, oi, s, i);
    if ((low == up) ? ob : (!ob && !(os == s && oi == i))) {
        s = os;
        i = oi;
    }
}

// Sort the 32 entries best first (bitonic network).
__device__ __forceinline__ void warp_sort_best_first(float& s, int& i, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) cmp_swap(s, i, j, (lane & k) == 0, lane);
    }
}

// (s, i) and (bs, bi) are both sorted best first; keep the best 32 of their union, sorted.
__device__ __forceinline__ void warp_merge_best_first(float& s, int& i, float bs, int bi, int lane) {
    const float rs = __shfl_sync(kFull, bs, 31 - lane);
    const int ri = __shfl_sync(kFull, bi, 31 - lane);
    if (better(rs, ri, s, i)) {
        s = rs;
        i = ri;
    }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) cmp_swap(s, i, j, true, lane);
}

#ifndef COBS_SELECT_WARPS
#define COBS_SELECT_WARPS 1
#endif
constexpr int kSelWarps = COBS_SELECT_WARPS;
constexpr int kMaxSplit = 32;

// grid (nsplit, units), 2 warps. Warp w of split s scores groups [(s*2 + w)*gpw, +gpw) of its
// unit: each group (32 blocks, 32 KiB) arrives with one bulk (TMA) copy into the warp's own
// buffer (two buffers when a warp has several groups), lane = block, and the warp keeps a sorted
// best-first list (bitonic sort + merge). The CTA's two lists are merged in shared memory. With
// one split the CTA writes the answer; otherwise every CTA deposits its list and takes an atomic
// ticket (nobody waits), and the CTA that takes the last ticket merges all lists of the unit
// with a shared-memory tree. The ticket counter returns to zero by itself. The result is the
// top-k under a strict total order, so it does not depend on arrival order.
template <typename T, int D>
__global__ void __launch_bounds__(kSelWarps * 32) select_decode_kernel(
    const T* __restrict__ Q, const float* __restrict__ summ, int32_t* __restrict__ idx, float* __restrict__ ws_s,
    int* __restrict__ ws_i, unsigned* __restrict__ ws_ctr, int G, int nG, int ncand, int k, int gpw, int nsplit,
    float isd, float c2, int* err) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bar[kSelWarps][2];
    __shared__ unsigned ticket_sh;
    constexpr uint32_t kTileBytes = 2 * D * 32 * 4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int unit = blockIdx.y;
    const int split = blockIdx.x;
    const int nGc = (ncand + kGroupBlocks - 1) / kGroupBlocks;
    const float* usum = summ + (size_t)unit * nG * 2 * D * 32;
    const int stages = gpw > 1 ? 2 : 1;
    float* tiles = reinterpret_cast<float*>(smem_raw) + (size_t)warp * stages * 2 * D * 32;
    const int g0 = (split * kSelWarps + warp) * gpw;
    const int g1 = min(nGc, g0 + gpw);
    if (lane == 0) {
        mbar_init(&bar[warp][0], 1);
        mbar_init(&bar[warp][1], 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (lane == 0) {
        for (int st = 0; st < stages && g0 + st < g1; ++st) {
            mbar_arrive_expect_tx(&bar[warp][st], kTileBytes);
            bulk_g2s(tiles + st * 2 * D * 32, usum + (size_t)(g0 + st) * 2 * D * 32, kTileBytes, &bar[warp][st]);
        }
    }
    // group query in registers: lane l holds channels 4l .. 4l + 3
    // (unit = b * Hkv + g and Hq = Hkv * G, so the group's first head row is unit * G)
    float4 qs4 = make_float4(0.f, 0.f, 0.f, 0.f), q24 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane * 4 < D) {
        const T* qg = Q + (size_t)unit * G * D;
        group_query(qg, G, D, 4 * lane + 0, qs4.x, q24.x);
        group_query(qg, G, D, 4 * lane + 1, qs4.y, q24.y);
        group_query(qg, G, D, 4 * lane + 2, qs4.z, q24.z);
        group_query(qg, G, D, 4 * lane + 3, qs4.w, q24.w);
    }

    float ls = -INFINITY;
    int li = kInvalid;
    bool ok = true;
    for (int g = g0, it = 0; g < g1; ++g, ++it) {
        const int st = it % stages;
        const uint32_t parity = (it / stages) & 1;
        if (ok) ok = mbar_wait(&bar[warp][st], parity, err);
        ok = __all_sync(kFull, ok);
        const int b = g * kGroupBlocks + lane;
        float sc = -INFINITY;
        int bi = kInvalid;
        if (ok) {  // warp-uniform: every lane takes part in the score's shuffles
            const float s_all = block_score_regq<D>(tiles + st * 2 * D * 32, qs4, q24, lane, isd, c2);
            if (b < ncand) {
                sc = s_all;
                bi = b;
            }
        }
        __syncwarp();
        if (lane == 0 && ok && g + stages < g1) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&bar[warp][st], kTileBytes);
            bulk_g2s(tiles + st * 2 * D * 32, usum + (size_t)(g + stages) * 2 * D * 32, kTileBytes, &bar[warp][st]);
        }
        warp_sort_best_first(sc, bi, lane);
        if (it == 0) {
            ls = sc;
            li = bi;
        } else {
            warp_merge_best_first(ls, li, sc, bi, lane);
        }
    }
    // the tile buffers are free once every warp is done: reuse them for the list merges
    __syncthreads();
    float (*ls_sh)[32] = reinterpret_cast<float (*)[32]>(smem_raw);
    int (*li_sh)[32] = reinterpret_cast<int (*)[32]>(smem_raw + kMaxSplit * 32 * sizeof(float));
    ls_sh[warp][lane] = ls;
    li_sh[warp][lane] = li;
    __syncthreads();
    if (warp == 0) {
        for (int w = 1; w < kSelWarps; ++w) warp_merge_best_first(ls, li, ls_sh[w][lane], li_sh[w][lane], lane);
        if (nsplit == 1) {
            const int key = warp_sort_asc(lane < k ? li : kInvalid, lane);
            if (lane < k) idx[(size_t)unit * k + lane] = key == kInvalid ? -1 : key;
        } else {
            float* us = ws_s + ((size_t)unit * nsplit + split) * 32;
            int* ui = ws_i + ((size_t)unit * nsplit + split) * 32;
            us[lane] = ls;
            ui[lane] = li;
            __threadfence();
            __syncwarp();
            unsigned t = 0;
            if (lane == 0) t = atomicInc(ws_ctr + unit, (unsigned)(nsplit - 1));
            t = __shfl_sync(kFull, t, 0);
            if (lane == 0) ticket_sh = t;
        }
    }
    if (nsplit == 1) return;
    __syncthreads();
    if (ticket_sh != (unsigned)(nsplit - 1)) return;
    // last CTA of the unit: all lists into shared memory, then a merge tree over the warps
    __threadfence();
    for (int e = tid; e < nsplit * 32; e += blockDim.x) {
        ls_sh[e >> 5][e & 31] = __ldcg(ws_s + (size_t)unit * nsplit * 32 + e);
        li_sh[e >> 5][e & 31] = __ldcg(ws_i + (size_t)unit * nsplit * 32 + e);
    }
    __syncthreads();
    for (int width = 1; width < nsplit; width *= 2) {
        for (int pair = warp; pair * 2 * width < nsplit; pair += kSelWarps) {
            const int x = pair * 2 * width, y = x + width;
            if (y < nsplit) {
                float s1 = ls_sh[x][lane];
                int i1 = li_sh[x][lane];
                warp_merge_best_first(s1, i1, ls_sh[y][lane], li_sh[y][lane], lane);
                ls_sh[x][lane] = s1;
                li_sh[x][lane] = i1;
            }
        }
        __syncthreads();
    }
    if (warp == 0) {
        const int key = warp_sort_asc(lane < k ? li_sh[0][lane] : kInvalid, lane);
        if (lane < k) idx[(size_t)unit * k + lane] = key == kInvalid ? -1 : key;
    }
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
        // scores of this lane's block against the warp's 8 positions: 16 independent chains,
        // each in the canonical order (ascending channels, one fma per term)
        float av[kPfPerWarp], vv[kPfPerWarp];
#pragma unroll
        for (int j = 0; j < kPfPerWarp; ++j) av[j] = vv[j] = 0.0f;
        const float4* mu4 = reinterpret_cast<const float4*>(tile) + lane;
        const float4* var4 = reinterpret_cast<const float4*>(tile + D * 32) + lane;
        const float* sqw = sq + (size_t)(warp * kPfPerWarp) * 2 * D;
#pragma unroll 4
        for (int c4 = 0; c4 < D / 4; ++c4) {
            const float4 m = mu4[c4 * 32];
            const float4 vr = var4[c4 * 32];
#pragma unroll
            for (int j = 0; j < kPfPerWarp; ++j) {
                const float4 qa = reinterpret_cast<const float4*>(sqw + (j * 2 + 0) * D)[c4];
                const float4 qb = reinterpret_cast<const float4*>(sqw + (j * 2 + 1) * D)[c4];
                av[j] = __fmaf_rn(qa.x, m.x, av[j]);
                av[j] = __fmaf_rn(qa.y, m.y, av[j]);
                av[j] = __fmaf_rn(qa.z, m.z, av[j]);
                av[j] = __fmaf_rn(qa.w, m.w, av[j]);
                vv[j] = __fmaf_rn(qb.x, vr.x, vv[j]);
                vv[j] = __fmaf_rn(qb.y, vr.y, vv[j]);
                vv[j] = __fmaf_rn(qb.z, vr.z, vv[j]);
                vv[j] = __fmaf_rn(qb.w, vr.w, vv[j]);
            }
        }
        __syncthreads();  // every warp is done with this stage
        if (tid == 0 && ok && gi + 2 < ngroups) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * 2 * D * 32, usum + (size_t)(gi + 2) * 2 * D * 32, kTileBytes, &bar[st]);
        }
#pragma unroll
        for (int j = 0; j < kPfPerWarp; ++j) {
            const int t = t0 + warp * kPfPerWarp + j;
            const int nc = (t + 1) / L;
            const bool valid = ok && t < Tctx && blk < nc;
            float sc = __fmaf_rn(c2, vv[j], __fmul_rn(av[j], isd));
            int bi = blk;
            if (!valid) {
                sc = -INFINITY;
                bi = kInvalid;
            }
            const int nbetter = __popc(__ballot_sync(kFull, valid && better(sc, bi, tk[j].ts, tk[j].ti)));
            if (nbetter > 4) {
                // many newcomers (early groups): sort them and merge with the list
                warp_sort_best_first(sc, bi, lane);
                warp_merge_best_first(tk[j].s, tk[j].i, sc, bi, lane);
                if (lane >= k) {
                    tk[j].s = -INFINITY;
                    tk[j].i = kInvalid;
                }
                tk[j].ts = __shfl_sync(kFull, tk[j].s, k - 1);
                tk[j].ti = __shfl_sync(kFull, tk[j].i, k - 1);
            } else if (nbetter > 0) {
                tk[j].offer(sc, bi, valid, k, lane);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kPfPerWarp; ++j) {
        const int t = t0 + warp * kPfPerWarp + j;
        if (t < Tctx) emit_sorted(tk[j], k, lane, idx + (((size_t)b * Tctx + t) * Hkv + g) * k);
    }
}

// Decode selection split: each warp scores gpw consecutive 32-block groups, a CTA holds 2 warps,
// and a unit is covered by nsplit <= 32 CTAs.
void decode_split(const Dims& m, int& gpw, int& nsplit) {
    const int nGc = (m.T / m.L + 31) / 32;
    gpw = std::max(1, (nGc + kSelWarps * kMaxSplit - 1) / (kSelWarps * kMaxSplit));
    nsplit = std::max(1, (nGc + kSelWarps * gpw - 1) / (kSelWarps * gpw));
}

template <typename T, int D>
cudaError_t launch_select_t(const Dims& m, const T* Q, const float* summ, int prefill, int32_t* idx, void* ws,
                            cudaStream_t s, int* err) {
    float isd, c2;
    score_constants(m.d, m.alpha, &isd, &c2);
    const size_t tile_bytes = (size_t)2 * D * 32 * 4;
    if (!prefill) {
        const int ncand = m.T / m.L;
        int gpw, nsplit;
        decode_split(m, gpw, nsplit);
        unsigned char* w = static_cast<unsigned char*>(ws);
        unsigned* ws_ctr = reinterpret_cast<unsigned*>(w);
        size_t off = ((size_t)m.units() * sizeof(unsigned) + 255) & ~(size_t)255;
        float* ws_s = reinterpret_cast<float*>(w + off);
        off += (size_t)m.units() * nsplit * 32 * sizeof(float);
        int* ws_i = reinterpret_cast<int*>(w + off);
        const size_t smem = (size_t)kSelWarps * (gpw > 1 ? 2 : 1) * tile_bytes;
        cudaError_t e = cudaFuncSetAttribute(select_decode_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        count_launch();
        select_decode_kernel<T, D><<<dim3(nsplit, m.units()), kSelWarps * 32, smem, s>>>(
            Q, summ, idx, ws_s, ws_i, ws_ctr, m.G, m.nG, ncand, m.k, gpw, nsplit, isd, c2, err);
        return cudaGetLastError();
    }
    const size_t smem = tile_bytes * 2 + (size_t)kPfPos * 2 * D * 4;
    auto kern = select_prefill_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kern<<<dim3((m.T + kPfPos - 1) / kPfPos, m.units()), 128, smem, s>>>(Q, summ, idx, m.T, m.Hq, m.Hkv, m.G,
                                                                        m.nG, m.L, m.k, isd, c2, err);
    return cudaGetLastError();
}

}  // namespace

size_t select_workspace_bytes(const Dims& m, int prefill) {
    if (prefill) return 0;
    int gpw, nsplit;
    decode_split(m, gpw, nsplit);
    const size_t off = ((size_t)m.units() * sizeof(unsigned) + 255) & ~(size_t)255;
    return off + (size_t)m.units() * nsplit * 32 * (sizeof(float) + sizeof(int));
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
