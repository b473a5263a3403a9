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

#include <cuda_fp16.h>

#include "common.cuh"
#include "dims.h"
#include "select_core.cuh"
#include "tma.h"

namespace cobs {
namespace {

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


// Write the list (lanes < k) in ascending block order, -1 for empty slots.
__device__ __forceinline__ void emit_sorted(const TopK& tk, int k, int lane, int32_t* out) {
    const int key = warp_sort_asc(lane < k ? tk.i : kInvalid, lane);
    if (lane < k) out[lane] = key == kInvalid ? -1 : key;
}


// Canonical score of the block held by this lane (channel-interleaved group tile in smem): the
// mean half and the variance half are independent chains, combined once.
template <int D>
__device__ __forceinline__ float block_score(const float* tile, const float* qs, const float* q2, int lane,
                                             float isd, float c2) {
    return score_combine(score_mean_part<D>(tile, qs, lane), score_var_part<D>(tile + D * 32, q2, lane), isd, c2);
}

// Canonical isotropic score: the same mean sum, then v = RN(Q2tot * sigma2_b) with the block's
// one variance scalar (stored after the group's means) and Q2tot = sum_c Q2_c.
template <int D>
__device__ __forceinline__ float block_score_iso(const float* tile, const float* qs, float q2tot, int lane, float isd,
                                                 float c2) {
    const float4* mu4 = reinterpret_cast<const float4*>(tile) + lane;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 m = mu4[c4 * 32];
        const float4 q = reinterpret_cast<const float4*>(qs)[c4];
        a0 = __fmaf_rn(q.x, m.x, a0);
        a1 = __fmaf_rn(q.y, m.y, a1);
        a2 = __fmaf_rn(q.z, m.z, a2);
        a3 = __fmaf_rn(q.w, m.w, a3);
    }
    const float v = __fmul_rn(q2tot, tile[D * 32 + lane]);
    return __fmaf_rn(c2, v, __fmul_rn(combine4(a0, a1, a2, a3), isd));
}

// Canonical low-rank score on S-coordinate eigenvectors: a = four-chain sum over c of Qsum_c mu_c, then
//   v = sum over j ascending of fma(lambda_j, e_j, .), e_j = sum over h ascending of fma(p, p, .),
//   p = four-chain sum over i < S of q~_{h,i} u~_{j,i} (coordinate i to chain i mod 4);
// the tile holds the 32 blocks' means, then the S coordinates of eigenvector j < R in an
// [S/4][32][4] interleaving, then the R x 32 eigenvalues. qt: the group's heads [G][S], projected
// on the subspace basis (query-subspace summaries) or as they are with S = D (low-rank summaries,
// whose layout is this one with S = D).
template <int D>
__device__ __forceinline__ float block_score_sub(const float* tile, const float* qs, const float* qt, int G, int R,
                                                 int S, int lane, float isd, float c2) {
    const float4* mu4 = reinterpret_cast<const float4*>(tile) + lane;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 m = mu4[c4 * 32];
        const float4 q = reinterpret_cast<const float4*>(qs)[c4];
        a0 = __fmaf_rn(q.x, m.x, a0);
        a1 = __fmaf_rn(q.y, m.y, a1);
        a2 = __fmaf_rn(q.z, m.z, a2);
        a3 = __fmaf_rn(q.w, m.w, a3);
    }
    const int S4 = S / 4;
    float v = 0.0f;
    for (int j = 0; j < R; ++j) {
        const float4* u4 = reinterpret_cast<const float4*>(tile + (size_t)32 * D + (size_t)j * S * 32) + lane;
        float e = 0.0f;
        for (int hb = 0; hb < G; hb += 4) {  // each coordinate of u~_j read once per four heads
            float p[4][4];
#pragma unroll
            for (int h = 0; h < 4; ++h) p[h][0] = p[h][1] = p[h][2] = p[h][3] = 0.0f;
#pragma unroll 3
            for (int i4 = 0; i4 < S4; ++i4) {
                const float4 uu = u4[i4 * 32];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    if (hb + h < G) {
                        const float4 q = reinterpret_cast<const float4*>(qt + (size_t)(hb + h) * S)[i4];
                        p[h][0] = __fmaf_rn(q.x, uu.x, p[h][0]);
                        p[h][1] = __fmaf_rn(q.y, uu.y, p[h][1]);
                        p[h][2] = __fmaf_rn(q.z, uu.z, p[h][2]);
                        p[h][3] = __fmaf_rn(q.w, uu.w, p[h][3]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                if (hb + h < G) {
                    const float pj = combine4(p[h][0], p[h][1], p[h][2], p[h][3]);
                    e = __fmaf_rn(pj, pj, e);
                }
            }
        }
        v = __fmaf_rn(tile[(size_t)32 * (D + R * S) + j * 32 + lane], e, v);
    }
    return __fmaf_rn(c2, v, __fmul_rn(combine4(a0, a1, a2, a3), isd));
}

// Query heads projected on the subspace basis, q~_{h,i} = four-chain sum over c of P[c][i] q_{h,c}
// (channel c to chain c mod 4, ascending c; chains combined as (s0 + s1) + (s2 + s3)).
// grid (units, ceil(G S / 64)), 256 threads: four threads per output, thread k of the four runs
// chain k (D/4 independent loads of P, then its fused multiply-adds), and two shuffles combine
// the chains. Out: qt [units][G][S] float32. The selection grid that follows is launched as its
// programmatic dependent and waits for this grid before reading qt.
template <typename T, int D>
__global__ void __launch_bounds__(256) project_queries_kernel(const T* __restrict__ Q, const float* __restrict__ P,
                                                              int G, int S, float* __restrict__ qt) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ __align__(16) float qh[kMaxGroup * D];
    const int u = blockIdx.x;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) qh[e] = to_f(Q[(size_t)u * G * D + e]);
    __syncthreads();
    const int o = blockIdx.y * 64 + (threadIdx.x >> 2), k = threadIdx.x & 3;
    const bool live = o < G * S;
    const int h = live ? o / S : 0, i = live ? o % S : 0;
    float acc = 0.0f;
    if (live) {
        float pv[D / 4];
#pragma unroll
        for (int n = 0; n < D / 4; ++n) pv[n] = __ldg(P + (size_t)(4 * n + k) * S + i);
#pragma unroll
        for (int n = 0; n < D / 4; ++n) acc = __fmaf_rn(pv[n], qh[h * D + 4 * n + k], acc);
    }
    // lanes 4m..4m+3 hold chains 0..3 of one output
    const float pair = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, 1));    // s0 + s1 at k = 0, s2 + s3 at k = 2
    const float all = __fadd_rn(pair, __shfl_xor_sync(kFull, pair, 2));   // (s0 + s1) + (s2 + s3) at k = 0
    if (live && k == 0) qt[(size_t)u * G * S + o] = all;
}

// Two E2M1 codes (one byte: the first channel in the low nibble) to two exact half values with
// sm_100a's FP4 conversion.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(out) : "r"(byte));
    return out;
}

// Canonical low-rank score from FP4 summaries: the bf16 means and the dequantized vectors
// u'_i = value(code_i) * scale_j (one rounded multiply), then the low-rank score's sums. Tile
// bytes: bf16 means [D/8][32][8], codes of vector j [CW/32][32][16] (entry 2i in the low nibble
// of byte i), scales [R][32] f32, eigenvalues [R][32] f32. SUB = false: the vectors are the
// eigenvectors (CW = S = D) and qh the heads [G][D]; SUB = true: the S coordinates of the
// eigenvectors in the query subspace (CW = S rounded up to 32, codes past S zero) and qh the
// projected heads [G][S] (S a multiple of 4: coordinate i to chain i mod 4, as the channels).
template <int D, bool SUB>
__device__ __forceinline__ float block_score_fp4(const float* tile, const float* qs, const float* qh, int G, int R,
                                                 int S_, int lane, float isd, float c2) {
    const int S = SUB ? S_ : D;
    const int CW = SUB ? (S_ + 31) / 32 * 32 : D;
    const unsigned char* t8 = reinterpret_cast<const unsigned char*>(tile);
    float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 wv = *reinterpret_cast<const uint4*>(t8 + ((size_t)c8 * 32 + lane) * 16);
        const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint32_t hw = (w4[t >> 1] >> ((t & 1) * 16)) & 0xFFFFu;
            const float mu = __uint_as_float(hw << 16);
            a[t & 3] = __fmaf_rn(qs[8 * c8 + t], mu, a[t & 3]);
        }
    }
    const float* scl = reinterpret_cast<const float*>(t8 + (size_t)64 * D + (size_t)R * 16 * CW);
    const float* lam = scl + R * 32;
    float v = 0.0f;
    for (int j = 0; j < R; ++j) {
        const float sj = scl[j * 32 + lane];
        const unsigned char* cj = t8 + (size_t)64 * D + (size_t)j * 16 * CW;
        // heads in fours: each 32-channel chunk is decoded once per four heads
        // (u'_c = value * scale, one rounded multiply)
        float e = 0.0f;
        for (int hb = 0; hb < G; hb += 4) {
            float p[4][4];
#pragma unroll
            for (int h = 0; h < 4; ++h) p[h][0] = p[h][1] = p[h][2] = p[h][3] = 0.0f;
            for (int w = 0; w < CW / 32; ++w) {
                const uint4 wv = *reinterpret_cast<const uint4*>(cj + ((size_t)w * 32 + lane) * 16);
                const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
                float u[32];
#pragma unroll
                for (int bi = 0; bi < 16; ++bi) {
                    const uint32_t h2 = e2m1x2_to_f16x2((w4[bi >> 2] >> ((bi & 3) * 8)) & 0xFFu);
                    u[2 * bi] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))), sj);
                    u[2 * bi + 1] = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h2 >> 16))), sj);
                }
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    if (hb + h < G) {
                        const float4* q4 = reinterpret_cast<const float4*>(qh + (size_t)(hb + h) * S) + w * 8;
#pragma unroll
                        for (int t4 = 0; t4 < 8; ++t4) {
                            if (SUB && w * 32 + t4 * 4 >= S) break;  // past the S coordinates
                            const float4 q = q4[t4];
                            p[h][0] = __fmaf_rn(q.x, u[4 * t4 + 0], p[h][0]);
                            p[h][1] = __fmaf_rn(q.y, u[4 * t4 + 1], p[h][1]);
                            p[h][2] = __fmaf_rn(q.z, u[4 * t4 + 2], p[h][2]);
                            p[h][3] = __fmaf_rn(q.w, u[4 * t4 + 3], p[h][3]);
                        }
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                if (hb + h < G) {
                    const float pj = combine4(p[h][0], p[h][1], p[h][2], p[h][3]);
                    e = __fmaf_rn(pj, pj, e);
                }
            }
        }
        v = __fmaf_rn(lam[j * 32 + lane], e, v);
    }
    return __fmaf_rn(c2, v, __fmul_rn(combine4(a[0], a[1], a[2], a[3]), isd));
}


// Floats of one 32-block summary group: means + per-channel variances, or means + 32 scalars.
template <int D, bool ISO>
constexpr int group_floats() { return ISO ? (D + 1) * 32 : 2 * D * 32; }

// ---------------------------------------------------------------------------- decode
#ifndef COBS_SELECT_STAGES
#define COBS_SELECT_STAGES 2
#endif
#ifndef COBS_SELECT_CTAS_PER_SM
#define COBS_SELECT_CTAS_PER_SM 3
#endif
constexpr int kSelStages = COBS_SELECT_STAGES;
// At most this many one-warp selection CTAs per SM (twice as many for the FP4
// summaries, whose scoring is bound by arithmetic and whose tiles are small); the grid takes the
// smaller of this and the number that fit an SM with the mode's shared memory (2 for the float32
// low-rank summaries), so that every CTA is resident from the start.
constexpr int kSelCtasPerSm = COBS_SELECT_CTAS_PER_SM;
// Upper bound of the decode selector's grid (any sm_100 part), fixing the workspace size
// without a device query.
constexpr int kSelGridCap = 192 * 2 * kSelCtasPerSm;

// Stream-K split of the decode selection: the n = units * nGc summary groups, unit-major, are
// cut into `grid` contiguous ranges [c n / grid, (c + 1) n / grid). CTA of group x:
__host__ __device__ __forceinline__ int sel_cta_of(long long x, long long n, int grid) {
    return (int)(((x + 1) * grid + n - 1) / n) - 1;
}

// Partial lists a unit can be split into (workspace slots per unit). The grid is capped so that
// a unit's groups meet at most min(nGc, ceil(grid / units) + 1) <= this many CTA ranges.
constexpr int kSelMaxSeg = 64;
inline int sel_max_segments(int units, int nGc) {
    return std::min(std::min(nGc, kSelMaxSeg), kSelGridCap / std::max(1, units) + 2);
}


// grid (G_sel), one warp per CTA, persistent. CTA c scores the summary groups of its stream-K
// range in order: each group (32 blocks, 2 d 32 floats) arrives by one bulk (TMA) copy into a
// kSelStages-deep ring, lane = block, and the group query of the current unit sits in shared
// memory (read as broadcasts). When the range leaves a unit, the CTA writes that unit's answer
// if it held the whole unit, else deposits its segment's exact top-k; select_merge_kernel (a
// dependent launch) merges the deposits. The result is the top-k under a strict total order,
// so it does not depend on the split.
// MODE 0: per-channel variance summaries, 1: isotropic, 2: low-rank (R eigenpairs, tile_floats
// floats per group, one ring stage, the group's query heads in shared memory after the ring),
// 3: low-rank with FP4 eigenvectors and bf16 means (as 2, with the ring of the other modes),
// 4: query subspace (as 2, with the projected heads qt_ws [units][G][S] written by
// project_queries_kernel, which this grid waits for, in place of the heads), 5: query subspace
// with FP4 coordinates and bf16 means (as 3, with the projected heads of 4).
template <typename T, int D, int MODE>
__global__ void __launch_bounds__(32) select_decode_kernel(const T* __restrict__ Q, const float* __restrict__ summ,
                                                           int32_t* __restrict__ idx, float* __restrict__ ws_s,
                                                           int* __restrict__ ws_i, int units, int G, int nG,
                                                           int ncand, int k, int maxseg,
                                                           float isd, float c2, int R, int tile_floats,
                                                           const float* qt_ws, int S, int* err) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bar[kSelStages];
    __shared__ __align__(16) float qsm[2][D];
    __shared__ float q2t_sm;
    constexpr bool ISO = MODE == 1;
    constexpr int kStg = (MODE == 2 || MODE == 4) ? 1 : kSelStages;
    constexpr bool kProj = MODE == 4 || MODE == 5;  // the projected heads of project_queries_kernel
    const int kTileFloats = MODE >= 2 ? tile_floats : group_floats<D, ISO>();
    const uint32_t kTileBytes = (uint32_t)kTileFloats * 4;
    // the merge grid may be scheduled now; it still waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x;
    const int grid = gridDim.x, c = blockIdx.x;
    const int nGc = (ncand + kGroupBlocks - 1) / kGroupBlocks;
    const long long n = (long long)units * nGc;
    float* tiles = reinterpret_cast<float*>(smem_raw);
    if (n == 0) {  // no complete block anywhere: every list is empty
        for (int u = c; u < units; u += grid)
            if (lane < k) idx[(size_t)u * k + lane] = -1;
        return;
    }
    const long long x0 = (long long)c * n / grid, x1 = (long long)(c + 1) * n / grid;
    if (x0 >= x1) return;
    auto group_src = [&](long long x) {
        const long long u = x / nGc, gl = x % nGc;
        return summ + ((size_t)u * nG + (size_t)gl) * kTileFloats;
    };
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < kStg; ++st) mbar_init(&bar[st], 1);
        fence_barrier_init();
    }
    __syncwarp();
    // the first kAhead tiles now; every later tile once the tile before it has landed (rings of
    // two or more stages) or once its stage is consumed (one stage). Issuing one tile per CTA at
    // first, not the whole ring, halves the grid's opening burst, so the first tiles land sooner;
    // refilling on landing rather than on consumption measured 0.6-1.3 us faster per decode step.
    constexpr int kAhead = kStg > 1 ? kStg - 1 : 1;
    if (lane == 0) {
        for (int st = 0; st < kAhead && x0 + st < x1; ++st) {
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * kTileFloats, group_src(x0 + st), kTileBytes, &bar[st]);
        }
    }

    RunList rl;
    rl.init();
    int cur = -1;
    bool ok = true;
    // Finish unit u: write its answer (this CTA held all of it) or deposit this segment's top-k.
    auto finish = [&](int u) {
        const int cf = sel_cta_of((long long)u * nGc, n, grid);
        const int cl = sel_cta_of((long long)(u + 1) * nGc - 1, n, grid);
        if (cl == cf) {
            const int key = warp_sort_asc(lane < k ? rl.i : kInvalid, lane);
            if (lane < k) idx[(size_t)u * k + lane] = key == kInvalid ? -1 : key;
            return;
        }
        if (lane < k) {
            ws_s[((size_t)u * maxseg + (c - cf)) * k + lane] = rl.s;
            ws_i[((size_t)u * maxseg + (c - cf)) * k + lane] = rl.i;
        }
    };

    for (long long x = x0; x < x1; ++x) {
        const int it = (int)(x - x0);
        const int st = it % kStg;
        const uint32_t parity = (uint32_t)(it / kStg) & 1u;
        const int u = (int)(x / nGc), gl = (int)(x % nGc);
        if (u != cur) {
            if (cur >= 0) finish(cur);
            rl.init();
            cur = u;
            // group query of unit u (heads u*G .. u*G+G-1 of Q [B, Hq, d]): Qsum and Q2 of
            // channels lane + 32 j, every head's value loaded at once
            __syncwarp();
            // lane l: channels [l D/32, (l + 1) D/32), one vector load per head
            group_query_chunk<T, D / 32>(Q + (size_t)u * G * D, G, D, lane * (D / 32), true, &qsm[0][lane * (D / 32)],
                                         &qsm[1][lane * (D / 32)]);
            __syncwarp();
            if (ISO) {
                if (lane == 0) q2t_sm = q2_total<D>(qsm[1]);
                __syncwarp();
            }
            if (kProj) {  // the group's projected heads, after the ring
                float* qh = tiles + kStg * kTileFloats;
                if (x == x0) asm volatile("griddepcontrol.wait;" ::: "memory");  // qt_ws is complete
                for (int e = lane; e < G * S; e += 32) qh[e] = __ldcg(qt_ws + (size_t)u * G * S + e);
                __syncwarp();
            } else if (MODE >= 2) {  // the group's heads as float32, after the ring
                float* qh = tiles + kStg * kTileFloats;
                for (int e = lane; e < G * D; e += 32) qh[e] = to_f(Q[(size_t)u * G * D + e]);
                __syncwarp();
            }
        }
        if (ok) ok = mbar_wait(&bar[st], parity, err);
        ok = __all_sync(kFull, ok);
        // ring: tile x + kStg - 1 into the stage of tile x - 1, which every lane finished reading
        // before the __syncwarp that closed the previous iteration
        if (kStg > 1 && lane == 0 && ok && x + kStg - 1 < x1) {
            const int sn = (int)((x + kStg - 1 - x0) % kStg);
            fence_proxy_async();
            mbar_arrive_expect_tx(&bar[sn], kTileBytes);
            bulk_g2s(tiles + sn * kTileFloats, group_src(x + kStg - 1), kTileBytes, &bar[sn]);
        }
        const int b = gl * kGroupBlocks + lane;
        float sc = -INFINITY;
        int bi = kInvalid;
        if (ok) {
            const float* tl = tiles + st * kTileFloats;
            const float* qh = tiles + kStg * kTileFloats;
            const float s_all = MODE == 5   ? block_score_fp4<D, true>(tl, qsm[0], qh, G, R, S, lane, isd, c2)
                                : MODE == 4 ? block_score_sub<D>(tl, qsm[0], qh, G, R, S, lane, isd, c2)
                                : MODE == 3 ? block_score_fp4<D, false>(tl, qsm[0], qh, G, R, D, lane, isd, c2)
                                : MODE == 2 ? block_score_sub<D>(tl, qsm[0], qh, G, R, D, lane, isd, c2)
                                : ISO       ? block_score_iso<D>(tl, qsm[0], q2t_sm, lane, isd, c2)
                                            : block_score<D>(tl, qsm[0], qsm[1], lane, isd, c2);
            if (b < ncand) {
                sc = s_all;
                bi = b;
            }
        }
        __syncwarp();
        if (kStg == 1 && lane == 0 && ok && x + 1 < x1) {  // one stage: refilled once consumed
            fence_proxy_async();
            mbar_arrive_expect_tx(&bar[0], kTileBytes);
            bulk_g2s(tiles, group_src(x + 1), kTileBytes, &bar[0]);
        }
        rl.add(sc, bi, k, lane);
    }
    finish(cur);
}

// grid (units), 8 warps: merges the segment lists select_decode_kernel deposited for each unit
// cut into several ranges (a shared-memory tree of warp merges, log2(segments) levels) and
// writes the unit's answer in ascending block order. Launched as a programmatic dependent of
// the selection grid: it waits for that grid to complete before reading the deposits.
__global__ void __launch_bounds__(256) select_merge_kernel(const float* __restrict__ ws_s,
                                                           const int* __restrict__ ws_i, int32_t* __restrict__ idx,
                                                           int nGc, long long n, int grid, int k, int maxseg) {
    // a dependent grid (the decode step's attention) may be scheduled now; it waits for this grid
    // to complete before it reads idx
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float ls[kSelMaxSeg][32];
    __shared__ int li[kSelMaxSeg][32];
    const int u = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (n == 0) return;
    const int cf = sel_cta_of((long long)u * nGc, n, grid);
    const int cl = sel_cta_of((long long)(u + 1) * nGc - 1, n, grid);
    const int nseg = cl - cf + 1;
    if (nseg == 1) return;  // written by the selection grid
    for (int e = threadIdx.x; e < nseg * 32; e += blockDim.x) {
        const int j = e >> 5, p = e & 31;
        const bool in = p < k;
        ls[j][p] = in ? ws_s[((size_t)u * maxseg + j) * k + p] : -INFINITY;
        li[j][p] = in ? ws_i[((size_t)u * maxseg + j) * k + p] : kInvalid;
    }
    __syncthreads();
    for (int width = 1; width < nseg; width *= 2) {
        for (int pair = warp; pair * 2 * width < nseg; pair += 8) {
            const int x = pair * 2 * width, y = x + width;
            if (y < nseg) {
                float s1 = ls[x][lane];
                int i1 = li[x][lane];
                warp_merge_best_first(s1, i1, ls[y][lane], li[y][lane], lane);
                ls[x][lane] = s1;
                li[x][lane] = i1;
            }
        }
        __syncthreads();
    }
    if (warp == 0) {
        const int key = warp_sort_asc(lane < k ? li[0][lane] : kInvalid, lane);
        if (lane < k) idx[(size_t)u * k + lane] = key == kInvalid ? -1 : key;
    }
}

// ---------------------------------------------------------------------------- prefill
// grid (ceil(T / 32), B * Hkv); 4 warps x 8 positions = a tile of 32 consecutive positions.
// Candidates at position t are blocks b < (t+1)/L. Each warp keeps one top-k list per
// position (lanes = list slots) and scores 32 blocks per smem tile (lane = block).
constexpr int kPfPos = 32;
constexpr int kPfWarps = 4;
constexpr int kPfPerWarp = kPfPos / kPfWarps;

template <typename T, int D, bool ISO>
__global__ void __launch_bounds__(128) select_prefill_kernel(const T* __restrict__ Q, const float* __restrict__ summ,
                                                             int32_t* __restrict__ idx, int Tctx, int Hq, int Hkv,
                                                             int G, int nG, int L, int k, float isd, float c2,
                                                             int* err) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    constexpr int kTileFloats = group_floats<D, ISO>();
    float* tiles = reinterpret_cast<float*>(smem_raw);           // [2][kTileFloats]
    float* sq = tiles + 2 * kTileFloats;                           // [kPfPos][2][D]: Qsum, Q2
    __shared__ __align__(8) uint64_t bar[2];
    __shared__ float q2t[kPfPos];                                  // Q2tot per position (isotropic)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int unit = blockIdx.y;
    const int b = unit / Hkv, g = unit % Hkv;
    const int t0 = blockIdx.x * kPfPos;
    const int tlast = min(Tctx - 1, t0 + kPfPos - 1);
    const int ncand_max = (tlast + 1) / L;
    const int ngroups = (ncand_max + kGroupBlocks - 1) / kGroupBlocks;
    const float* usum = summ + (size_t)unit * nG * kTileFloats;
    constexpr uint32_t kTileBytes = kTileFloats * 4;

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int st = 0; st < 2 && st < ngroups; ++st) {
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * kTileFloats, usum + (size_t)st * kTileFloats, kTileBytes, &bar[st]);
        }
    }
    // group queries of the tile's positions: thread -> (position, 8-channel chunk), every head's
    // chunk loaded at once (16-byte loads for bf16)
    for (int e = tid; e < kPfPos * (D / 8); e += blockDim.x) {
        const int p = e / (D / 8), c0 = (e % (D / 8)) * 8;
        const int t = t0 + p;
        const T* qr = Q + (((size_t)b * Tctx + (t < Tctx ? t : 0)) * Hq + (size_t)g * G) * D;
        group_query_chunk<T, 8>(qr, G, D, c0, t < Tctx, &sq[(p * 2 + 0) * D + c0], &sq[(p * 2 + 1) * D + c0]);
    }
    __syncthreads();
    if (ISO) {
        if (tid < kPfPos) q2t[tid] = q2_total<D>(sq + (tid * 2 + 1) * D);
        __syncthreads();
    }

    TopK tk[kPfPerWarp];
#pragma unroll
    for (int j = 0; j < kPfPerWarp; ++j) tk[j].init();
    bool ok = true;
    for (int gi = 0; gi < ngroups; ++gi) {
        const int st = gi & 1;
        const uint32_t parity = (gi >> 1) & 1;
        if (ok) ok = mbar_wait(&bar[st], parity, err);
        ok = __syncthreads_and(ok) != 0;
        const float* tile = tiles + st * kTileFloats;
        const int blk = gi * kGroupBlocks + lane;
        // scores of this lane's block against the warp's 8 positions: 16 independent chains,
        // each in the canonical order (ascending channels, one fma per term)
        float av[kPfPerWarp][4], vv[kPfPerWarp][4];
#pragma unroll
        for (int j = 0; j < kPfPerWarp; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) av[j][q] = vv[j][q] = 0.0f;
        const float4* mu4 = reinterpret_cast<const float4*>(tile) + lane;
        const float4* var4 = reinterpret_cast<const float4*>(tile + D * 32) + lane;
        const float* sqw = sq + (size_t)(warp * kPfPerWarp) * 2 * D;
        if (ISO) {
#pragma unroll 4
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 m = mu4[c4 * 32];
#pragma unroll
                for (int j = 0; j < kPfPerWarp; ++j) {
                    const float4 qa = reinterpret_cast<const float4*>(sqw + (j * 2 + 0) * D)[c4];
                    av[j][0] = __fmaf_rn(qa.x, m.x, av[j][0]);
                    av[j][1] = __fmaf_rn(qa.y, m.y, av[j][1]);
                    av[j][2] = __fmaf_rn(qa.z, m.z, av[j][2]);
                    av[j][3] = __fmaf_rn(qa.w, m.w, av[j][3]);
                }
            }
        } else {
#pragma unroll 4
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 m = mu4[c4 * 32];
                const float4 vr = var4[c4 * 32];
#pragma unroll
                for (int j = 0; j < kPfPerWarp; ++j) {
                    const float4 qa = reinterpret_cast<const float4*>(sqw + (j * 2 + 0) * D)[c4];
                    const float4 qb = reinterpret_cast<const float4*>(sqw + (j * 2 + 1) * D)[c4];
                    av[j][0] = __fmaf_rn(qa.x, m.x, av[j][0]);
                    av[j][1] = __fmaf_rn(qa.y, m.y, av[j][1]);
                    av[j][2] = __fmaf_rn(qa.z, m.z, av[j][2]);
                    av[j][3] = __fmaf_rn(qa.w, m.w, av[j][3]);
                    vv[j][0] = __fmaf_rn(qb.x, vr.x, vv[j][0]);
                    vv[j][1] = __fmaf_rn(qb.y, vr.y, vv[j][1]);
                    vv[j][2] = __fmaf_rn(qb.z, vr.z, vv[j][2]);
                    vv[j][3] = __fmaf_rn(qb.w, vr.w, vv[j][3]);
                }
            }
        }
        float aj[kPfPerWarp], vj[kPfPerWarp];
        const float sig = ISO ? tile[D * 32 + lane] : 0.0f;
#pragma unroll
        for (int j = 0; j < kPfPerWarp; ++j) {
            aj[j] = combine4(av[j][0], av[j][1], av[j][2], av[j][3]);
            vj[j] = ISO ? __fmul_rn(q2t[warp * kPfPerWarp + j], sig) : combine4(vv[j][0], vv[j][1], vv[j][2], vv[j][3]);
        }
        __syncthreads();  // every warp is done with this stage
        if (tid == 0 && ok && gi + 2 < ngroups) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&bar[st], kTileBytes);
            bulk_g2s(tiles + st * kTileFloats, usum + (size_t)(gi + 2) * kTileFloats, kTileBytes, &bar[st]);
        }
#pragma unroll
        for (int j = 0; j < kPfPerWarp; ++j) {
            const int t = t0 + warp * kPfPerWarp + j;
            const int nc = (t + 1) / L;
            const bool valid = ok && t < Tctx && blk < nc;
            float sc = __fmaf_rn(c2, vj[j], __fmul_rn(aj[j], isd));
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

// The projected query heads of the query-subspace form: the 16-byte aligned region that follows
// the segment lists in the decode selection workspace.
float* select_qt_region(const Dims& m, void* ws) {
    const int nGc = (m.T / m.L + kGroupBlocks - 1) / kGroupBlocks;
    const int maxseg = sel_max_segments(m.units(), std::max(1, nGc));
    const size_t lists = (size_t)m.units() * maxseg * m.k * (sizeof(float) + sizeof(int));
    return reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + (lists + 15) / 16 * 16);
}

template <typename T, int D, int MODE>
cudaError_t launch_select_t(const Dims& m, const T* Q, const float* summ, int prefill, int32_t* idx, void* ws,
                            cudaStream_t s, int* err) {
    constexpr bool ISO = MODE == 1;
    float isd, c2;
    score_constants(m.d, m.alpha, &isd, &c2);
    const int tile_floats = (int)m.group_floats();
    const size_t tile_bytes = (size_t)tile_floats * 4;
    if (!prefill) {
        const int ncand = m.T / m.L;
        const int nGc = (ncand + kGroupBlocks - 1) / kGroupBlocks;
        const long long n = (long long)m.units() * nGc;
        const int maxseg = sel_max_segments(m.units(), std::max(1, nGc));
        const size_t smem = MODE == 2   ? tile_bytes + (size_t)kMaxGroup * D * 4
                            : MODE == 3 ? (size_t)kSelStages * tile_bytes + (size_t)kMaxGroup * D * 4
                            : MODE == 4 ? tile_bytes + (size_t)m.G * m.sub * 4
                            : MODE == 5 ? (size_t)kSelStages * tile_bytes + (size_t)m.G * m.sub * 4
                                        : (size_t)kSelStages * tile_bytes;
        if (smem > 227 * 1024) return cudaErrorNotSupported;
        cudaError_t e = cudaFuncSetAttribute(select_decode_kernel<T, D, MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_decode_kernel<T, D, MODE>, 32, smem);
        if (e != cudaSuccess) return e;
        per_sm = std::max(1, std::min(per_sm, (MODE == 3 || MODE == 5) ? 2 * kSelCtasPerSm : kSelCtasPerSm));
        // grid: the resident CTAs of every SM and at least one group each. A unit's groups then
        // meet at most min(nGc, ceil(grid / units) + 1) <= maxseg ranges (grid <= kSelGridCap).
        long long grid = std::min<long long>((long long)sm_count() * per_sm, kSelGridCap);
        grid = std::min<long long>(grid, std::max<long long>(1, n));
        grid = std::min<long long>(grid, (long long)(kSelMaxSeg - 1) * m.units());
        if (n == 0) grid = std::min(m.units(), 1024);
        grid = std::max<long long>(1, grid);
        float* ws_s = static_cast<float*>(ws);
        int* ws_i = reinterpret_cast<int*>(ws_s + (size_t)m.units() * maxseg * m.k);
        constexpr bool kProj = MODE == 4 || MODE == 5;
        float* qt_ws = kProj ? select_qt_region(m, ws) : nullptr;
        if (kProj && n > 0) {  // the projected heads, then the selection grid as their dependent
            count_launch();
            project_queries_kernel<T, D><<<dim3(m.units(), (m.G * m.sub + 63) / 64), 256, 0, s>>>(Q, m.basis, m.G,
                                                                                                   m.sub, qt_ws);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)grid);
            cfg.blockDim = dim3(32);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = s;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            count_launch();
            e = cudaLaunchKernelEx(&cfg, select_decode_kernel<T, D, MODE>, Q, summ, idx, ws_s, ws_i, m.units(), m.G,
                                   m.nG, ncand, m.k, maxseg, isd, c2, m.lr, tile_floats, (const float*)qt_ws, m.sub,
                                   err);
        } else {
            count_launch();
            select_decode_kernel<T, D, MODE><<<(unsigned)grid, 32, smem, s>>>(Q, summ, idx, ws_s, ws_i, m.units(),
                                                                              m.G, m.nG, ncand, m.k, maxseg, isd, c2,
                                                                              m.lr, tile_floats, qt_ws, m.sub, err);
            e = cudaGetLastError();
        }
        // a unit is cut into several ranges only if it has several groups and the grid several CTAs
        if (e != cudaSuccess || n == 0 || nGc == 1 || grid == 1) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(m.units());
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        count_launch();
        return cudaLaunchKernelEx(&cfg, select_merge_kernel, (const float*)ws_s, (const int*)ws_i, idx, nGc, n,
                                  (int)grid, m.k, maxseg);
    }
    const size_t smem = tile_bytes * 2 + (size_t)kPfPos * 2 * D * 4;
    if (MODE >= 2) return cudaErrorNotSupported;  // the API rejects it before this point
    auto kern = select_prefill_kernel<T, D, ISO>;
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
    const int nGc = (m.T / m.L + kGroupBlocks - 1) / kGroupBlocks;
    const int maxseg = sel_max_segments(m.units(), std::max(1, nGc));
    const size_t lists = (size_t)m.units() * maxseg * m.k * (sizeof(float) + sizeof(int));
    if (!m.sub) return lists;
    // query-subspace summaries: the projected heads [units][G][sub] float32 after the lists
    return (lists + 15) / 16 * 16 + (size_t)m.units() * m.G * m.sub * sizeof(float);
}

template <int MODE>
cudaError_t launch_select_v(const Dims& m, const void* Q, const float* summ, int prefill, int32_t* idx, void* ws,
                            cudaStream_t s, int* err) {
    if (m.dtype == COBS_BF16) {
        if (m.d == 128)
            return launch_select_t<__nv_bfloat16, 128, MODE>(m, (const __nv_bfloat16*)Q, summ, prefill, idx, ws, s,
                                                             err);
        return launch_select_t<__nv_bfloat16, 64, MODE>(m, (const __nv_bfloat16*)Q, summ, prefill, idx, ws, s, err);
    }
    if (m.d == 128) return launch_select_t<float, 128, MODE>(m, (const float*)Q, summ, prefill, idx, ws, s, err);
    return launch_select_t<float, 64, MODE>(m, (const float*)Q, summ, prefill, idx, ws, s, err);
}

cudaError_t launch_select(const Dims& m, const void* Q, const float* summ, int prefill, int32_t* idx, void* ws,
                          cudaStream_t s, int* err) {
    if (m.sub) return m.fp4 ? launch_select_v<5>(m, Q, summ, prefill, idx, ws, s, err)
                            : launch_select_v<4>(m, Q, summ, prefill, idx, ws, s, err);
    if (m.lr) return m.fp4 ? launch_select_v<3>(m, Q, summ, prefill, idx, ws, s, err)
                           : launch_select_v<2>(m, Q, summ, prefill, idx, ws, s, err);
    return m.iso ? launch_select_v<1>(m, Q, summ, prefill, idx, ws, s, err)
                 : launch_select_v<0>(m, Q, summ, prefill, idx, ws, s, err);
}

}  // namespace cobs
