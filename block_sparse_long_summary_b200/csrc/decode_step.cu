// Decode step, bf16: block selection and the three-branch decode attention in one persistent
// kernel, so that the summaries, the window, the compressed tokens and the selected blocks
// stream through HBM back to back instead of in three dependent launches.
//
// What is computed is exactly cobs_select (decode) followed by cobs_sparse_attn_decode:
// COBS (gist.science explainer §2.3) ranks the complete blocks by the second-order score and
// keeps the top-k per GQA group; the NSA paths (Janus issue #181: compression, selection,
// sliding window) are attended with softmaxes of their own and mixed by the gates. Decode is
// bound by the KV-cache read (explainer, "Problemstellung"), so the kernel is scheduled for HBM:
//
// * One CTA per SM, 4 warps, each warp an independent worker with a private 3-stage ring of
//   shared-memory tiles filled by bulk / TMA copies (no multicast).
// * The work is three phases, each cut into contiguous per-warp ranges (stream-K), and every
//   warp walks its ranges in phase order:
//     S  the summary groups of every unit (32 blocks; the mean half and the variance half of
//        a group are two tiles): canonical float32 scores and a warp top-k list;
//     A  the window and compressed-token tiles of every unit (they do not depend on S);
//     B  the tiles of the selected blocks of every unit.
//   The range of phase A is sized so that every warp streams the same number of tiles in all.
// * A unit's selection may be cut across warps: each deposits its segment list, and the last
//   to arrive (a per-unit counter) merges them, writes idx and publishes the unit with the
//   launch's epoch number. A phase-B tile of the unit waits for that flag (bounded) before it
//   reads idx; every warp finishes its own phase-S segments before it waits on any flag, and
//   phase S itself waits on nothing, so the waits cannot form a cycle.
// * An attention piece (the tiles of one (unit, branch) a warp covers) leaves a partial
//   record (m, l, o); the last piece of a (unit, branch) folds its records into the gated
//   branch output, and the last branch of a unit sums the branches into O. The counters are
//   re-armed by the warps that complete them, and the epoch advances when the last CTA ends.
#include <algorithm>

#include "common.cuh"
#include "dims.h"
#include "select_core.cuh"
#include "stream_tile.cuh"
#include "tma.h"

namespace cobs {
namespace {

constexpr int kStepWarps = 4;   // workers per CTA
constexpr int kStepStages = 3;  // ring depth per worker

struct StepArgs {
    const __nv_bfloat16* Q;
    const float* summ;
    const float* gates;
    int32_t* idx;
    __nv_bfloat16* O;
    int* err;
    // workspace (control words at the start)
    unsigned* ctl;       // [0] epoch of the last completed launch, [1] CTAs finished in this launch
    unsigned* ready;     // [units] epoch at which idx[u] was published
    unsigned* sel_cnt;   // [units] selection segments deposited
    unsigned* br_cnt;    // [units][3] attention pieces flushed, per branch
    unsigned* unit_cnt;  // [units] branches finalised
    float* seg_s;        // [units][maxseg][32] segment lists (scores, best first)
    int* seg_i;          // [units][maxseg][32] (block indices)
    float* rec;          // [units][3][maxw][G][D + 4] attention partial records
    float* bout;         // [units][3][G][D] gated branch outputs
    // shape
    int units, G, T, k, W, nB, nC, nG, nGc, ncand, iso, D;
    int tS, tW, tC, tA;  // tiles per unit: selected blocks, window, compressed tokens, tW + tC
    int tpg;             // ring tiles per summary group (2: means + variances, 1: isotropic)
    int gfloats;         // floats per stored summary group
    int nwarps;
    long long nS, nA, nBt, tot;  // phase sizes (groups, tiles, tiles) and tpg nS + nA + nBt
    int balanced;        // phase A sized so that every warp's total is equal
    int dense[3];        // phase S, A, B: every warp's range is nonempty (else at most one element each)
    int nbr;             // branches with tiles (selected blocks always; window, compressed tokens if any)
    int maxseg, maxw;
    float isd, c2, sl2;
    // reciprocals of the divisors of the partition arithmetic (exact quotients: see div_floor)
    double inv_nw, inv_nS, inv_nA, inv_nBt;
};

// floor(x / n) for 0 <= x < 2^50 and 1 <= n < 2^40 without an integer division: the double
// quotient estimate x * (1/n) is within 1 of the true quotient, and one integer remainder check
// corrects it. (64-bit integer division is a long dependent instruction sequence on the GPU.)
__host__ __device__ __forceinline__ long long div_floor(long long x, long long n, double inv) {
    long long q = (long long)((double)x * inv);
    long long r = x - q * n;
    if (r < 0) { --q; r += n; }
    if (r >= n) ++q;
    return q;
}

// Per-warp ranges of the three phases: warp v takes [f(v), f(v + 1)) of each.
__host__ __device__ __forceinline__ long long fS(const StepArgs& a, long long v) {
    return div_floor(v * a.nS, a.nwarps, a.inv_nw);
}
__host__ __device__ __forceinline__ long long fB(const StepArgs& a, long long v) {
    return div_floor(v * a.nBt, a.nwarps, a.inv_nw);
}
__host__ __device__ __forceinline__ long long fA(const StepArgs& a, long long v) {
    if (!a.balanced) return div_floor(v * a.nA, a.nwarps, a.inv_nw);
    return div_floor(v * a.tot, a.nwarps, a.inv_nw) - a.tpg * fS(a, v) - fB(a, v);
}
// The largest v with floor(v n / N) <= x: v = ceil((x + 1) N / n) - 1 (at most N - 1).
__host__ __device__ __forceinline__ int floor_part_inverse(long long x, long long n, double inv_n, int N) {
    const long long v = div_floor((x + 1) * N + n - 1, n, inv_n) - 1;
    return (int)(v < N - 1 ? v : N - 1);
}
// The warp whose range of phase PH holds element x (the largest v with f(v) <= x). The floor
// partitions invert in closed form; the balanced phase-A starts differ from v nA / N by less
// than tpg + 2, so the closed-form inverse of that floor partition is a few steps from the answer.
template <int PH>
__host__ __device__ __forceinline__ int warp_of(const StepArgs& a, long long x) {
    if (PH == 0) return floor_part_inverse(x, a.nS, a.inv_nS, a.nwarps);
    if (PH == 2) return floor_part_inverse(x, a.nBt, a.inv_nBt, a.nwarps);
    int v = floor_part_inverse(x, a.nA, a.inv_nA, a.nwarps);
    if (!a.balanced) return v;
    while (v > 0 && fA(a, v) > x) --v;
    while (v < a.nwarps - 1 && fA(a, v + 1) <= x) ++v;
    return v;
}

// A piece is the part of a run [x0, x0 + len) of one phase (a unit's summary groups, or the
// tiles of one (unit, branch)) that one warp covers. Number of pieces of the run: the warps whose
// ranges meet it. In a dense phase every warp's range is nonempty; otherwise (a floor partition
// of fewer elements than warps) every range holds at most one element.
template <int PH>
__host__ __device__ __forceinline__ int run_pieces(const StepArgs& a, long long x0, long long len) {
    if (len <= 0) return 0;
    if (!a.dense[PH]) return (int)len;
    return warp_of<PH>(a, x0 + len - 1) - warp_of<PH>(a, x0) + 1;
}
// Slot (0 .. pieces - 1) of the piece of warp v, whose range of the phase starts at r0.
template <int PH>
__host__ __device__ __forceinline__ int run_slot(const StepArgs& a, int v, long long r0, long long x0) {
    return a.dense[PH] ? v - warp_of<PH>(a, x0) : (int)((r0 > x0 ? r0 : x0) - x0);
}
// Run of unit u's branch br (0 selected blocks: phase B; 1 window, 2 compressed tokens: phase A).
__host__ __device__ __forceinline__ void branch_run(const StepArgs& a, int u, int br, long long* x0, long long* len) {
    if (br == 0) { *x0 = (long long)u * a.tS; *len = a.tS; }
    else if (br == 1) { *x0 = (long long)u * a.tA; *len = a.tW; }
    else { *x0 = (long long)u * a.tA + a.tW; *len = a.tC; }
}
__host__ __device__ __forceinline__ int branch_pieces(const StepArgs& a, int u, int br) {
    long long x0, len;
    branch_run(a, u, br, &x0, &len);
    return br == 0 ? run_pieces<2>(a, x0, len) : run_pieces<1>(a, x0, len);
}
__host__ __device__ __forceinline__ int sel_segments(const StepArgs& a, int u) {
    return run_pieces<0>(a, (long long)u * a.nGc, a.nGc);
}

struct Item {
    int kind;       // 0 summary means (or isotropic tile), 1 summary variances, 2 attention tile
    int unit;
    int a;          // summary group (kinds 0, 1) or branch (kind 2)
    int row;        // attention: first row of K / V (branches 0, 1) or Kc / Vc (branch 2)
    unsigned mask;  // attention: valid keys of the tile (0: nothing to load)
};

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ int ld_relaxed(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait for a published flag (one thread). False (and kErrWaitTimeout recorded) if it
// did not arrive within kWaitLimitNs.
__device__ __forceinline__ bool wait_flag(const unsigned* f, unsigned want, int* err) {
    if (ld_acquire(f) == want) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kMaxWaitIters; ++i) {
        __nanosleep(128);
        if (ld_acquire(f) == want) return true;
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
    report_error(err, kErrWaitTimeout);
    return false;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}

// Selection segment of unit u held by warp v (list rl): write idx directly when the warp held the
// whole unit; else deposit it, and if it is the last to arrive, merge all segments of the unit
// and write idx. Either way the writer publishes the unit with the epoch.
__device__ void sel_finish(const StepArgs& a, int v, long long r0, int u, const RunList& rl, unsigned ep,
                           int lane) {
    const int nseg = sel_segments(a, u);
    float s = rl.s;
    int i = rl.i;
    if (nseg > 1) {
        const int slot = run_slot<0>(a, v, r0, (long long)u * a.nGc);
        const size_t base = ((size_t)u * a.maxseg + slot) * 32;
        a.seg_s[base + lane] = s;
        a.seg_i[base + lane] = i;
        __threadfence();
        __syncwarp();
        unsigned old = 0;
        if (lane == 0) old = atomicAdd(&a.sel_cnt[u], 1u);
        old = __shfl_sync(kFull, old, 0);
        if (old != (unsigned)(nseg - 1)) return;
        __threadfence();
        // the other segments, 16 at a time; a segment whose best entry does not beat the current
        // k-th best cannot contribute and costs one comparison
        float ts = __shfl_sync(kFull, s, a.k - 1);
        int ti = __shfl_sync(kFull, i, a.k - 1);
        for (int j0 = 0; j0 < nseg; j0 += 16) {
            float bs[16];
            int bi[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int j = j0 + q;
                bs[q] = -INFINITY;
                bi[q] = kInvalid;
                if (j < nseg && j != slot) {
                    const size_t o = ((size_t)u * a.maxseg + j) * 32 + lane;
                    bs[q] = __ldcg(a.seg_s + o);
                    bi[q] = __ldcg(a.seg_i + o);
                }
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float b0s = __shfl_sync(kFull, bs[q], 0);
                const int b0i = __shfl_sync(kFull, bi[q], 0);
                if (b0i == kInvalid || !better(b0s, b0i, ts, ti)) continue;  // uniform
                warp_merge_best_first(s, i, bs[q], bi[q], lane);
                ts = __shfl_sync(kFull, s, a.k - 1);
                ti = __shfl_sync(kFull, i, a.k - 1);
            }
        }
        if (lane == 0) a.sel_cnt[u] = 0u;  // re-armed for the next launch
    }
    const int key = warp_sort_asc(lane < a.k ? i : kInvalid, lane);
    if (lane < a.k) a.idx[(size_t)u * a.k + lane] = key == kInvalid ? -1 : key;
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release(&a.ready[u], ep);
}

// Fold the records of unit u's branch br into the gated branch output bout[u][br] (all heads):
// o_h = g_{h,br} * (sum_j 2^(m_j - M) o_j) / (sum_j 2^(m_j - M) l_j), zero for an empty branch.
// Heads in fours; lane = D/32 consecutive channels; pieces 32 at a time (lane = piece for the
// maxima and sums), the running maximum rescaled between chunks.
template <int D>
__device__ void finalize_branch(const StepArgs& a, int u, int br, int np, int lane) {
    constexpr int CPL = D / 32;  // channels per lane
    constexpr int RF = D + 4;
    const size_t rs = (size_t)a.G * RF;  // floats per record slot
    const float* base = a.rec + ((size_t)u * 3 + br) * a.maxw * rs;
    const int gate_col = br == 0 ? 1 : (br == 1 ? 2 : 0);  // gates are (cmp, slc, win)
    for (int h0 = 0; h0 < a.G; h0 += 4) {
        float M[4], Ls[4], acc[4][CPL];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            M[q] = -INFINITY;
            Ls[q] = 0.0f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[q][c] = 0.0f;
        }
        for (int c0 = 0; c0 < np; c0 += 32) {
            const int nj = min(32, np - c0);
            float mj[4], lj[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                mj[q] = -INFINITY;
                lj[q] = 0.0f;
                if (lane < nj && h0 + q < a.G) {
                    const float* r = base + (size_t)(c0 + lane) * rs + (size_t)(h0 + q) * RF;
                    mj[q] = __ldcg(r);
                    lj[q] = __ldcg(r + 1);
                }
            }
            float fj[4], sc[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float nM = fmaxf(M[q], warp_max(mj[q]));
                sc[q] = (M[q] == -INFINITY || nM == -INFINITY) ? 0.0f : exp2f(M[q] - nM);
                fj[q] = (mj[q] == -INFINITY) ? 0.0f : exp2f(mj[q] - nM);
                Ls[q] = Ls[q] * sc[q] + warp_sum(lj[q] * fj[q]);
                M[q] = nM;
#pragma unroll
                for (int c = 0; c < CPL; ++c) acc[q][c] *= sc[q];
            }
#pragma unroll 4
            for (int j = 0; j < nj; ++j) {
                const float* r = base + (size_t)(c0 + j) * rs + 4 + lane * CPL;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float f = __shfl_sync(kFull, fj[q], j);
                    if (h0 + q < a.G) {
                        float o[CPL];
                        if constexpr (CPL == 4) {
                            const float4 t = __ldcg(reinterpret_cast<const float4*>(r + (size_t)(h0 + q) * RF));
                            o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
                        } else {
                            const float2 t = __ldcg(reinterpret_cast<const float2*>(r + (size_t)(h0 + q) * RF));
                            o[0] = t.x; o[1] = t.y;
                        }
#pragma unroll
                        for (int c = 0; c < CPL; ++c) acc[q][c] = fmaf(f, o[c], acc[q][c]);
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int h = h0 + q;
            if (h >= a.G) break;
            const float g = a.gates[((size_t)u * a.G + h) * 3 + gate_col];
            const float w = Ls[q] > 0.0f ? g / Ls[q] : 0.0f;
            float* out = a.bout + (((size_t)u * 3 + br) * a.G + h) * D + lane * CPL;
#pragma unroll
            for (int c = 0; c < CPL; ++c) out[c] = acc[q][c] * w;
        }
    }
}

// Sum the finalised branch outputs of unit u into O (bf16).
template <int D>
__device__ void finalize_unit(const StepArgs& a, int u, int lane) {
    constexpr int CPL = D / 32;
    for (int h = 0; h < a.G; ++h) {
        float s[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) s[c] = 0.0f;
#pragma unroll
        for (int br = 0; br < 3; ++br) {
            if ((br == 1 && a.tW == 0) || (br == 2 && a.tC == 0)) continue;  // branches without tiles
            const float* src = a.bout + (((size_t)u * 3 + br) * a.G + h) * D + lane * CPL;
#pragma unroll
            for (int c = 0; c < CPL; ++c) s[c] += __ldcg(src + c);
        }
        __nv_bfloat16* o = a.O + ((size_t)u * a.G + h) * D + lane * CPL;
#pragma unroll
        for (int c = 0; c < CPL; c += 2) *reinterpret_cast<__nv_bfloat162*>(o + c) = __floats2bfloat162_rn(s[c], s[c + 1]);
    }
}

// Partial record of warp v's piece of (unit u, branch br); the last piece of the branch
// finalises it, and the last branch of the unit writes O.
template <int D>
__device__ void att_flush(const StepArgs& a, int v, long long rstart, int u, int br, WState<D>& st, int lane) {
    constexpr int RF = D + 4;
    float l0 = st.l0, l1 = st.l1;
    l0 += __shfl_xor_sync(kFull, l0, 1);
    l0 += __shfl_xor_sync(kFull, l0, 2);
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);
    long long x0, len;
    branch_run(a, u, br, &x0, &len);
    const int np = br == 0 ? run_pieces<2>(a, x0, len) : run_pieces<1>(a, x0, len);
    const int slot = br == 0 ? run_slot<2>(a, v, rstart, x0) : run_slot<1>(a, v, rstart, x0);
    float* rec = a.rec + (((size_t)u * 3 + br) * a.maxw + (size_t)slot) * a.G * RF;
    const int r0 = lane >> 2, r1 = r0 + 8, c = 2 * (lane & 3);
    if ((lane & 3) == 0) {
        if (r0 < a.G) {
            rec[r0 * RF + 0] = st.m0;
            rec[r0 * RF + 1] = l0;
        }
        if (r1 < a.G) {
            rec[r1 * RF + 0] = st.m1;
            rec[r1 * RF + 1] = l1;
        }
    }
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        if (r0 < a.G) *reinterpret_cast<float2*>(rec + r0 * RF + 4 + nd * 8 + c) = make_float2(st.o[nd][0], st.o[nd][1]);
        if (r1 < a.G) *reinterpret_cast<float2*>(rec + r1 * RF + 4 + nd * 8 + c) = make_float2(st.o[nd][2], st.o[nd][3]);
    }
    __threadfence();
    __syncwarp();
    unsigned old = 0;
    if (lane == 0) old = atomicAdd(&a.br_cnt[(size_t)u * 3 + br], 1u);
    old = __shfl_sync(kFull, old, 0);
    if (old != (unsigned)(np - 1)) return;
    __threadfence();
    finalize_branch<D>(a, u, br, np, lane);
    if (lane == 0) a.br_cnt[(size_t)u * 3 + br] = 0u;
    __threadfence();
    __syncwarp();
    if (lane == 0) old = atomicAdd(&a.unit_cnt[u], 1u);
    old = __shfl_sync(kFull, old, 0);
    if (old != (unsigned)(a.nbr - 1)) return;
    __threadfence();
    finalize_unit<D>(a, u, lane);
    if (lane == 0) a.unit_cnt[u] = 0u;
}

template <int D>
__global__ void __launch_bounds__(kStepWarps * 32, 1) decode_step_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                          const __grid_constant__ CUtensorMap tmV,
                                                                          const __grid_constant__ CUtensorMap tmKc,
                                                                          const __grid_constant__ CUtensorMap tmVc,
                                                                          StepArgs a) {
    constexpr int kBox = kTK * 128;        // one 64-column box of a 32-row tile
    constexpr int kMat = (D / 64) * kBox;  // K or V part of an attention tile
    constexpr int kStage = 2 * kMat;       // = D * 128 bytes = one half of a summary group
    static_assert(kStage == D * 32 * 4, "an attention tile and a summary half-group fill one stage");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[kStepWarps][kStepStages];
    __shared__ __align__(16) float qsm[kStepWarps][2][D];         // group query: Qsum, Q2
    __shared__ __align__(16) float iso_sm[kStepWarps][kStepStages][32];
    __shared__ float q2t_sm[kStepWarps];
    __shared__ Item desc[kStepWarps][kStepStages];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* ring = base + (size_t)warp * kStepStages * kStage;
    uint64_t* bar = bars[warp];
    const int v = blockIdx.x * kStepWarps + warp;
    const unsigned ep = *reinterpret_cast<volatile unsigned*>(a.ctl) + 1u;

    // this warp's ranges
    const long long s0 = fS(a, v), s1 = fS(a, v + 1);
    const long long a0 = fA(a, v), a1 = fA(a, v + 1);
    const long long b0 = fB(a, v), b1 = fB(a, v + 1);
    const int nSi = (int)(s1 - s0) * a.tpg, nAi = (int)(a1 - a0), nBi = (int)(b1 - b0);
    const int n = nSi + nAi + nBi;

    if (lane == 0) {
        for (int s = 0; s < kStepStages; ++s) mbar_init(&bar[s], 1);
        fence_barrier_init();
    }
    // no complete block: every list is empty (written by the first warps)
    if (a.nGc == 0)
        for (int u = v; u < a.units; u += a.nwarps) {
            if (lane < a.k) a.idx[(size_t)u * a.k + lane] = -1;
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release(&a.ready[u], ep);
        }
    __syncwarp();

    const int t = a.T - 1;
    int ready_u = -1;
    // descriptor of this warp's item i (uniform across the warp)
    auto item_at = [&](int i) {
        Item it;
        it.row = 0;
        it.mask = 0u;
        if (i < nSi) {
            const int x = (int)s0 + (a.tpg == 2 ? i >> 1 : i);
            it.kind = a.tpg == 2 ? i & 1 : 0;
            it.unit = x / a.nGc;
            it.a = x - it.unit * a.nGc;
            it.mask = 1u;
        } else if (i < nSi + nAi) {
            const int y = (int)a0 + (i - nSi);
            it.kind = 2;
            it.unit = y / a.tA;
            const int l = y - it.unit * a.tA;
            if (l < a.tW) {
                it.a = 1;
                const int r0 = max(0, t - a.W + 1) + l * kTK;
                it.row = it.unit * a.T + r0;
                const int nk = min(kTK, t + 1 - r0);
                it.mask = nk >= 32 ? kFull : ((1u << nk) - 1u);
            } else {
                it.a = 2;
                const int c0 = (l - a.tW) * kTK;
                it.row = it.unit * a.nC + c0;
                const int nk = min(kTK, a.nC - c0);
                it.mask = nk >= 32 ? kFull : ((1u << nk) - 1u);
            }
        } else {
            const int z = (int)b0 + (i - nSi - nAi);
            it.kind = 2;
            it.a = 0;
            it.unit = z / a.tS;
            const int l = z - it.unit * a.tS;
            int bi = -1;
            if (lane == 0) {
                if (it.unit != ready_u) wait_flag(&a.ready[it.unit], ep, a.err);  // gives up after a bound
                bi = ld_relaxed(a.idx + (size_t)it.unit * a.k + l / (64 / kTK));
            }
            ready_u = it.unit;
            bi = __shfl_sync(kFull, bi, 0);
            if (bi >= 0) {
                if (bi >= a.nB) {
                    if (lane == 0) report_error(a.err, kErrBadIndex);
                } else {
                    it.row = it.unit * a.T + bi * 64 + (l % (64 / kTK)) * kTK;
                    it.mask = kTK == 32 ? kFull : 0xFFFFu;
                }
            }
        }
        return it;
    };
    uint32_t phase = 0;    // bit s: parity of the next completion of stage s
    bool ok = true;        // false after a timed-out wait (uniform across the warp)
    uint32_t pending = 0;  // stages with a copy in flight (lane 0's view)
    auto issue = [&](const Item& it, int s) {  // lane 0 only
        unsigned char* dst = ring + (size_t)s * kStage;
        if (it.kind < 2 || it.mask != 0u) pending |= 1u << s;
        if (it.kind < 2) {
            const float* g = a.summ + ((size_t)it.unit * a.nG + it.a) * a.gfloats;
            if (it.kind == 0) {
                mbar_arrive_expect_tx(&bar[s], kStage + (a.iso ? 128u : 0u));
                bulk_g2s(dst, g, kStage, &bar[s]);
                if (a.iso) bulk_g2s(iso_sm[warp][s], g + D * 32, 128, &bar[s]);
            } else {
                mbar_arrive_expect_tx(&bar[s], kStage);
                bulk_g2s(dst, g + D * 32, kStage, &bar[s]);
            }
            return;
        }
        if (it.mask == 0u) return;
        const CUtensorMap* mk = it.a == 2 ? &tmKc : &tmK;
        const CUtensorMap* mv = it.a == 2 ? &tmVc : &tmV;
        mbar_arrive_expect_tx(&bar[s], kStage);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
            tma_load_2d(dst + h * kBox, mk, h * 64, it.row, &bar[s]);
            tma_load_2d(dst + kMat + h * kBox, mv, h * 64, it.row, &bar[s]);
        }
    };

    int next_issue = 0;
    bool sel_flushed = nSi == 0;
    // issue every item whose stage is free; a phase-B item only once this warp's own selection
    // segments are deposited (its descriptor may wait on a unit that one of them completes)
    auto issue_ahead = [&](int consumed) {
        while (next_issue < n && next_issue < consumed + kStepStages &&
               (next_issue < nSi + nAi || sel_flushed)) {
            const Item it = item_at(next_issue);
            const int s = next_issue % kStepStages;
            if (lane == 0) {
                desc[warp][s] = it;
                fence_proxy_async();
                if (ok) issue(it, s);  // after a timed-out wait nothing more is loaded
            }
            ++next_issue;
        }
        __syncwarp();
    };

    RunList rl;
    rl.init();
    int sel_u = -1;
    float apart = 0.0f;
    WState<D> st;
    st.init();
    uint32_t qa[D / 16][4];
    int att_u = -1, att_br = -1, q_u = -1;

    issue_ahead(0);
    for (int i = 0; i < n; ++i) {
        issue_ahead(i);
        const int s = i % kStepStages;
        const Item it = desc[warp][s];
        const unsigned char* stage = ring + (size_t)s * kStage;
        if (it.kind < 2) {
            if (it.unit != sel_u) {
                if (sel_u >= 0) sel_finish(a, v, s0, sel_u, rl, ep, lane);
                __syncwarp();  // every lane is done with the previous unit's group query
                rl.init();
                sel_u = it.unit;
                // group query of the unit: lane l forms channels [l D/32, (l + 1) D/32)
                group_query_chunk<__nv_bfloat16, D / 32>(a.Q + (size_t)sel_u * a.G * D, a.G, D, lane * (D / 32), true,
                                                         &qsm[warp][0][lane * (D / 32)],
                                                         &qsm[warp][1][lane * (D / 32)]);
                __syncwarp();
                if (a.iso) {
                    if (lane == 0) q2t_sm[warp] = q2_total<D>(qsm[warp][1]);
                    __syncwarp();
                }
            }
            if (ok) ok = mbar_wait(&bar[s], (phase >> s) & 1u, a.err);
            ok = __all_sync(kFull, ok);
            if (ok) pending &= ~(1u << s);
            phase ^= 1u << s;
            const float* tile = reinterpret_cast<const float*>(stage);
            const int b = it.a * 32 + lane;
            bool done_group = false;
            float sc = -INFINITY;
            if (it.kind == 0) {
                apart = ok ? score_mean_part<D>(tile, qsm[warp][0], lane) : 0.0f;
                if (a.iso) {
                    sc = score_combine(apart, __fmul_rn(q2t_sm[warp], iso_sm[warp][s][lane]), a.isd, a.c2);
                    done_group = true;
                }
            } else {
                const float vpart = ok ? score_var_part<D>(tile, qsm[warp][1], lane) : 0.0f;
                sc = score_combine(apart, vpart, a.isd, a.c2);
                done_group = true;
            }
            if (done_group) {
                const bool valid = ok && b < a.ncand;
                rl.add(valid ? sc : -INFINITY, valid ? b : kInvalid, a.k, lane);
            }
            if (i == nSi - 1) {  // the last summary tile of this warp: deposit / publish now
                __syncwarp();
                sel_finish(a, v, s0, sel_u, rl, ep, lane);
                sel_u = -1;
                sel_flushed = true;
            }
        } else {
            if (it.unit != att_u || it.a != att_br) {
                if (att_u >= 0) att_flush<D>(a, v, att_br == 0 ? b0 : a0, att_u, att_br, st, lane);
                st.init();
                att_u = it.unit;
                att_br = it.a;
                if (att_u != q_u) {
                    load_q<D>(a.Q + (size_t)att_u * a.G * D, a.G, qa, lane);
                    q_u = att_u;
                }
            }
            if (it.mask != 0u) {
                if (ok) ok = mbar_wait(&bar[s], (phase >> s) & 1u, a.err);
                ok = __all_sync(kFull, ok);
                if (ok) pending &= ~(1u << s);
                phase ^= 1u << s;
                if (ok) tile_mma<D>(st, qa, stage, stage + kMat, it.mask, a.sl2, lane);
            }
        }
        __syncwarp();
    }
    if (att_u >= 0) att_flush<D>(a, v, att_br == 0 ? b0 : a0, att_u, att_br, st, lane);
    // after a timed-out wait: let the copies still in flight land (bounded) before the CTA exits
    if (lane == 0 && !ok)
        for (int s = 0; s < kStepStages; ++s)
            if ((pending >> s) & 1u) mbar_wait(&bar[s], (phase >> s) & 1u, nullptr);

    // the last CTA to finish advances the epoch (the next launch on the stream reads it)
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned old = atomicAdd(&a.ctl[1], 1u);
        if (old == gridDim.x - 1) {
            a.ctl[1] = 0u;
            __threadfence();
            a.ctl[0] = ep;
        }
    }
}

// Workspace layout: control words, then the counters, segment lists, records and branch outputs
// (each region 256-byte aligned).
struct StepLayout {
    size_t ctl, ready, sel_cnt, br_cnt, unit_cnt, seg_s, seg_i, rec, bout, total;
};

inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }

StepLayout step_layout(const StepArgs& a) {
    StepLayout L;
    size_t o = 0;
    L.ctl = o; o = al256(o + 2 * sizeof(unsigned));
    L.ready = o; o = al256(o + (size_t)a.units * sizeof(unsigned));
    L.sel_cnt = o; o = al256(o + (size_t)a.units * sizeof(unsigned));
    L.br_cnt = o; o = al256(o + (size_t)a.units * 3 * sizeof(unsigned));
    L.unit_cnt = o; o = al256(o + (size_t)a.units * sizeof(unsigned));
    L.seg_s = o; o = al256(o + (size_t)a.units * a.maxseg * 32 * sizeof(float));
    L.seg_i = o; o = al256(o + (size_t)a.units * a.maxseg * 32 * sizeof(int));
    L.rec = o; o = al256(o + (size_t)a.units * 3 * a.maxw * a.G * (a.D + 4) * sizeof(float));
    L.bout = o; o = al256(o + (size_t)a.units * 3 * a.G * a.D * sizeof(float));
    L.total = o;
    return L;
}

StepArgs make_step_args(const Dims& m) {
    StepArgs a{};
    a.units = m.units(); a.G = m.G; a.T = m.T; a.k = m.k; a.W = m.W; a.nB = m.nB; a.nC = m.nC; a.nG = m.nG;
    a.D = m.d;
    a.ncand = m.nB;  // decode at T - 1: every complete block is a candidate
    a.nGc = (a.ncand + 31) / 32;
    a.iso = m.iso;
    a.tpg = m.iso ? 1 : 2;
    a.gfloats = (int)m.group_floats();
    a.tS = m.k * (64 / kTK);
    a.tW = (std::min(m.W, m.T) + kTK - 1) / kTK;
    a.tC = (m.nC + kTK - 1) / kTK;
    a.tA = a.tW + a.tC;
    a.nwarps = sm_count() * kStepWarps;
    a.nS = (long long)a.units * a.nGc;
    a.nA = (long long)a.units * a.tA;
    a.nBt = (long long)a.units * a.tS;
    a.tot = a.tpg * a.nS + a.nA + a.nBt;
    a.nbr = 1 + (a.tW > 0) + (a.tC > 0);
    a.inv_nw = 1.0 / a.nwarps;
    a.inv_nS = a.nS > 0 ? 1.0 / (double)a.nS : 0.0;
    a.inv_nA = a.nA > 0 ? 1.0 / (double)a.nA : 0.0;
    a.inv_nBt = a.nBt > 0 ? 1.0 / (double)a.nBt : 0.0;
    // balanced phase-A ranges when every warp's is nonempty (strictly increasing starts)
    a.balanced = 1;
    for (long long v = 0; v < a.nwarps; ++v)
        if (fA(a, v + 1) <= fA(a, v)) { a.balanced = 0; break; }
    a.dense[0] = a.nS >= a.nwarps;
    a.dense[1] = a.balanced || a.nA >= a.nwarps;
    a.dense[2] = a.nBt >= a.nwarps;
    // workspace slots: the most pieces any unit's selection or (unit, branch) is cut into
    a.maxseg = 1;
    a.maxw = 1;
    for (int u = 0; u < a.units; ++u) {
        if (a.nGc > 0) a.maxseg = std::max(a.maxseg, sel_segments(a, u));
        for (int br = 0; br < 3; ++br) a.maxw = std::max(a.maxw, branch_pieces(a, u, br));
    }
    float isd, c2;
    score_constants(m.d, m.alpha, &isd, &c2);
    a.isd = isd;
    a.c2 = c2;
    a.sl2 = 1.4426950408889634f / sqrtf((float)m.d);
    return a;
}

template <int D>
size_t step_smem() { return (size_t)kStepWarps * kStepStages * D * 128 + 1024; }

template <int D>
cudaError_t launch_step_d(const Dims& m, StepArgs a, const void* K, const void* V, const void* Kc, const void* Vc,
                          cudaStream_t s) {
    CUtensorMap tk, tv, tkc, tvc;
    const uint64_t kvrows = (uint64_t)m.units() * m.T;
    const uint64_t crows = m.nC > 0 ? (uint64_t)m.units() * m.nC : kvrows;
    if (!encode_tmap_bf16_2d(&tk, K, kvrows, D, kTK) || !encode_tmap_bf16_2d(&tv, V, kvrows, D, kTK) ||
        !encode_tmap_bf16_2d(&tkc, m.nC > 0 ? Kc : K, crows, D, kTK) ||
        !encode_tmap_bf16_2d(&tvc, m.nC > 0 ? Vc : V, crows, D, kTK))
        return cudaErrorInvalidValue;
    const size_t smem = step_smem<D>();
    cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_step_kernel<D>, kStepWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorNotSupported;
    count_launch();
    decode_step_kernel<D><<<a.nwarps / kStepWarps, kStepWarps * 32, smem, s>>>(tk, tv, tkc, tvc, a);
    return cudaGetLastError();
}

}  // namespace

bool decode_step_supported(const Dims& m) {
    return m.dtype == COBS_BF16 && !m.lr && (m.d == 128 || m.d == 64) && m.L == 64;
}

size_t decode_step_workspace_bytes(const Dims& m) {
    if (!decode_step_supported(m)) return 0;
    return step_layout(make_step_args(m)).total;
}

cudaError_t launch_decode_step(const Dims& m, const void* Q, const float* summ, const void* K, const void* V,
                               const void* Kc, const void* Vc, int32_t* idx, const float* gates, void* O, void* ws,
                               cudaStream_t s, int* err) {
    StepArgs a = make_step_args(m);
    const StepLayout L = step_layout(a);
    unsigned char* w = static_cast<unsigned char*>(ws);
    a.Q = static_cast<const __nv_bfloat16*>(Q);
    a.summ = summ;
    a.gates = gates;
    a.idx = idx;
    a.O = static_cast<__nv_bfloat16*>(O);
    a.err = err;
    a.ctl = reinterpret_cast<unsigned*>(w + L.ctl);
    a.ready = reinterpret_cast<unsigned*>(w + L.ready);
    a.sel_cnt = reinterpret_cast<unsigned*>(w + L.sel_cnt);
    a.br_cnt = reinterpret_cast<unsigned*>(w + L.br_cnt);
    a.unit_cnt = reinterpret_cast<unsigned*>(w + L.unit_cnt);
    a.seg_s = reinterpret_cast<float*>(w + L.seg_s);
    a.seg_i = reinterpret_cast<int*>(w + L.seg_i);
    a.rec = reinterpret_cast<float*>(w + L.rec);
    a.bout = reinterpret_cast<float*>(w + L.bout);
    return m.d == 128 ? launch_step_d<128>(m, a, K, V, Kc, Vc, s) : launch_step_d<64>(m, a, K, V, Kc, Vc, s);
}

}  // namespace cobs
