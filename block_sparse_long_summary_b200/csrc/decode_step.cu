// Decode step, bf16: block selection and the three-branch decode attention in one persistent
// kernel, so that the summaries, the window, the compressed tokens and the selected blocks
// stream through HBM back to back instead of in dependent launches.
//
// What is computed is exactly cobs_select (decode) followed by cobs_sparse_attn_decode:
// COBS (gist.science explainer §2.3) ranks the complete blocks by the second-order score and
// keeps the top-k per GQA group; the NSA paths (Janus issue #181: compression, selection,
// sliding window) are attended with softmaxes of their own and mixed by the gates. Decode is
// bound by the KV-cache read (explainer, "Problemstellung"), so the kernel is scheduled for HBM,
// and nothing on a streaming warp's path waits for a global-memory round trip (under a
// saturated HBM each one costs microseconds):
//
// * One CTA per SM: 4 streaming warps (one per scheduler) and 1 helper warp. Every streaming
//   warp has a private 3-stage ring of 16 KiB shared-memory tiles (d = 128) filled by bulk / TMA
//   copies (no multicast). An attention tile is 32 keys of K and V; a summary group (32 blocks)
//   is two tiles: its means and its variances. (Each warp's path is latency-bound: larger tiles
//   cost fewer per-tile steps per byte, which measured faster than more warps with 16-key tiles.)
// * The work is three phases, each cut into contiguous per-warp ranges (stream-K), and every
//   streaming warp walks its ranges in phase order:
//     S  the summary groups of every unit: canonical float32 scores (the four channel chains
//        run on across a group's tiles) and a warp top-k list per unit;
//     A  the window and compressed-token tiles of every unit (they do not depend on S);
//     B  the tiles of the selected blocks of every unit.
//   The ranges of phase A are sized so that every warp streams the same number of tiles.
// * A unit's selection may be cut across warps: each deposits its sorted segment list with
//   plain 64-bit stores that carry the launch's epoch tag next to the block index (no fence,
//   no counter). The helper warp of every CTA merges the segments of the units its streaming
//   warps need in phase B (polling until every word carries this launch's tag), writes idx
//   for the units whose first selected tile it holds, and publishes the block indices in shared
//   memory behind one mbarrier per unit.
// * An attention piece (the tiles of one (unit, branch) a warp covers) leaves a partial record
//   (m, l, o) with plain stores. The launch is cooperative (every CTA resident): after a grid
//   barrier (an arrival counter, bounded wait) every CTA folds the records of a share of the
//   (unit, head) pairs, applies the gates and writes O; CTA 0 then advances the epoch.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "dims.h"
#include "select_core.cuh"
#include "stream_tile.cuh"
#include "tma.h"

namespace cobs {
namespace {

#ifndef COBS_STEP_WARPS
#define COBS_STEP_WARPS 4
#endif
#ifndef COBS_STEP_STAGES
#define COBS_STEP_STAGES 3
#endif
constexpr int kStepWarps = COBS_STEP_WARPS;    // streaming warps per CTA (one per scheduler; the helper is the fifth)
constexpr int kStepStages = COBS_STEP_STAGES;  // ring depth per streaming warp
constexpr int kStepThreads = (kStepWarps + 1) * 32;
#ifndef COBS_STEP_TK
#define COBS_STEP_TK 32
#endif
constexpr int kStepTK = COBS_STEP_TK;    // keys per attention tile (16 or 32; a ring stage is 16 KiB at d = 128)
constexpr int kParts = 32 / kStepTK;     // tiles per half of a summary group (means or variances)
constexpr uint32_t kIdxBits = 25;                      // block index field of a segment word
constexpr uint32_t kIdxNone = (1u << kIdxBits) - 1u;   // an empty entry
constexpr uint32_t kTagMask = 0x7Fu;                   // epoch tag field (7 bits)

// Bytes of one ring stage: the K and V halves of a kStepTK-key tile (= one part of a summary group).
template <int D>
constexpr size_t step_stage_bytes() { return (size_t)2 * (D / 64) * kStepTK * 128; }

struct StepArgs {
    const __nv_bfloat16* Q;
    const float* summ;
    const float* gates;
    int32_t* idx;
    __nv_bfloat16* O;
    int* err;
    // workspace
    unsigned* ctl;                // [0] epoch of the last completed step, [1] grid-barrier arrivals
    unsigned long long* seg;      // [units][maxseg][32] segment lists: score bits << 32 | tag << 25 | index
    float* rec;                   // [units][3][maxw][G][D + 4] attention partial records
    // shape
    int units, G, T, k, W, nB, nC, nG, nGc, ncand, iso, D;
    int tS, tW, tC, tA;  // tiles per unit: selected blocks, window, compressed tokens, tW + tC
    int tpg;             // ring tiles per summary group (2 kParts: means + variances, kParts: isotropic)
    int gfloats;         // floats per stored summary group
    int nwarps;          // streaming warps in the grid
    long long nS, nA, nBt, tot;  // phase sizes (groups, tiles, tiles) and tpg nS + nA + nBt
    int balanced;        // phase A sized so that every warp's total is equal
    int dense[3];        // phase S, A, B: every warp's range is nonempty (else at most one element each)
    int maxseg, maxw;
    int maxbu;           // most phase-B units any CTA holds
    int mgroups;         // record merge: warp groups per CTA (pairs folded at once)
    float isd, c2, sl2;
    // reciprocals of the divisors of the partition arithmetic (exact quotients: see div_floor)
    double inv_nw, inv_nS, inv_nA, inv_nBt;
    // the same divisors' 32-bit multipliers floor((2^32 - 1) / n), set when every numerator of the
    // partition arithmetic is below 2^32 (else 0: the double path)
    uint32_t mg_nw, mg_nS, mg_nA, mg_nBt;
};

// floor(x / n) for 0 <= x < 2^50 and 1 <= n < 2^40 without an integer division. (Integer division
// and the 64-bit integer <-> double conversions are long dependent instruction sequences on the
// GPU, and the partition arithmetic sits on every warp's path.) With a multiplier mg =
// floor((2^32 - 1) / n) and x < 2^32, the high word of x mg is within 2 below the quotient
// (x mg / 2^32 > x / n - x / (n 2^32) - x / 2^32 > x / n - 2); two remainder checks correct it.
// Otherwise the double quotient estimate x * (1/n) is within 1 of the true quotient, and one
// remainder check corrects it.
__host__ __device__ __forceinline__ long long div_floor(long long x, long long n, double inv, uint32_t mg) {
#ifdef __CUDA_ARCH__
    if (mg != 0u) {
        const uint32_t xx = (uint32_t)x, nn = (uint32_t)n;
        uint32_t q = __umulhi(xx, mg);
        uint32_t r = xx - q * nn;
        if (r >= nn) { ++q; r -= nn; }
        if (r >= nn) ++q;
        return q;
    }
#endif
    long long q = (long long)((double)x * inv);
    long long r = x - q * n;
    if (r < 0) { --q; r += n; }
    if (r >= n) ++q;
    return q;
}

// Per-warp ranges of the three phases: warp v takes [f(v), f(v + 1)) of each.
__host__ __device__ __forceinline__ long long fS(const StepArgs& a, long long v) {
    return div_floor(v * a.nS, a.nwarps, a.inv_nw, a.mg_nw);
}
__host__ __device__ __forceinline__ long long fB(const StepArgs& a, long long v) {
    return div_floor(v * a.nBt, a.nwarps, a.inv_nw, a.mg_nw);
}
__host__ __device__ __forceinline__ long long fA(const StepArgs& a, long long v) {
    if (!a.balanced) return div_floor(v * a.nA, a.nwarps, a.inv_nw, a.mg_nw);
    return div_floor(v * a.tot, a.nwarps, a.inv_nw, a.mg_nw) - a.tpg * fS(a, v) - fB(a, v);
}
// The largest v with floor(v n / N) <= x: v = ceil((x + 1) N / n) - 1 (at most N - 1).
__host__ __device__ __forceinline__ int floor_part_inverse(long long x, long long n, double inv_n, uint32_t mg_n,
                                                           int N) {
    const long long v = div_floor((x + 1) * N + n - 1, n, inv_n, mg_n) - 1;
    return (int)(v < N - 1 ? v : N - 1);
}
// The warp whose range of phase PH holds element x (the largest v with f(v) <= x). The floor
// partitions invert in closed form; the balanced phase-A starts differ from v nA / N by less
// than tpg + 2, so the closed-form inverse of that floor partition is a few steps from the answer.
template <int PH>
__host__ __device__ __forceinline__ int warp_of(const StepArgs& a, long long x) {
    if (PH == 0) return floor_part_inverse(x, a.nS, a.inv_nS, a.mg_nS, a.nwarps);
    if (PH == 2) return floor_part_inverse(x, a.nBt, a.inv_nBt, a.mg_nBt, a.nwarps);
    int v = floor_part_inverse(x, a.nA, a.inv_nA, a.mg_nA, a.nwarps);
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
// Slot (0 .. pieces - 1) of the piece of warp v, whose range of the phase starts at r0. A run that
// starts inside the range (x0 >= r0) has its first piece there: slot 0, nothing to invert.
template <int PH>
__host__ __device__ __forceinline__ int run_slot(const StepArgs& a, int v, long long r0, long long x0) {
    if (x0 >= r0) return 0;
    return a.dense[PH] ? v - warp_of<PH>(a, x0) : (int)(r0 - x0);
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
// Phase-B units of CTA c: [first, last] (last < first when its warps hold no phase-B tile).
__host__ __device__ __forceinline__ void cta_bunits(const StepArgs& a, int c, int* first, int* last) {
    const long long z0 = fB(a, (long long)c * kStepWarps), z1 = fB(a, (long long)(c + 1) * kStepWarps);
    if (z1 <= z0) { *first = 0; *last = -1; return; }
    *first = (int)(z0 / a.tS);
    *last = (int)((z1 - 1) / a.tS);
}

struct Item {
    int kind;       // 0 summary means, 1 summary variances, 2 attention tile
    int unit;
    int a;          // summary group (kinds 0, 1) or branch (kind 2)
    int part;       // summary tiles: the part (channel range) of the half
    int row;        // attention: first row of K / V (branches 0, 1) or Kc / Vc (branch 2)
    unsigned mask;  // attention: valid keys of the tile (0: nothing to load)
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long seg_word(float s, int i, unsigned tag) {
    const uint32_t ix = i == kInvalid ? kIdxNone : (uint32_t)i;
    return ((unsigned long long)__float_as_uint(s) << 32) | ((unsigned long long)(tag & kTagMask) << kIdxBits) | ix;
}

// Deposit the sorted segment list of warp v for unit u (one 64-bit store per lane, tagged).
__device__ __forceinline__ void sel_deposit(const StepArgs& a, int v, long long r0, int u, const RunList& rl,
                                            unsigned ep, int lane) {
    const int slot = run_slot<0>(a, v, r0, (long long)u * a.nGc);
    a.seg[((size_t)u * a.maxseg + slot) * 32 + lane] = seg_word(rl.s, rl.i, ep);
}

// Helper warp: the merged top-k of unit u from its deposited segment lists, sorted by block index
// (-1 padded) into out[0 .. k). The segments are loaded 16 at a time (one round trip) and polled
// (bounded) until every word carries this launch's tag, staged in shared memory (hbuf, [16][32]
// words) and merged one by one; a segment whose best entry does not beat the current k-th best is
// skipped.
constexpr int kHelperRound = 16;

__device__ void helper_merge(const StepArgs& a, int u, unsigned ep, int lane, int* out, unsigned long long* hbuf) {
    float s = -INFINITY;
    int i = kInvalid;
    if (a.nGc > 0) {
        const int nseg = sel_segments(a, u);
        float ts = -INFINITY;
        int ti = kInvalid;
        const unsigned tag = ep & kTagMask;
        for (int j0 = 0; j0 < nseg; j0 += kHelperRound) {
            const int nj = min(kHelperRound, nseg - j0);
            const uint64_t t0 = global_ns();
            for (uint32_t it = 0;; ++it) {
                unsigned long long w[kHelperRound];
                bool ready = true;
#pragma unroll
                for (int q = 0; q < kHelperRound; ++q)
                    w[q] = q < nj ? ld_relaxed_u64(a.seg + ((size_t)u * a.maxseg + j0 + q) * 32 + lane) : 0ull;
#pragma unroll
                for (int q = 0; q < kHelperRound; ++q)
                    if (q < nj) ready &= (uint32_t)((w[q] >> kIdxBits) & kTagMask) == tag;
                const bool all = __all_sync(kFull, ready);
                const bool late = !all && (it >= kMaxWaitIters || global_ns() - t0 > kWaitLimitNs);
                if (all || late) {
                    if (late && lane == 0) report_error(a.err, kErrWaitTimeout);
#pragma unroll
                    for (int q = 0; q < kHelperRound; ++q) hbuf[q * 32 + lane] = w[q];
                    break;
                }
                __nanosleep(500);
            }
            __syncwarp();
#pragma unroll 1
            for (int q = 0; q < nj; ++q) {
                const unsigned long long w = hbuf[q * 32 + lane];
                const uint32_t ix = (uint32_t)w & kIdxNone;
                const float bs = __uint_as_float((uint32_t)(w >> 32));
                const int bi = ix == kIdxNone ? kInvalid : (int)ix;
                const float b0s = __shfl_sync(kFull, bs, 0);
                const int b0i = __shfl_sync(kFull, bi, 0);
                if (b0i == kInvalid || !better(b0s, b0i, ts, ti)) continue;  // uniform
                warp_merge_best_first(s, i, bs, bi, lane);
                ts = __shfl_sync(kFull, s, a.k - 1);
                ti = __shfl_sync(kFull, i, a.k - 1);
            }
            __syncwarp();
        }
    }
    const int key = warp_sort_asc(lane < a.k ? i : kInvalid, lane);
    if (lane < a.k) out[lane] = key == kInvalid ? -1 : key;
}

// Partial record of warp v's piece of (unit u, branch br): (m, l) per head in scaled log2 units
// and the unnormalised o, plain stores (folded by every CTA after the grid barrier).
template <int D>
__device__ __forceinline__ void att_flush(const StepArgs& a, int v, long long rstart, int u, int br, WState<D>& st,
                                          int lane) {
    constexpr int RF = D + 4;
    float l0 = st.l0, l1 = st.l1;
    l0 += __shfl_xor_sync(kFull, l0, 1);
    l0 += __shfl_xor_sync(kFull, l0, 2);
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);
    long long x0, len;
    branch_run(a, u, br, &x0, &len);
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
}

// The same record from the keys-as-rows state (thread t holds heads 2 (t % 4), + 1 and channels
// mt 16 + t / 4 (+ 8) of O^T).
template <int D>
__device__ __forceinline__ void att_flush_t(const StepArgs& a, int v, long long rstart, int u, int br, WStateT<D>& st,
                                            int lane) {
    constexpr int RF = D + 4;
    float l0 = st.l[0], l1 = st.l[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, o);
        l1 += __shfl_xor_sync(kFull, l1, o);
    }
    long long x0, len;
    branch_run(a, u, br, &x0, &len);
    const int slot = br == 0 ? run_slot<2>(a, v, rstart, x0) : run_slot<1>(a, v, rstart, x0);
    float* rec = a.rec + (((size_t)u * 3 + br) * a.maxw + (size_t)slot) * a.G * RF;
    const int g = lane >> 2, h0 = 2 * (lane & 3);
    const bool in0 = h0 < a.G, in1 = h0 + 1 < a.G;
    if (g == 0) {
        if (in0) {
            rec[h0 * RF + 0] = st.m[0];
            rec[h0 * RF + 1] = l0;
        }
        if (in1) {
            rec[(h0 + 1) * RF + 0] = st.m[1];
            rec[(h0 + 1) * RF + 1] = l1;
        }
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
        if (in0) {
            rec[h0 * RF + 4 + mt * 16 + g] = st.o[mt][0];
            rec[h0 * RF + 4 + mt * 16 + g + 8] = st.o[mt][2];
        }
        if (in1) {
            rec[(h0 + 1) * RF + 4 + mt * 16 + g] = st.o[mt][1];
            rec[(h0 + 1) * RF + 4 + mt * 16 + g + 8] = st.o[mt][3];
        }
    }
}

// Record merge (after the grid barrier). The CTA's NW warps form ng groups of NW / ng warps; in
// round r, group g folds pair p = blockIdx.x + (r ng + g) gridDim.x, p = unit G + head. The
// records of a pair (its selected-block, window and compressed-token pieces, in that order) are
// dealt to the group's warps in turn; each warp stages its records in its share of the free rings
// (16-byte asynchronous copies, as many per round trip as fit), folds them in order (maxima in
// log2 units) and leaves one (M, L, acc) per branch. The group's first warp then combines its warps per branch,
// applies the gates (cmp, slc, win) and writes O. The loops are kept rolled: this code runs once
// per launch, from a cold instruction cache.

// Groups of the record merge: a power of two, at most nw (every group has at least one warp), and
// no more than the pairs of the busiest CTA need.
inline int merge_groups(const StepArgs& a, int grid, int nw) {
    const long long pairs = (long long)a.units * a.G;
    const long long per = (pairs + grid - 1) / grid;  // pairs of the busiest CTA
    int ng = 1;
    while (ng * 2 <= nw && ng < per) ng *= 2;
    return ng;
}

// Running (M, L, acc) of one branch; fold one record (m, l, o) into it.
template <int CPL>
struct MergeAcc {
    float M, L, o[CPL];
    __device__ __forceinline__ void init() {
        M = -INFINITY;
        L = 0.0f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] = 0.0f;
    }
    __device__ __forceinline__ void fold(float m, float l, const float (&x)[CPL]) {
        const float nM = fmaxf(M, m);
        const float fa = M == -INFINITY ? 0.0f : exp2f(M - nM);
        const float fb = exp2f(m - nM);
        L = L * fa + l * fb;
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] = o[c] * fa + x[c] * fb;
        M = nM;
    }
    __device__ __forceinline__ void store(float* wM, float* wL, float* wO, int slot, int lane) const {
        if (lane == 0) {
            wM[slot] = M;
            wL[slot] = L;
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) wO[(size_t)slot * (CPL * 32) + lane * CPL + c] = o[c];
    }
};

// The group's first warp: combine warps w0 .. w0 + gsize - 1 per branch, gate and write O.
template <int D>
__device__ void merge_pair_finish(const StepArgs& a, int pair, int w0, int gsize, const float* gate,
                                  const float* wM, const float* wL, const float* wO) {
    constexpr int CPL = D / 32;
    const int lane = threadIdx.x & 31;
    float out[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) out[c] = 0.0f;
#pragma unroll
    for (int b = 0; b < 3; ++b) {
        float GM = -INFINITY;
        for (int w = w0; w < w0 + gsize; ++w) GM = fmaxf(GM, wM[w * 3 + b]);
        if (GM == -INFINITY) continue;
        float GL = 0.0f, sum[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) sum[c] = 0.0f;
        for (int w = w0; w < w0 + gsize; ++w) {
            const float mw = wM[w * 3 + b];
            if (mw == -INFINITY) continue;
            const float f = exp2f(mw - GM);
            GL += wL[w * 3 + b] * f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) sum[c] += wO[((size_t)w * 3 + b) * D + lane * CPL + c] * f;
        }
        if (!(GL > 0.0f)) continue;
        const float gw = gate[b == 0 ? 1 : (b == 1 ? 2 : 0)] / GL;  // gates are stored (cmp, slc, win)
#pragma unroll
        for (int c = 0; c < CPL; ++c) out[c] += gw * sum[c];
    }
    __nv_bfloat16* o = a.O + (size_t)pair * D + lane * CPL;  // pair = unit G + head = query-head row
#pragma unroll
    for (int c = 0; c < CPL; c += 2)
        *reinterpret_cast<__nv_bfloat162*>(o + c) = __floats2bfloat162_rn(out[c], out[c + 1]);
}

// TR: keys as the mma rows (groups of at most 8 heads), else the heads as the rows.
template <int D, bool TR>
__global__ void __launch_bounds__(kStepThreads, 1) decode_step_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                       const __grid_constant__ CUtensorMap tmV,
                                                                       const __grid_constant__ CUtensorMap tmKc,
                                                                       const __grid_constant__ CUtensorMap tmVc,
                                                                       StepArgs a) {
    constexpr int kBox = kStepTK * 128;    // one 64-column box of a 16-row tile
    constexpr int kMat = (D / 64) * kBox;  // K or V part of an attention tile
    constexpr int kStage = 2 * kMat;       // one K + V tile
    static_assert(kStage == step_stage_bytes<D>(), "the launch sizes the rings with the same stage bytes");
    static_assert(kStage * kParts == D * 32 * 4, "an attention tile and a summary part fill one stage");
    static_assert((size_t)(kStepWarps + 1) * 3 * D * 4 <= (size_t)kStepWarps * kStepStages * kStage,
                  "the merge scratch fits in the rings");
    constexpr int kPartC = D / kParts;     // channels of a summary part
    constexpr bool kIL = D == 128;         // K / V tiles as one [rows][2][64] box (both column halves)
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[kStepWarps][kStepStages];
    __shared__ __align__(16) float qsm[kStepWarps][2][D];         // group query: Qsum, Q2
    __shared__ __align__(16) float iso_sm[kStepWarps][kStepStages][32];
    __shared__ float q2t_sm[kStepWarps];
    __shared__ Item desc[kStepWarps][kStepStages];
    __shared__ __align__(16) unsigned long long hbuf[kHelperRound * 32];  // helper staging
    __shared__ float wM[(kStepWarps + 1) * 3], wL[(kStepWarps + 1) * 3];  // record merge scratch
    __shared__ float gsm[(kStepWarps + 1) * 3];                           // gates of the first merge round
    __shared__ int merge_ok;
    __shared__ int npc[(kStepWarps + 1) * 3];  // pieces of each branch of the first merge round's pairs
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // phase-B block indices published by the helper warp: [maxbu][32] int, then [maxbu] mbarriers
    int* bidx = reinterpret_cast<int*>(base + (size_t)kStepWarps * kStepStages * kStage);
    uint64_t* ubar = reinterpret_cast<uint64_t*>(bidx + (size_t)a.maxbu * 32);
    const unsigned ep = *reinterpret_cast<volatile unsigned*>(a.ctl) + 1u;
    int bu_first, bu_last;
    cta_bunits(a, blockIdx.x, &bu_first, &bu_last);

    if (threadIdx.x == 0) {
        for (int j = 0; j <= bu_last - bu_first; ++j) mbar_init(&ubar[j], 32);  // every helper lane arrives
        fence_barrier_init();
    }
    __syncthreads();

    // ------------------------------------------------------------------ helper warp
    if (warp == kStepWarps) {
        for (int u = bu_first; u <= bu_last; ++u) {
            int* out = bidx + (size_t)(u - bu_first) * 32;
            helper_merge(a, u, ep, lane, out, hbuf);
            // the CTA that holds the unit's first selected tile writes idx
            if (lane < a.k && fB(a, (long long)blockIdx.x * kStepWarps) <= (long long)u * a.tS)
                a.idx[(size_t)u * a.k + lane] = out[lane];
            mbar_arrive(&ubar[u - bu_first]);  // each lane releases the indices it wrote
        }
        // while the streaming warps finish: the piece counts of the first merge round's pairs
        if (lane < a.mgroups * 3) {
            const long long p = blockIdx.x + (long long)(lane / 3) * gridDim.x;
            if (p < (long long)a.units * a.G) npc[lane] = branch_pieces(a, (int)(p / a.G), lane % 3);
        }
    } else {
        // ------------------------------------------------------------------ streaming warps
        unsigned char* ring = base + (size_t)warp * kStepStages * kStage;
        uint64_t* bar = bars[warp];
        const int v = blockIdx.x * kStepWarps + warp;
        const long long s0 = fS(a, v), s1 = fS(a, v + 1);
        const long long a0 = fA(a, v), a1 = fA(a, v + 1);
        const long long b0 = fB(a, v), b1 = fB(a, v + 1);
        const int nSi = (int)(s1 - s0) * a.tpg, nAi = (int)(a1 - a0), nBi = (int)(b1 - b0);
        const int n = nSi + nAi + nBi;

        if (lane == 0) {
            for (int s = 0; s < kStepStages; ++s) mbar_init(&bar[s], 1);
            fence_barrier_init();
        }
        __syncwarp();

        const int t = a.T - 1;
        uint32_t phase = 0;    // bit s: parity of the next completion of stage s
        bool ok = true;        // false after a timed-out wait (uniform across the warp)
        uint32_t pending = 0;  // stages with a copy in flight (lane 0's view)
        int ready_u = -1;      // phase-B unit whose indices this warp has seen published
        // descriptor of this warp's item i (uniform across the warp); element indices fit in int32
        // descriptor of item i; a phase-B item first waits for its unit's published indices
        auto item_at = [&](int i) {
            Item it;
            it.row = 0;
            it.mask = 0u;
            if (i < nSi) {
                const int x = (int)s0 + i / a.tpg;
                const int r = i - (i / a.tpg) * a.tpg;
                it.kind = r / kParts;
                it.part = r % kParts;
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
                    const int r0 = max(0, t - a.W + 1) + l * kStepTK;
                    it.row = it.unit * a.T + r0;
                    const int nk = min(kStepTK, t + 1 - r0);
                    it.mask = nk >= 32 ? kFull : ((1u << nk) - 1u);
                } else {
                    it.a = 2;
                    const int c0 = (l - a.tW) * kStepTK;
                    it.row = it.unit * a.nC + c0;
                    const int nk = min(kStepTK, a.nC - c0);
                    it.mask = nk >= 32 ? kFull : ((1u << nk) - 1u);
                }
            } else {
                const int z = (int)b0 + (i - nSi - nAi);
                it.kind = 2;
                it.a = 0;
                it.unit = z / a.tS;
                const int l = z - it.unit * a.tS;
                const int j = it.unit - bu_first;  // this CTA's slot of the unit
                if (it.unit != ready_u) {
                    if (ok) ok = mbar_wait(&ubar[j], 0, a.err);  // the helper published the unit's indices
                    ok = __all_sync(kFull, ok);
                    ready_u = it.unit;
                }
                const int bi = ok ? bidx[(size_t)j * 32 + l / (64 / kStepTK)] : -1;
                if (bi >= 0) {
                    if (bi >= a.nB) {
                        if (lane == 0) report_error(a.err, kErrBadIndex);
                    } else {
                        it.row = it.unit * a.T + bi * 64 + (l % (64 / kStepTK)) * kStepTK;
                        it.mask = kStepTK == 32 ? kFull : 0xFFFFu;
                    }
                }
            }
            return it;
        };
        auto issue = [&](const Item& it, int s) {  // lane 0 only
            unsigned char* dst = ring + (size_t)s * kStage;
            if (it.kind < 2) {
                pending |= 1u << s;
                const float* g = a.summ + ((size_t)it.unit * a.nG + it.a) * a.gfloats;
                // the isotropic scalars come with the last part of the means
                const bool iso_here = a.iso && it.part == kParts - 1;
                mbar_arrive_expect_tx(&bar[s], kStage + (iso_here ? 128u : 0u));
                bulk_g2s(dst, g + (size_t)it.kind * D * 32 + (size_t)it.part * (kStage / 4), kStage, &bar[s]);
                if (iso_here) bulk_g2s(iso_sm[warp][s], g + D * 32, 128, &bar[s]);
                return;
            }
            if (it.mask == 0u) return;
            pending |= 1u << s;
            const CUtensorMap* mk = it.a == 2 ? &tmKc : &tmK;
            const CUtensorMap* mv = it.a == 2 ? &tmVc : &tmV;
            mbar_arrive_expect_tx(&bar[s], kStage);
            if (kIL) {  // one 3-D box per tensor: rows it.row .. it.row + 15, both column halves
                tma_load_3d(dst, mk, 0, 0, it.row, &bar[s]);
                tma_load_3d(dst + kMat, mv, 0, 0, it.row, &bar[s]);
            } else {
                tma_load_2d(dst, mk, 0, it.row, &bar[s]);
                tma_load_2d(dst + kMat, mv, 0, it.row, &bar[s]);
            }
        };


        int next_issue = 0;
        bool sel_done = nSi == 0;  // this warp's selection segments are all deposited
        // issue every item whose stage is free (item i uses stage i % kStepStages); a phase-B item only
        // once this warp's own segments are deposited (the helper it waits for may need them)
        auto issue_ahead = [&](int consumed) {
            while (next_issue < n && next_issue < consumed + kStepStages && (next_issue < nSi + nAi || sel_done)) {
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
        float ch[4] = {0.f, 0.f, 0.f, 0.f};  // the four canonical chains of the current half
        std::conditional_t<TR, WStateT<D>, WState<D>> st;
        st.init();
        uint32_t qa[D / 16][TR ? 2 : 4];
        int att_u = -1, att_br = -1, q_u = -1;

        issue_ahead(0);
        for (int i = 0; i < n; ++i) {
            issue_ahead(i);
            const int s = i % kStepStages;
            const Item it = desc[warp][s];
            const unsigned char* stage = ring + (size_t)s * kStage;
            if (it.kind < 2) {
                if (it.unit != sel_u) {
                    if (sel_u >= 0) sel_deposit(a, v, s0, sel_u, rl, ep, lane);
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
                if (it.part == 0) ch[0] = ch[1] = ch[2] = ch[3] = 0.0f;
                // channels [part kPartC, (part + 1) kPartC) of the means (Qsum) or variances (Q2)
                if (ok) score_chains<kPartC / 4>(tile, qsm[warp][it.kind] + it.part * kPartC, lane, ch);
                if (it.part == kParts - 1) {
                    const float half_sum = combine4(ch[0], ch[1], ch[2], ch[3]);
                    if (it.kind == 0) {
                        apart = half_sum;
                        if (a.iso) {
                            sc = score_combine(apart, __fmul_rn(q2t_sm[warp], iso_sm[warp][s][lane]), a.isd, a.c2);
                            done_group = true;
                        }
                    } else {
                        sc = score_combine(apart, half_sum, a.isd, a.c2);
                        done_group = true;
                    }
                }
                if (done_group) {
                    const bool valid = ok && b < a.ncand;
                    rl.add(valid ? sc : -INFINITY, valid ? b : kInvalid, a.k, lane);
                }
                if (i == nSi - 1) {  // the last summary tile of this warp
                    sel_deposit(a, v, s0, sel_u, rl, ep, lane);
                    sel_u = -1;
                    sel_done = true;
                }
            } else {
                if (it.unit != att_u || it.a != att_br) {
                    if (att_u >= 0) {
                        if constexpr (TR) att_flush_t<D>(a, v, att_br == 0 ? b0 : a0, att_u, att_br, st, lane);
                        else att_flush<D>(a, v, att_br == 0 ? b0 : a0, att_u, att_br, st, lane);
                    }
                    st.init();
                    att_u = it.unit;
                    att_br = it.a;
                    if (att_u != q_u) {
                        if constexpr (TR) load_qt<D>(a.Q + (size_t)att_u * a.G * D, a.G, qa, lane);
                        else load_q<D>(a.Q + (size_t)att_u * a.G * D, a.G, qa, lane);
                        q_u = att_u;
                    }
                }
                if (it.mask != 0u) {
                    if (ok) ok = mbar_wait(&bar[s], (phase >> s) & 1u, a.err);
                    ok = __all_sync(kFull, ok);
                    if (ok) pending &= ~(1u << s);
                    phase ^= 1u << s;
                    if (ok) {
                        if constexpr (TR) tile_mma_t<D, kStepTK, kIL>(st, qa, stage, stage + kMat, it.mask, a.sl2, lane);
                        else tile_mma<D, kStepTK, kIL>(st, qa, stage, stage + kMat, it.mask, a.sl2, lane);
                    }
                }
            }
            __syncwarp();
        }
        if (att_u >= 0) {
            if constexpr (TR) att_flush_t<D>(a, v, att_br == 0 ? b0 : a0, att_u, att_br, st, lane);
            else att_flush<D>(a, v, att_br == 0 ? b0 : a0, att_u, att_br, st, lane);
        }
        // after a timed-out wait: let the copies still in flight land (bounded) before the CTA exits
        if (lane == 0 && !ok)
            for (int s = 0; s < kStepStages; ++s)
                if ((pending >> s) & 1u) mbar_wait(&bar[s], (phase >> s) & 1u, nullptr);
    }

    // ------------------------------------------------------------------ grid barrier, record merge
    // Every CTA is resident (cooperative launch, one per SM). The arrival counter ctl[1] grows by
    // the grid size per step, so this step's barrier is complete at ep x gridDim.x arrivals.
    constexpr int kNW = kStepWarps + 1;
    const int ng = min(max(a.mgroups, 1), kNW), gsize = kNW / ng;  // gsize >= 1 (the loops step by it)
    const int grp = warp / gsize, gw = warp - grp * gsize;  // warps past ng groups (kNW % ng) stay idle
    const long long pairs = (long long)a.units * a.G;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();  // this CTA's records and idx are visible before its arrival
        atomicAdd(&a.ctl[1], 1u);
        const unsigned target = ep * gridDim.x;
        const uint64_t t0 = global_ns();
        bool late = false;
        for (uint32_t it = 0; (int)(ld_acquire_u32(&a.ctl[1]) - target) < 0; ++it) {
            if (it >= kMaxWaitIters || global_ns() - t0 > kWaitLimitNs) {
                late = true;
                break;
            }
            __nanosleep(64);
        }
        if (late) report_error(a.err, kErrWaitTimeout);
        __threadfence();
        merge_ok = late ? 0 : 1;
    } else if (threadIdx.x < 1 + ng * 3) {  // meanwhile: the gates of the first round's pairs
        const int g = (threadIdx.x - 1) / 3, j = (threadIdx.x - 1) % 3;
        const long long p = blockIdx.x + (long long)g * gridDim.x;
        if (p < pairs) gsm[g * 3 + j] = __ldg(a.gates + p * 3 + j);
    }
    __syncthreads();
    if (merge_ok) {
        constexpr int CPL = D / 32;
        constexpr int kRecBytes = (D + 4) * 4;  // one head's record: m, l, 2 pad, o[D]
        constexpr int kRecChunks = kRecBytes / 16;
        constexpr size_t kRingBytes = (size_t)kStepWarps * kStepStages * kStage;
        constexpr size_t kScratch = (size_t)kNW * 3 * D * 4;
        constexpr int kCap = (int)((kRingBytes - kScratch) / kNW / kRecBytes);  // records per warp per round trip
        static_assert(kRecBytes % 16 == 0 && kCap >= 1, "records are staged in 16-byte pieces");
        float* wO = reinterpret_cast<float*>(base + kRingBytes - kScratch);  // [kNW][3][D]
        unsigned char* mine = base + (size_t)warp * kCap * kRecBytes;      // this warp's staging slots
        const size_t rs = (size_t)a.G * (D + 4);
        for (int r = 0;; ++r) {
            const long long p0 = blockIdx.x + (long long)r * ng * gridDim.x;
            if (p0 >= pairs) break;  // uniform across the CTA
            const long long p = p0 + (long long)grp * gridDim.x;
            const int pair = grp < ng && p < pairs ? (int)p : -1;
            if (lane == 0)
                for (int b = 0; b < 3; ++b) wM[warp * 3 + b] = -INFINITY;
            MergeAcc<CPL> acc;
            acc.init();
            int cb = 0;  // branch of acc
            if (pair >= 0) {
                const int unit = pair / a.G, h = pair - unit * a.G;
                const int n0 = r == 0 ? npc[grp * 3] : branch_pieces(a, unit, 0);
                const int n01 = n0 + (r == 0 ? npc[grp * 3 + 1] : branch_pieces(a, unit, 1));
                const int nr = n01 + (r == 0 ? npc[grp * 3 + 2] : branch_pieces(a, unit, 2));
                const float* rbase = a.rec + (size_t)unit * 3 * a.maxw * rs + (size_t)h * (D + 4);
                // this warp's records: gw, gw + gsize, ...; kCap of them per round trip
#pragma unroll 1
                for (int x0 = gw; x0 < nr; x0 += kCap * gsize) {
                    int nx = 0;
#pragma unroll 1
                    for (int x = x0; x < nr && nx < kCap; x += gsize, ++nx) {
                        const int b = x < n0 ? 0 : (x < n01 ? 1 : 2);
                        const int sl = x - (b == 0 ? 0 : (b == 1 ? n0 : n01));
                        const unsigned char* src =
                            reinterpret_cast<const unsigned char*>(rbase + ((size_t)b * a.maxw + sl) * rs);
                        for (int j = lane; j < kRecChunks; j += 32)
                            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                                             smem_addr(mine + (size_t)nx * kRecBytes + j * 16)),
                                         "l"(src + j * 16)
                                         : "memory");
                    }
                    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
                    __syncwarp();
#pragma unroll 1
                    for (int q = 0; q < nx; ++q) {
                        const int x = x0 + q * gsize;
                        const int b = x < n0 ? 0 : (x < n01 ? 1 : 2);
                        if (b != cb) {
                            acc.store(wM, wL, wO, warp * 3 + cb, lane);
                            acc.init();
                            cb = b;
                        }
                        const float* rp = reinterpret_cast<const float*>(mine + (size_t)q * kRecBytes);
                        const float m = rp[0];
                        if (m == -INFINITY) continue;
                        float o[CPL];
#pragma unroll
                        for (int c = 0; c < CPL; ++c) o[c] = rp[4 + lane * CPL + c];
                        acc.fold(m, rp[1], o);
                    }
                    __syncwarp();  // the slots are read before the next copies
                }
            }
            acc.store(wM, wL, wO, warp * 3 + cb, lane);
            __syncthreads();
            if (gw == 0 && pair >= 0)
                merge_pair_finish<D>(a, pair, warp, gsize, r == 0 ? gsm + grp * 3 : a.gates + (size_t)pair * 3, wM,
                                     wL, wO);
            __syncthreads();
        }
    }
    // the epoch advances once every CTA has passed the barrier (all read it at their start)
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(&a.ctl[0], 1u);

}

// Workspace layout: the control word, the segment lists and the attention records (each region
// 256-byte aligned).
struct StepLayout {
    size_t ctl, seg, rec, total;
};

inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }

StepLayout step_layout(const StepArgs& a) {
    StepLayout L;
    size_t o = 0;
    L.ctl = o; o = al256(o + 2 * sizeof(unsigned));
    L.seg = o; o = al256(o + (size_t)a.units * a.maxseg * 32 * sizeof(unsigned long long));
    L.rec = o; o = al256(o + (size_t)a.units * 3 * a.maxw * a.G * (a.D + 4) * sizeof(float));
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
    a.tpg = (m.iso ? 1 : 2) * kParts;
    a.gfloats = (int)m.group_floats();
    a.tS = m.k * (64 / kStepTK);
    a.tW = (std::min(m.W, m.T) + kStepTK - 1) / kStepTK;
    a.tC = (m.nC + kStepTK - 1) / kStepTK;
    a.tA = a.tW + a.tC;
    a.nwarps = sm_count() * kStepWarps;
    a.nS = (long long)a.units * a.nGc;
    a.nA = (long long)a.units * a.tA;
    a.nBt = (long long)a.units * a.tS;
    a.tot = a.tpg * a.nS + a.nA + a.nBt;
    a.inv_nw = 1.0 / a.nwarps;
    a.inv_nS = a.nS > 0 ? 1.0 / (double)a.nS : 0.0;
    a.inv_nA = a.nA > 0 ? 1.0 / (double)a.nA : 0.0;
    a.inv_nBt = a.nBt > 0 ? 1.0 / (double)a.nBt : 0.0;
    // 32-bit division multipliers when every numerator fits: v n <= nwarps tot and
    // (x + 1) nwarps + n - 1 <= (nwarps + 1) tot
    const bool narrow = (unsigned long long)(a.nwarps + 1) * (unsigned long long)(a.tot + 1) < (1ull << 32);
    auto mg = [&](long long n) { return narrow && n > 0 ? (uint32_t)(0xFFFFFFFFull / (unsigned long long)n) : 0u; };
    a.mg_nw = mg(a.nwarps);
    a.mg_nS = mg(a.nS);
    a.mg_nA = mg(a.nA);
    a.mg_nBt = mg(a.nBt);
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
    a.mgroups = merge_groups(a, a.nwarps / kStepWarps, kStepWarps + 1);
    a.maxbu = 1;
    for (int c = 0; c < a.nwarps / kStepWarps; ++c) {
        int f, l;
        cta_bunits(a, c, &f, &l);
        a.maxbu = std::max(a.maxbu, l - f + 1);
    }
    float isd, c2;
    score_constants(m.d, m.alpha, &isd, &c2);
    a.isd = isd;
    a.c2 = c2;
    a.sl2 = 1.4426950408889634f / sqrtf((float)m.d);
    return a;
}

// Dynamic shared memory: the rings, then the phase-B index table and its mbarriers, plus the
// alignment slack of the ring base.
template <int D>
size_t step_smem(const StepArgs& a) {
    return (size_t)kStepWarps * kStepStages * step_stage_bytes<D>() +
           (size_t)a.maxbu * (32 * sizeof(int) + sizeof(uint64_t)) + 1024;
}

template <int D, bool TR>
cudaError_t launch_step_d(const Dims& m, StepArgs a, const void* K, const void* V, const void* Kc, const void* Vc,
                          cudaStream_t s) {
    CUtensorMap tk, tv, tkc, tvc;
    const uint64_t kvrows = (uint64_t)m.units() * m.T;
    const uint64_t crows = m.nC > 0 ? (uint64_t)m.units() * m.nC : kvrows;
    // d = 128: a [rows][2][64] view (row pitch 256 bytes, half pitch 128) read in boxes of
    // kStepTK rows x both halves; d = 64: [rows][64] in boxes of kStepTK rows
    auto enc = [&](CUtensorMap* map, const void* base, uint64_t rows) {
        if (D == 128) {
            const uint64_t dims[3] = {64, 2, rows};
            const uint64_t strides[2] = {128, 256};
            const uint32_t box[3] = {64, 2, (uint32_t)kStepTK};
            return encode_tmap_bf16_3d(map, base, dims, strides, box);
        }
        return encode_tmap_bf16_2d(map, base, rows, D, kStepTK);
    };
    if (!enc(&tk, K, kvrows) || !enc(&tv, V, kvrows) || !enc(&tkc, m.nC > 0 ? Kc : K, crows) ||
        !enc(&tvc, m.nC > 0 ? Vc : V, crows))
        return cudaErrorInvalidValue;
    const size_t smem = step_smem<D>(a);
    cudaError_t e =
        cudaFuncSetAttribute(decode_step_kernel<D, TR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_step_kernel<D, TR>, kStepThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorNotSupported;
    // cooperative: every CTA resident at once (the record merge follows a grid barrier)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.nwarps / kStepWarps);
    cfg.blockDim = dim3(kStepThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, decode_step_kernel<D, TR>, tk, tv, tkc, tvc, a);
}

}  // namespace

bool decode_step_supported(const Dims& m) {
    // the phase-B index table of a CTA must fit beside the rings (checked on the host sizes)
    if (!(m.dtype == COBS_BF16 && !m.lr && (m.d == 128 || m.d == 64) && m.L == 64 &&
          (long long)m.nB < (1ll << kIdxBits) - 1))
        return false;
    const StepArgs a = make_step_args(m);
    return (m.d == 128 ? step_smem<128>(a) : step_smem<64>(a)) <= 200 * 1024;
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
    a.seg = reinterpret_cast<unsigned long long*>(w + L.seg);
    a.rec = reinterpret_cast<float*>(w + L.rec);
    // groups of at most 8 heads: keys as the mma rows
    if (m.G <= 8)
        return m.d == 128 ? launch_step_d<128, true>(m, a, K, V, Kc, Vc, s) : launch_step_d<64, true>(m, a, K, V, Kc, Vc, s);
    return m.d == 128 ? launch_step_d<128, false>(m, a, K, V, Kc, Vc, s) : launch_step_d<64, false>(m, a, K, V, Kc, Vc, s);
}

}  // namespace cobs
