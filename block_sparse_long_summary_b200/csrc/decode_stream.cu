// Decode attention, bf16: stream-K over 32-key tiles with TMA tensor tiles.
//
// What is computed is the decode attention of the NSA paths (Janus issue #181: CMP, SLC,
// WIN) with COBS-selected blocks (gist.science explainer §2.3); only the selected blocks,
// the window and the compressed tokens are read ("Problemstellung": decode is bound by the
// KV-cache read). How it is scheduled:
//
// * The tiles form two sequences: phase A, every (batch, KV-head) unit's WIN tiles (the window
//   rows in 32-row tiles) then its CMP tiles (compressed tokens in 32-row tiles), unit after
//   unit; phase B, every unit's SLC tiles (2 per selected block). Each phase is cut into
//   equal, contiguous ranges, one per warp, and every warp streams its phase-A range and then
//   its phase-B range, so every SM streams the same number of bytes in each phase.
// * After a selection in the same stream (the decode step) the grid is launched as a
//   programmatic dependent of the selection: phase A, which does not depend on it, streams
//   while the selection runs; a warp waits for the selection grid (griddepcontrol.wait)
//   before it reads its first selected-block index.
// * Each warp is its own producer: TMA 2-D loads (128-byte swizzle, no multicast) of the
//   K and V halves of a tile into a private 2-stage ring (one tile first, the second once it
//   has landed, then each stage refilled once consumed, or after the decode step's selection
//   once the tile before has landed), an mbarrier per stage (2 stages of
//   16 KiB per warp: the 128 KiB a CTA holds leave room on the SM for the selection grid the
//   attention overlaps in the decode step; measured faster in the step than 3 stages).
// * The G query heads of the unit are the m16 rows of mma.sync tiles (rows >= G are zero);
//   the online softmax state lives in registers.
// * A warp flushes one partial record (m, l, o) per (unit, branch) piece it covers;
//   decode_stream_merge combines the records of each (unit, branch), applies the gates
//   and writes O.
#include <algorithm>

#include "common.cuh"
#include "dims.h"
#include "stream_tile.cuh"
#include "tma.h"

namespace cobs {
namespace {

#ifndef COBS_DECODE_STAGES
#define COBS_DECODE_STAGES 2
#endif
#ifndef COBS_DECODE_WARPS
#define COBS_DECODE_WARPS 4
#endif
constexpr int kStages = COBS_DECODE_STAGES;  // ring depth per warp
constexpr int kWarps = COBS_DECODE_WARPS;    // independent warps per CTA
static_assert(kStages >= 2, "ring of at least two stages");

struct StreamArgs {
    const __nv_bfloat16* Q;
    const int32_t* idx;
    const float* gates;
    __nv_bfloat16* O;
    float* rec;
    int* err;
    int Hq, Hkv, G, T, L, k, W, nB, nC;
    int tS, tW, tC, tAu;  // tiles per unit: SLC, WIN, CMP, WIN + CMP
    long long nA, nBt;    // tiles of phase A (units * tAu) and phase B (units * tS)
    int tpwA, tpwB;       // tiles per warp in each phase
    int maxw;             // record slots per (unit, branch)
    int lazy;             // refill a stage only once the tile before the one in it has landed
    float sl2;            // log2(e) / sqrt(d)
};

__host__ __device__ __forceinline__ int rec_floats(int D) { return D + 4; }  // m, l, pad, pad, o[D]

// First tile of (unit, br) in its phase's sequence and that phase's tiles per warp: WIN
// [0, tW) and CMP [tW, tAu) of the unit's phase-A tiles, SLC [0, tS) of its phase-B tiles.
__host__ __device__ __forceinline__ long long piece_begin(const StreamArgs& a, int unit, int br) {
    return br == 0 ? (long long)unit * a.tS : (long long)unit * a.tAu + (br == 2 ? a.tW : 0);
}
__host__ __device__ __forceinline__ int phase_tpw(const StreamArgs& a, int br) { return br == 0 ? a.tpwB : a.tpwA; }
__host__ __device__ __forceinline__ int branch_len(const StreamArgs& a, int br) {
    return br == 0 ? a.tS : (br == 1 ? a.tW : a.tC);
}

struct Tile {
    int unit, br, j;   // branch 0 SLC, 1 WIN, 2 CMP; j = tile within the branch
    int row;           // first global row in K/V (SLC, WIN) or Kc/Vc (CMP)
    uint32_t mask;     // valid keys of the tile
};

// Tile gt of the joint numbering (phase A in [0, nA), phase B from nA). Uniform across the
// warp. Before the first selected-block index it reads, the warp waits for the grid it depends
// on (the selection), once.
__device__ __forceinline__ Tile tile_at(const StreamArgs& a, long long gt, bool& waited) {
    Tile tl;
    const int t = a.T - 1;
    if (gt >= a.nA) {
        if (!waited) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            waited = true;
        }
        const long long q = gt - a.nA;
        tl.unit = (int)(q / a.tS);
        const int l = (int)(q - (long long)tl.unit * a.tS);
        tl.br = 0;
        tl.j = l;
        const int bi = a.idx[(size_t)tl.unit * a.k + l / (64 / kTK)];
        tl.mask = 0u;
        tl.row = 0;
        if (bi >= 0) {
            if (bi >= a.nB) {
                report_error(a.err, kErrBadIndex);
            } else {
                tl.row = tl.unit * a.T + bi * a.L + (l % (64 / kTK)) * kTK;
                tl.mask = kTK == 32 ? kFull : 0xFFFFu;
            }
        }
        return tl;
    }
    tl.unit = (int)(gt / a.tAu);
    const int l = (int)(gt - (long long)tl.unit * a.tAu);
    if (l < a.tW) {
        tl.br = 1;
        tl.j = l;
        const int r0 = max(0, t - a.W + 1) + tl.j * kTK;
        tl.row = tl.unit * a.T + r0;
        const int n = min(kTK, t + 1 - r0);
        tl.mask = n >= 32 ? kFull : ((1u << n) - 1u);  // n <= kTK
    } else {
        tl.br = 2;
        tl.j = l - a.tW;
        const int c0 = tl.j * kTK;
        tl.row = tl.unit * a.nC + c0;
        const int n = min(kTK, a.nC - c0);
        tl.mask = n >= 32 ? kFull : ((1u << n) - 1u);
    }
    return tl;
}

// Partial record of (unit, br) written by warp v.
template <int D>
__device__ __forceinline__ void flush(const StreamArgs& a, long long v, int unit, int br, WState<D>& st, int lane) {
    float l0 = st.l0, l1 = st.l1;
    l0 += __shfl_xor_sync(kFull, l0, 1);
    l0 += __shfl_xor_sync(kFull, l0, 2);
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);
    const long long first_v = piece_begin(a, unit, br) / phase_tpw(a, br);
    float* rec = a.rec + (((size_t)unit * 3 + br) * a.maxw + (size_t)(v - first_v)) * a.G * rec_floats(D);
    const int r0 = lane >> 2, r1 = r0 + 8, c = 2 * (lane & 3);
    if ((lane & 3) == 0) {
        if (r0 < a.G) {
            rec[r0 * rec_floats(D) + 0] = st.m0;
            rec[r0 * rec_floats(D) + 1] = l0;
        }
        if (r1 < a.G) {
            rec[r1 * rec_floats(D) + 0] = st.m1;
            rec[r1 * rec_floats(D) + 1] = l1;
        }
    }
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        if (r0 < a.G)
            *reinterpret_cast<float2*>(rec + r0 * rec_floats(D) + 4 + nd * 8 + c) = make_float2(st.o[nd][0], st.o[nd][1]);
        if (r1 < a.G)
            *reinterpret_cast<float2*>(rec + r1 * rec_floats(D) + 4 + nd * 8 + c) = make_float2(st.o[nd][2], st.o[nd][3]);
    }
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) decode_stream_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const __grid_constant__ CUtensorMap tmKc,
                                                                     const __grid_constant__ CUtensorMap tmVc,
                                                                     StreamArgs a) {
    constexpr int kBox = kTK * 128;              // one 64-column box
    constexpr int kMat = (D / 64) * kBox;        // K or V tile
    constexpr int kStage = 2 * kMat;             // K + V
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[kWarps][kStages];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // 1024-byte aligned ring of this warp
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* ring = base + (size_t)warp * kStages * kStage;
    uint64_t* bar = bars[warp];

    // the merge grid may be scheduled now; it still waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const long long v = (long long)blockIdx.x * kWarps + warp;
    // this warp's ranges: [a0, a0 + nAw) of phase A, then [b0, b0 + nBw) of phase B
    const long long a0 = v * a.tpwA, b0 = v * a.tpwB;
    const int nAw = (int)max(0LL, min(a.nA, a0 + a.tpwA) - a0);
    const int nBw = (int)max(0LL, min(a.nBt, b0 + a.tpwB) - b0);
    const int n = nAw + nBw;
    if (n == 0) return;
    auto gt_of = [&](int i) -> long long { return i < nAw ? a0 + i : a.nA + b0 + (i - nAw); };

    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bar[s], 1);
        fence_barrier_init();
    }
    __syncwarp();

    auto issue = [&](const Tile& tl, int s) {  // lane 0 only
        if (tl.mask == 0u) return;
        const CUtensorMap* mk = tl.br == 2 ? &tmKc : &tmK;
        const CUtensorMap* mv = tl.br == 2 ? &tmVc : &tmV;
        unsigned char* dst = ring + (size_t)s * kStage;
        mbar_arrive_expect_tx(&bar[s], kStage);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
            tma_load_2d(dst + h * kBox, mk, h * 64, tl.row, &bar[s]);
            tma_load_2d(dst + kMat + h * kBox, mv, h * 64, tl.row, &bar[s]);
        }
    };
    // descriptors of the next kStages tiles, in registers: a selected block's index is read
    // when its tile is prefetched, not when it is consumed
    Tile tq[kStages];
    bool waited = false;
#pragma unroll
    for (int j = 0; j < kStages; ++j) tq[j] = j < n ? tile_at(a, gt_of(j), waited) : Tile{0, 0, 0, 0, 0u};
    // one tile now and the rest of the ring once it has landed: the grid's opening burst is one
    // tile per warp, so the first tiles land sooner. From then on each stage is refilled as soon
    // as its tile has been consumed or, lazy (the decode step, where the grid streams beside the
    // selection's tail), only once the tile before has landed: fewer loads in flight per warp,
    // measured 1 us faster per step there and 2 us slower alone
    if (lane == 0 && n > 0) issue(tq[0], 0);

    uint32_t phase = 0;  // bit s: parity of the next completion of stage s
    uint32_t qa[D / 16][4];
    WState<D> st;
    st.init();
    Tile cur = tq[0];
    load_q<D>(a.Q + (size_t)cur.unit * a.G * D, a.G, qa, lane);
    bool ok = true;
    for (int i = 0; i < n; ++i) {
        const int s = i % kStages;
        const Tile tl = tq[0];
#pragma unroll
        for (int j = 0; j + 1 < kStages; ++j) tq[j] = tq[j + 1];
        const bool more = i + kStages < n;
        tq[kStages - 1] = more ? tile_at(a, gt_of(i + kStages), waited) : Tile{0, 0, 0, 0, 0u};
        if (tl.unit != cur.unit || tl.br != cur.br) {
            flush<D>(a, v, cur.unit, cur.br, st, lane);
            st.init();
            if (tl.unit != cur.unit) load_q<D>(a.Q + (size_t)tl.unit * a.G * D, a.G, qa, lane);
            cur = tl;
        }
        if (tl.mask != 0u) {
            if (ok) ok = mbar_wait(&bar[s], (phase >> s) & 1u, a.err);
            ok = __all_sync(kFull, ok);
            phase ^= 1u << s;
        }
        if (a.lazy) {  // tile i + kStages - 1 into the stage of tile i - 1, read by every lane by now
            if (lane == 0 && ok && i + kStages - 1 < n) {
                fence_proxy_async();
                issue(tq[kStages - 2], (i + kStages - 1) % kStages);
            }
        } else if (i == 0 && lane == 0 && ok) {  // the rest of the ring: tiles 1 .. kStages - 1
#pragma unroll
            for (int j = 0; j + 1 < kStages; ++j)
                if (1 + j < n) issue(tq[j], 1 + j);
        }
        if (tl.mask != 0u && ok)
            tile_mma<D>(st, qa, ring + (size_t)s * kStage, ring + (size_t)s * kStage + kMat, tl.mask, a.sl2, lane);
        __syncwarp();
        if (!a.lazy && lane == 0 && ok && more) {  // tile i + kStages into the stage just consumed
            fence_proxy_async();
            issue(tq[kStages - 1], s);
        }
    }
    flush<D>(a, v, cur.unit, cur.br, st, lane);
}

// grid (G, units), 8 warps per (unit, head): warps 0-2 fold the SLC records (every third slot),
// warp 3 the WIN records, warps 4-7 the CMP records (every fourth slot); each warp keeps the
// loads of 8 records in flight. Warp 0 then combines the warps of each branch, applies the
// gates (cmp, slc, win) and writes O. Launched as a programmatic dependent of the decode
// kernel: it waits for that grid before reading records.
constexpr int kMergeWarps = 8;
constexpr int kMergeBatch = 8;
__host__ __device__ __forceinline__ int merge_branch(int w) { return w < 3 ? 0 : (w == 3 ? 1 : 2); }

template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32) decode_stream_merge(StreamArgs a) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float wM[kMergeWarps], wL[kMergeWarps];
    __shared__ float wO[kMergeWarps][D];
    const int h = blockIdx.x, unit = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int hq_row = unit * a.G + h;  // = b * Hq + g * G + h
    const int c0 = lane * 4;
    const int br = merge_branch(warp);
    const int len = branch_len(a, br);
    int nslots = 0;
    if (len > 0) {
        const long long s0 = piece_begin(a, unit, br);
        const int tpw = phase_tpw(a, br);
        nslots = (int)((s0 + len - 1) / tpw - s0 / tpw) + 1;
    }
    const int sl0 = br == 0 ? warp : (br == 1 ? 0 : warp - 4), step = br == 0 ? 3 : (br == 1 ? 1 : 4);
    const float* base = a.rec + ((size_t)unit * 3 + br) * a.maxw * a.G * rec_floats(D) + (size_t)h * rec_floats(D);
    const size_t rs = (size_t)a.G * rec_floats(D);
    float M = -INFINITY, Lsum = 0.0f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sl = sl0; sl < nslots; sl += kMergeBatch * step) {
        float m[kMergeBatch], l[kMergeBatch];
        float4 o[kMergeBatch];
#pragma unroll
        for (int q = 0; q < kMergeBatch; ++q) {
            const int s = sl + q * step;
            m[q] = -INFINITY;
            l[q] = 0.0f;
            o[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s < nslots) {
                const float* rec = base + (size_t)s * rs;
                m[q] = __ldcg(rec);
                l[q] = __ldcg(rec + 1);
                if (c0 < D) o[q] = __ldcg(reinterpret_cast<const float4*>(rec + 4 + c0));
            }
        }
#pragma unroll
        for (int q = 0; q < kMergeBatch; ++q) {
            if (m[q] == -INFINITY) continue;
            const float nM = fmaxf(M, m[q]);
            const float fa = M == -INFINITY ? 0.0f : exp2f(M - nM);  // maxima are in log2 units
            const float fb = exp2f(m[q] - nM);
            Lsum = Lsum * fa + l[q] * fb;
            acc[0] = acc[0] * fa + o[q].x * fb;
            acc[1] = acc[1] * fa + o[q].y * fb;
            acc[2] = acc[2] * fa + o[q].z * fb;
            acc[3] = acc[3] * fa + o[q].w * fb;
            M = nM;
        }
    }
    if (lane == 0) {
        wM[warp] = M;
        wL[warp] = Lsum;
    }
    if (c0 < D)
        for (int j = 0; j < 4; ++j) wO[warp][c0 + j] = acc[j];
    __syncthreads();
    if (warp != 0 || c0 >= D) return;
    const float* gate = a.gates + (size_t)hq_row * 3;
    float out[4] = {0.f, 0.f, 0.f, 0.f};
    // branch results: SLC = warps 0-2, WIN = warp 3, CMP = warps 4-7
    for (int b2 = 0; b2 < 3; ++b2) {
        const int w0 = b2 == 0 ? 0 : (b2 == 1 ? 3 : 4), w1 = b2 == 0 ? 3 : (b2 == 1 ? 4 : kMergeWarps);
        float GM = -INFINITY;
        for (int w = w0; w < w1; ++w) GM = fmaxf(GM, wM[w]);
        if (GM == -INFINITY) continue;
        float GL = 0.0f, ob[4] = {0.f, 0.f, 0.f, 0.f};
        for (int w = w0; w < w1; ++w) {
            if (wM[w] == -INFINITY) continue;
            const float f = exp2f(wM[w] - GM);
            GL += wL[w] * f;
            for (int j = 0; j < 4; ++j) ob[j] += wO[w][c0 + j] * f;
        }
        if (!(GL > 0.0f)) continue;
        const float gw = gate[b2 == 0 ? 1 : (b2 == 1 ? 2 : 0)] / GL;  // gates are (cmp, slc, win)
        for (int j = 0; j < 4; ++j) out[j] += gw * ob[j];
    }
    __nv_bfloat16* o = a.O + (size_t)hq_row * D + c0;
    for (int j = 0; j < 4; ++j) o[j] = __float2bfloat16_rn(out[j]);
}

StreamArgs make_stream_args(const Dims& m) {
    StreamArgs a{};
    a.Hq = m.Hq; a.Hkv = m.Hkv; a.G = m.G; a.T = m.T; a.L = m.L; a.k = m.k; a.W = m.W; a.nB = m.nB; a.nC = m.nC;
    a.tS = m.k * (m.L / kTK);
    a.tW = (std::min(m.W, m.T) + kTK - 1) / kTK;
    a.tC = (m.nC + kTK - 1) / kTK;
    a.tAu = a.tW + a.tC;
    a.nA = (long long)m.units() * a.tAu;
    a.nBt = (long long)m.units() * a.tS;
    const long long warps_wanted = (long long)sm_count() * kWarps;
    a.tpwA = (int)std::max<long long>(1, (a.nA + warps_wanted - 1) / warps_wanted);
    a.tpwB = (int)std::max<long long>(1, (a.nBt + warps_wanted - 1) / warps_wanted);
    // pieces of one (unit, branch): at most len / tpw + 2 warps meet its tiles
    a.maxw = std::max(a.tS / a.tpwB, std::max(a.tW, a.tC) / a.tpwA) + 2;
    a.sl2 = 1.4426950408889634f / sqrtf((float)m.d);
    return a;
}

template <int D>
size_t stream_smem() { return (size_t)kWarps * kStages * 2 * (D / 64) * kTK * 128 + 1024; }

template <int D>
cudaError_t launch_stream_d(const Dims& m, StreamArgs a, const void* K, const void* V, const void* Kc, const void* Vc,
                            bool after_select, cudaStream_t s) {
    CUtensorMap tk, tv, tkc, tvc;
    const uint64_t kvrows = (uint64_t)m.units() * m.T;
    const uint64_t crows = m.nC > 0 ? (uint64_t)m.units() * m.nC : kvrows;
    if (!encode_tmap_bf16_2d(&tk, K, kvrows, D, kTK) || !encode_tmap_bf16_2d(&tv, V, kvrows, D, kTK) ||
        !encode_tmap_bf16_2d(&tkc, m.nC > 0 ? Kc : K, crows, D, kTK) ||
        !encode_tmap_bf16_2d(&tvc, m.nC > 0 ? Vc : V, crows, D, kTK))
        return cudaErrorInvalidValue;
    const size_t smem = stream_smem<D>();
    cudaError_t e = cudaFuncSetAttribute(decode_stream_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nwarps = std::max((a.nA + a.tpwA - 1) / a.tpwA, (a.nBt + a.tpwB - 1) / a.tpwB);
    const int grid = (int)((nwarps + kWarps - 1) / kWarps);
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kWarps * 32);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = after_select ? 1 : 0;  // else: after whatever precedes it, in stream order
        count_launch();
        e = cudaLaunchKernelEx(&cfg, decode_stream_kernel<D>, tk, tv, tkc, tvc, a);
        if (e != cudaSuccess) return e;
    }
    // the merge grid may launch while the decode grid drains; it waits for it on the device
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(m.G, m.units());
    cfg.blockDim = dim3(kMergeWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, decode_stream_merge<D>, a);
}

}  // namespace

size_t decode_stream_workspace_bytes(const Dims& m) {
    const StreamArgs a = make_stream_args(m);
    return (size_t)m.units() * 3 * a.maxw * m.G * rec_floats(m.d) * sizeof(float);
}

cudaError_t launch_decode_stream(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                                 const void* Vc, const int32_t* idx, const float* gates, void* O, void* ws,
                                 bool after_select, cudaStream_t s, int* err) {
    StreamArgs a = make_stream_args(m);
    a.Q = static_cast<const __nv_bfloat16*>(Q);
    a.idx = idx;
    a.gates = gates;
    a.O = static_cast<__nv_bfloat16*>(O);
    a.rec = static_cast<float*>(ws);
    a.err = err;
    a.lazy = after_select ? 1 : 0;
    return m.d == 128 ? launch_stream_d<128>(m, a, K, V, Kc, Vc, after_select, s)
                      : launch_stream_d<64>(m, a, K, V, Kc, Vc, after_select, s);
}

}  // namespace cobs
