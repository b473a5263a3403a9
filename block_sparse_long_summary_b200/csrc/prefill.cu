// Causal prefill attention on the fifth-generation tensor cores (tcgen05 + TMEM), bf16, d = 128,
// GQA group of 16 query heads.
//
// What is computed (per position t and head h): the gated sum of three softmax attentions of
// NSA (Janus issue #181: compression, selection and sliding-window paths) with the blocks
// picked by the COBS selector (gist.science explainer §2.3) at that position.
//
// How: a CTA owns 8 consecutive positions of one GQA group, i.e. 8 x 16 = 128 query rows (row
// r = 16 p + h), the M of every MMA. It walks a list of 64-key items:
//   SLC  the union of the blocks selected by its 8 positions (a per-item 8-bit mask says which
//        positions selected it; the other rows are masked),
//   WIN  the 64-aligned key blocks covering the 8 windows,
//   CMP  the compressed-token blocks visible to its last position.
// Per item: S = Q K^T (M 128, N 64, K 128) into a TMEM buffer (two, alternating); the 128
// softmax threads (thread = row) read their S row, mask it, keep a per-branch running max
// (rescaling the branch accumulator only when the max grows by more than 2^8) and write P
// (bf16) into a swizzled shared-memory tile; then O_branch += P V (M 128, N 128, K 64), V being
// read MN-major. The three branch accumulators live in TMEM (3 x 128 columns); the epilogue
// divides by the row sums, applies the gates and writes bf16. A producer warp streams K/V
// tiles with TMA (no multicast) through a 3-stage ring; one thread issues all MMAs.
// Every wait on an mbarrier is bounded; a timeout sets the device error flag.
#include <algorithm>

#include "attn.cuh"
#include "dims.h"
#include "tc.cuh"
#include "tma.h"

namespace cobs {
namespace {

constexpr int kP = 8;            // positions per tile
constexpr int kGH = 16;          // query heads per group handled by this kernel
constexpr int kRows = kP * kGH;  // 128 MMA rows
constexpr int kKB = 64;          // keys per item
constexpr int kD = 128;          // head dimension handled by this kernel
constexpr int kStagesKV = 3;
constexpr int kSoftmaxThreads = 256;            // two threads per row: S / O column halves
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = kSoftmaxThreads + 64;  // + producer warp + MMA warp

constexpr uint32_t kQBytes = kRows * kD * 2;          // 32 KiB (two 64-column halves)
constexpr uint32_t kKVBox = kKB * 128;                 // 8 KiB: 64 rows x 64 columns
constexpr uint32_t kKVStage = 4 * kKVBox;              // K (2 halves) + V (2 halves) = 32 KiB
constexpr uint32_t kPBytes = kRows * kKB * 2;          // 16 KiB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 384, kColS1 = 448;         // S buffers; O_br at 128 * br

constexpr uint32_t kIdescS = tc::idesc_bf16(128, kKB, 0, 0);   // A = Q (K-major), B = K (K-major)
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, kD, 0, 1);   // A = P (K-major), B = V (MN-major)

struct PfArgs {
    const int32_t* idx;
    const float* gates;
    __nv_bfloat16* O;
    int* err;
    int Hq, Hkv, T, k, W, lc, sc, nB, nC;
    int max_items;
    float sl2;  // log2(e) / sqrt(d)
};

__device__ __forceinline__ void named_sync_softmax() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// warps w and w + 4 hold the two halves of the same 32 rows: barrier ids 2..5, 64 threads each
__device__ __forceinline__ void named_sync_pair(int w4) { asm volatile("bar.sync %0, 64;" ::"r"(2 + w4) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                 const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 const __grid_constant__ CUtensorMap tmKc,
                                                                 const __grid_constant__ CUtensorMap tmVc,
                                                                 PfArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t barQ, barKV[kStagesKV], barFree[kStagesKV], barS[2], barP[2], barO[2], barDone;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int n_sh[4];       // item counts: SLC, WIN, CMP, total
    __shared__ int warp_cnt[kThreads / 32];
    __shared__ float mx_sh[2][2][kRows];  // [item parity][half][row] row-max exchange

    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* sQ = base;                                  // 2 x 16 KiB
    unsigned char* sKV = base + kQBytes;                       // kStagesKV x 32 KiB
    unsigned char* sP = sKV + kStagesKV * kKVStage;            // 2 x 16 KiB
    int* item_row = reinterpret_cast<int*>(sP + 2 * kPBytes);  // [max_items]
    int* item_info = item_row + a.max_items;                   // br | (position mask << 8)
    uint32_t* selw = reinterpret_cast<uint32_t*>(item_info + a.max_items);  // [ceil(nB / 4)]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.y;
    const int b = unit / a.Hkv, g = unit % a.Hkv;
    const int t0 = blockIdx.x * kP;
    const int tlast = min(a.T - 1, t0 + kP - 1);
    const int ncand_max = (tlast + 1) / kKB;  // blocks any position of the tile may select

    // ---------------------------------------------------------------- set-up
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base_sh, kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&barQ, 1);
        for (int s = 0; s < kStagesKV; ++s) {
            mbar_init(&barKV[s], 1);
            mbar_init(&barFree[s], 1);
        }
        mbar_init(&barS[0], 1);
        mbar_init(&barS[1], 1);
        mbar_init(&barP[0], kSoftmaxThreads / 32);  // one arrival per softmax warp
        mbar_init(&barP[1], kSoftmaxThreads / 32);
        mbar_init(&barO[0], 1);
        mbar_init(&barO[1], 1);
        mbar_init(&barDone, 1);
        fence_barrier_init();
    }
    const int nwords = (ncand_max + 3) / 4;
    for (int i = tid; i < nwords; i += kThreads) selw[i] = 0u;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base_sh;

    // selected blocks of the tile's positions -> per-block position masks
    for (int e = tid; e < kP * a.k; e += kThreads) {
        const int p = e / a.k, j = e % a.k;
        const int t = t0 + p;
        if (t >= a.T) continue;
        const int bi = a.idx[(((size_t)b * a.T + t) * a.Hkv + g) * a.k + j];
        if (bi < 0) continue;
        if (bi >= (t + 1) / kKB) {
            report_error(a.err, kErrBadIndex);
            continue;
        }
        atomicOr(&selw[bi >> 2], (1u << p) << ((bi & 3) * 8));
    }
    __syncthreads();
    // compaction in ascending block order
    int nS = 0;
    for (int base_b = 0; base_b < ncand_max; base_b += kThreads) {
        const int bb = base_b + tid;
        const uint32_t msk = bb < ncand_max ? (selw[bb >> 2] >> ((bb & 3) * 8)) & 0xFFu : 0u;
        const unsigned bal = __ballot_sync(0xffffffffu, msk != 0u);
        if (lane == 0) warp_cnt[warp] = __popc(bal);
        __syncthreads();
        int off = nS;
        for (int w = 0; w < warp; ++w) off += warp_cnt[w];
        int tot = 0;
        for (int w = 0; w < kThreads / 32; ++w) tot += warp_cnt[w];
        if (msk != 0u) {
            const int pos = off + __popc(bal & ((1u << lane) - 1u));
            if (pos < a.max_items) {
                item_row[pos] = unit * a.T + bb * kKB;
                item_info[pos] = 0 | (int)(msk << 8);
            }
        }
        nS += tot;
        __syncthreads();
    }
    // window blocks and compressed-token blocks
    const int w_lo = max(0, t0 - a.W + 1);
    const int kb0 = w_lo / kKB, kb1 = tlast / kKB;
    const int nW = kb1 - kb0 + 1;
    const int ncv = tlast < a.lc - 1 ? 0 : min(a.nC, (tlast - a.lc + 1) / a.sc + 1);
    const int nCi = (ncv + kKB - 1) / kKB;
    const int n = min(a.max_items, nS + nW + nCi);
    for (int i = tid; i < nW + nCi; i += kThreads) {
        const int pos = nS + i;
        if (pos >= a.max_items) continue;
        if (i < nW) {
            item_row[pos] = unit * a.T + (kb0 + i) * kKB;
            item_info[pos] = 1;
        } else {
            item_row[pos] = unit * a.nC + (i - nW) * kKB;
            item_info[pos] = 2;
        }
    }
    if (tid == 0) {
        n_sh[0] = nS;
        n_sh[1] = nW;
        n_sh[2] = nCi;
        n_sh[3] = n;
        if (nS + nW + nCi > a.max_items) report_error(a.err, kErrBadIndex);
    }
    __syncthreads();

    // ---------------------------------------------------------------- producer warp
    if (warp == kProducerWarp) {
        if (lane == 0) {
            bool ok = true;
            mbar_arrive_expect_tx(&barQ, kQBytes);
            const int qz = b * a.T + t0;  // position coordinate (b, t)
            tma_load_3d(sQ, &tmQ, 0, g * kGH, qz, &barQ);
            tma_load_3d(sQ + kQBytes / 2, &tmQ, 64, g * kGH, qz, &barQ);
            for (int i = 0; i < n && ok; ++i) {
                const int s = i % kStagesKV;
                if (i >= kStagesKV) ok = mbar_wait(&barFree[s], ((i / kStagesKV) - 1) & 1, a.err);
                if (!ok) break;
                const int br = item_info[i] & 3;
                const int row = item_row[i];
                const CUtensorMap* mk = br == 2 ? &tmKc : &tmK;
                const CUtensorMap* mv = br == 2 ? &tmVc : &tmV;
                unsigned char* dst = sKV + (size_t)s * kKVStage;
                mbar_arrive_expect_tx(&barKV[s], kKVStage);
                tma_load_2d(dst, mk, 0, row, &barKV[s]);
                tma_load_2d(dst + kKVBox, mk, 64, row, &barKV[s]);
                tma_load_2d(dst + 2 * kKVBox, mv, 0, row, &barKV[s]);
                tma_load_2d(dst + 3 * kKVBox, mv, 64, row, &barKV[s]);
            }
            // stay until every MMA (and so every copy it consumed) has completed
            if (ok) mbar_wait(&barDone, 0, a.err);
        }
        return;
    }

    // ---------------------------------------------------------------- MMA warp (one thread issues)
    const uint32_t q_addr = smem_addr(sQ), kv_addr = smem_addr(sKV), p_addr = smem_addr(sP);
    const int first1 = nS, first2 = nS + nW;  // first item of the WIN and CMP branches
    if (warp == kMmaWarp) {
        if (lane == 0) {
            bool ok = mbar_wait(&barQ, 0, a.err);
            auto issue_pv = [&](int i) {
                // P_i and any rescale of O are ready
                if (ok) ok = mbar_wait(&barP[i & 1], (i >> 1) & 1, a.err);
                if (!ok) return;
                tc::fence_after_sync();
                const int br = item_info[i] & 3;
                const int fb = br == 0 ? 0 : (br == 1 ? first1 : first2);
                const int s_kv = i % kStagesKV;
                const uint32_t vbase = kv_addr + s_kv * kKVStage + 2 * kKVBox;
                const uint32_t pbase = p_addr + (i & 1) * kPBytes;
#pragma unroll
                for (int kk = 0; kk < kKB / 16; ++kk) {
                    const uint64_t ad = tc::smem_desc_sw128(pbase + kk * 32, 16, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(vbase + kk * 16 * 128, kKVBox, 1024);
                    tc::mma_f16_ss(tmem + br * 128, ad, bd, kIdescPV, (i > fb || kk > 0) ? 1u : 0u);
                }
                tc::commit(&barO[i & 1]);  // PV_i completes phase i / 2 of barO[i % 2]
                tc::commit(&barFree[s_kv]);
            };
            for (int i = 0; i < n && ok; ++i) {
                const int s = i % kStagesKV;
                ok = mbar_wait(&barKV[s], (i / kStagesKV) & 1, a.err);
                // S buffer i % 2 was read by softmax i - 2, which finished before signalling P_{i-2}
                if (ok && i >= 2) ok = mbar_wait(&barP[i & 1], ((i - 2) >> 1) & 1, a.err);
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t kbase = kv_addr + s * kKVStage;
                const uint32_t dS = tmem + ((i & 1) ? kColS1 : kColS0);
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint64_t ad = tc::smem_desc_sw128(q_addr + (ks >> 2) * (kQBytes / 2) + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(kbase + (ks >> 2) * kKVBox + (ks & 3) * 32, 16, 1024);
                    tc::mma_f16_ss(dS, ad, bd, kIdescS, ks > 0 ? 1u : 0u);
                }
                tc::commit(&barS[i & 1]);
                if (i >= 1) issue_pv(i - 1);
            }
            if (ok && n > 0) issue_pv(n - 1);
            // the issuing thread must outlive its MMAs: wait for all of them before leaving
            if (ok) {
                tc::commit(&barDone);
                mbar_wait(&barDone, 0, a.err);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- softmax warps (two threads per row)
    const int row = tid & (kRows - 1);   // TMEM lane / MMA row
    const int half = tid >> 7;           // S columns [32 half, +32), O columns [64 half, +64)
    const int p = row / kGH, h = row % kGH;
    const int t = t0 + p;
    const bool row_ok = t < a.T;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY;  // per-branch reference maxima (scaled log2 units)
    float l0 = 0.f, l1 = 0.f, l2 = 0.f;                     // per-branch partial row sums (this half)
    bool ok = true;
    // Wait until PV_j (and so every earlier MMA) has completed. PV_j completes phase j / 2 of
    // barO[j % 2]; that barrier cannot run a phase ahead of this wait (PV_{j+2} needs this
    // thread's P_{j+2}), so the parity names the phase unambiguously.
    auto wait_pv = [&](int j) {
        if (j >= 0 && ok && !mbar_wait(&barO[j & 1], (j >> 1) & 1, a.err)) ok = false;
    };
    const float sl2 = a.sl2;
    for (int i = 0; i < n; ++i) {
        const int br = item_info[i] & 3;
        const uint32_t pmask = ((uint32_t)item_info[i] >> 8) & 0xFFu;
        const int fb = br == 0 ? 0 : (br == 1 ? first1 : first2);
        float mref = br == 0 ? m0 : (br == 1 ? m1 : m2);
        float lsum = br == 0 ? l0 : (br == 1 ? l1 : l2);
        // key range [lo, hi] of this row within this thread's 32 keys of the item
        int lo = 0, hi = -1;
        const int rowi = item_row[i];
        if (row_ok) {
            if (br == 0) {
                if ((pmask >> p) & 1u) { lo = 0; hi = kKB - 1; }
            } else if (br == 1) {
                const int kbase = rowi - unit * a.T;
                lo = max(0, t - a.W + 1) - kbase;
                hi = t - kbase;
            } else {
                const int cbase = rowi - unit * a.nC;
                const int vis = t < a.lc - 1 ? 0 : min(a.nC, (t - a.lc + 1) / a.sc + 1);
                lo = 0;
                hi = vis - 1 - cbase;
            }
            lo = max(lo, 0) - 32 * half;
            hi = min(hi, kKB - 1) - 32 * half;
            lo = max(lo, 0);
            hi = min(hi, 31);
        }
        if (ok && !mbar_wait(&barS[i & 1], (i >> 1) & 1, a.err)) ok = false;
        tc::fence_after_sync();
        float s[32];
        tc::ld32(tmem + lane_off + ((i & 1) ? kColS1 : kColS0) + 32 * half, s);
        tc::wait_ld();
        const bool none = hi < lo;
        const bool full = lo == 0 && hi == 31;
        if (!full) {
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = (j >= lo && j <= hi) ? s[j] : -INFINITY;
        }
        // row maximum of the raw scores over both halves (the scale is positive)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 32; ++j) mx[j & 3] = fmaxf(mx[j & 3], s[j]);
        mx_sh[i & 1][half][row] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        named_sync_pair(warp & 3);  // this warp and the one holding the other half of its rows
        const float mt = fmaxf(mx_sh[i & 1][0][row], mx_sh[i & 1][1][row]) * sl2;
        // lazy rescale: only when the row maximum grows by more than 8 (a factor 2^8)
        float f = 1.0f;
        bool scale = false;
        if (mt != -INFINITY && (mref == -INFINITY || mt - mref > 8.0f)) {
            const float nm = mref == -INFINITY ? mt : fmaxf(mref, mt);
            if (mref != -INFINITY && i > fb) {
                f = tc::ex2(mref - nm);
                lsum *= f;
                scale = true;
            }
            mref = nm;
        }
        // O_br may be rescaled only after every earlier PV into it; P buffer i % 2 only after PV_{i-2}
        const bool wscale = __any_sync(0xffffffffu, scale);
        wait_pv(wscale ? i - 1 : i - 2);
        tc::fence_after_sync();
        if (wscale) {
#pragma unroll
            for (int c = 0; c < 64; c += 32) {
                float v[32];
                tc::ld32(tmem + lane_off + br * 128 + 64 * half + c, v);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= f;
                tc::st32(tmem + lane_off + br * 128 + 64 * half + c, v);
            }
            tc::wait_st();
        }
        // this half of the P row (bf16) into the swizzled tile P[i % 2]: chunks 4 half .. 4 half + 3;
        // p = 2^(s * scale - m), masked keys are -inf and give 0
        unsigned char* prow = sP + (size_t)(i & 1) * kPBytes + (size_t)row * 128;
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
        if (none || mref == -INFINITY) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(prow + (((4 * half + c) ^ (row & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        } else {
            const float neg = -mref;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t w4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = tc::ex2(fmaf(s[8 * c + 2 * q], sl2, neg));
                    const float x1 = tc::ex2(fmaf(s[8 * c + 2 * q + 1], sl2, neg));
                    ps[q] += x0 + x1;
                    w4[q] = pack_bf16(x0, x1);
                }
                *reinterpret_cast<uint4*>(prow + (((4 * half + c) ^ (row & 7)) << 4)) =
                    make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        }
        lsum += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        if (br == 0) { m0 = mref; l0 = lsum; } else if (br == 1) { m1 = mref; l1 = lsum; } else { m2 = mref; l2 = lsum; }
        // every lane's P stores and TMEM accesses are ordered before the warp's single arrival
        fence_proxy_async();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&barP[i & 1]);
    }
    // all MMAs done
    wait_pv(n - 1);
    tc::fence_after_sync();
    // full row sums: add the partner half's partial sums
    __shared__ float lsh[3][2][kRows];
    lsh[0][half][row] = l0;
    lsh[1][half][row] = l1;
    lsh[2][half][row] = l2;
    named_sync_softmax();
    const float lsum_br[3] = {lsh[0][0][row] + lsh[0][1][row], lsh[1][0][row] + lsh[1][1][row],
                              lsh[2][0][row] + lsh[2][1][row]};
    const int cnt[3] = {nS, nW, nCi};

    // ---------------------------------------------------------------- epilogue
    // Every lane of a warp executes the (warp-collective) TMEM loads; rows past T store nothing.
    {
        const size_t orow = ((size_t)b * a.T + (row_ok ? t : 0)) * a.Hq + (size_t)g * kGH + h;
        float wgt[3];
#pragma unroll
        for (int br = 0; br < 3; ++br) {
            const float gw = row_ok ? a.gates[orow * 3 + gate_slot(br)] : 0.0f;
            wgt[br] = (lsum_br[br] > 0.0f) ? gw / lsum_br[br] : 0.0f;
        }
        __nv_bfloat16* out = a.O + orow * kD + 64 * half;
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
            float acc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
#pragma unroll
            for (int br = 0; br < 3; ++br) {
                if (cnt[br] == 0) continue;  // uniform: no item of this branch in the tile
                float v[32];
                tc::ld32(tmem + lane_off + br * 128 + 64 * half + c, v);
                tc::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) acc[j] += wgt[br] * v[j];
            }
            if (row_ok) {
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    uint4 w;
                    w.x = pack_bf16(acc[j], acc[j + 1]);
                    w.y = pack_bf16(acc[j + 2], acc[j + 3]);
                    w.z = pack_bf16(acc[j + 4], acc[j + 5]);
                    w.w = pack_bf16(acc[j + 6], acc[j + 7]);
                    *reinterpret_cast<uint4*>(out + c + j) = w;
                }
            }
        }
    }
    tc::fence_before_sync();
    named_sync_softmax();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

// Handles bf16, d = 128, 16 query heads per group; returns cudaErrorNotSupported otherwise so that
// the caller uses the per-position kernel.
cudaError_t launch_prefill_tc(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                              const void* Vc, const int32_t* idx, const float* gates, void* O, cudaStream_t s,
                              int* err) {
    if (m.dtype != COBS_BF16 || m.d != kD || m.G != kGH || m.L != kKB) return cudaErrorNotSupported;
    PfArgs a{};
    a.idx = idx; a.gates = gates; a.O = static_cast<__nv_bfloat16*>(O); a.err = err;
    a.Hq = m.Hq; a.Hkv = m.Hkv; a.T = m.T; a.k = m.k; a.W = m.W; a.lc = m.lc; a.sc = m.sc; a.nB = m.nB;
    a.nC = m.nC;
    a.max_items = kP * m.k + (m.W + kP) / kKB + 2 + (m.nC + kKB - 1) / kKB + 1;
    a.sl2 = 1.4426950408889634f / sqrtf((float)m.d);
    const size_t smem = 1024 + kQBytes + (size_t)kStagesKV * kKVStage + 2 * kPBytes +
                        (size_t)2 * a.max_items * sizeof(int) + (size_t)((m.nB + 3) / 4 + 1) * sizeof(uint32_t);
    if (smem > 227 * 1024) return cudaErrorNotSupported;
    CUtensorMap tq, tk, tv, tkc, tvc;
    const uint64_t qd[3] = {(uint64_t)kD, (uint64_t)m.Hq, (uint64_t)m.B * m.T};
    const uint64_t qs[2] = {(uint64_t)kD * 2, (uint64_t)m.Hq * kD * 2};
    const uint32_t qb[3] = {64, (uint32_t)kGH, (uint32_t)kP};
    const uint64_t kvrows = (uint64_t)m.units() * m.T;
    const uint64_t crows = m.nC > 0 ? (uint64_t)m.units() * m.nC : kvrows;
    if (!encode_tmap_bf16_3d(&tq, Q, qd, qs, qb) || !encode_tmap_bf16_2d(&tk, K, kvrows, kD, kKB) ||
        !encode_tmap_bf16_2d(&tv, V, kvrows, kD, kKB) || !encode_tmap_bf16_2d(&tkc, m.nC > 0 ? Kc : K, crows, kD, kKB) ||
        !encode_tmap_bf16_2d(&tvc, m.nC > 0 ? Vc : V, crows, kD, kKB))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    prefill_tc_kernel<<<dim3((m.T + kP - 1) / kP, m.units()), kThreads, smem, s>>>(tq, tk, tv, tkc, tvc, a);
    return cudaGetLastError();
}

}  // namespace cobs
