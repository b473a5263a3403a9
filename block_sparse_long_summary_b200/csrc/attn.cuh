// Shared pieces of the decode and prefill attention kernels: which keys a branch chunk
// covers, staging a chunk into shared memory with bulk (TMA) copies, and the warp-level
// tensor-core (bf16) and CUDA-core (float32) online-softmax updates.
//
// Branches (NSA paths, Janus issue #181; kept by COBS, gist.science explainer §2.3):
//   SLC  tokens of the selected blocks idx (entries -1 skipped)
//   WIN  tokens max(0, t-W+1) .. t
//   CMP  compressed tokens i with cmp_stride*i + cmp_block - 1 <= t
// each with its own softmax(q k^T / sqrt(d)); outputs mixed by the gates (g_cmp, g_slc, g_win).
#pragma once

#include "common.cuh"

namespace cobs {

enum Branch : int { kSLC = 0, kWIN = 1, kCMP = 2 };
// gate slot of each branch in the (g_cmp, g_slc, g_win) triple
__host__ __device__ __forceinline__ int gate_slot(int br) { return br == kSLC ? 1 : (br == kWIN ? 2 : 0); }

struct AttnArgs {
    const void* Q;
    const void* K;
    const void* V;
    const void* Kc;
    const void* Vc;
    const int32_t* idx;
    const float* gates;
    void* O;
    float* part;     // decode partials
    int* err;
    int B, Hq, Hkv, G, T, L, lc, sc, k, W, nB, nC;
    int Tq;          // query positions per batch row: 1 (decode) or T (prefill)
    int nS, nW, nCk, nchunks;  // decode chunk counts per unit
    float sl2;       // log2(e) / sqrt(d)
};

__device__ __forceinline__ int visible_compressed(const AttnArgs& a, int t) {
    if (t < a.lc - 1) return 0;
    return min(a.nC, (t - a.lc + 1) / a.sc + 1);
}

template <int CK>
__device__ __forceinline__ int branch_chunks(const AttnArgs& a, int br, int t) {
    if (br == kSLC) return (a.k + (CK / 64) - 1) / (CK / 64);
    if (br == kWIN) return (min(a.W, t + 1) + CK - 1) / CK;
    return (visible_compressed(a, t) + CK - 1) / CK;
}

// Source rows of slot `slot` of chunk `ch` of branch `br` for query position t of unit (b, g).
template <typename T, int D, int CK>
__device__ __forceinline__ bool resolve_slot(const AttnArgs& a, int unit, const int32_t* idx_row, int t, int br,
                                             int ch, int slot, const T*& ksrc, const T*& vsrc) {
    if (br == kSLC) {
        constexpr int CB = CK / 64;
        const int j = ch * CB + slot / 64;
        if (j >= a.k) return false;
        const int bi = idx_row[j];
        if (bi < 0) return false;
        if (bi >= (t + 1) / a.L) {  // not a complete block at or before t
            report_error(a.err, kErrBadIndex);
            return false;
        }
        const size_t row = (size_t)unit * a.T + (size_t)bi * a.L + (slot & 63);
        ksrc = static_cast<const T*>(a.K) + row * D;
        vsrc = static_cast<const T*>(a.V) + row * D;
        return true;
    }
    if (br == kWIN) {
        const int w0 = max(0, t - a.W + 1);
        const int r = w0 + ch * CK + slot;
        if (r > t) return false;
        const size_t row = (size_t)unit * a.T + r;
        ksrc = static_cast<const T*>(a.K) + row * D;
        vsrc = static_cast<const T*>(a.V) + row * D;
        return true;
    }
    const int ci = ch * CK + slot;
    if (ci >= visible_compressed(a, t)) return false;
    const size_t row = (size_t)unit * a.nC + ci;
    ksrc = static_cast<const T*>(a.Kc) + row * D;
    vsrc = static_cast<const T*>(a.Vc) + row * D;
    return true;
}

// Stage one chunk (CK rows of K and V, row stride D + 16/sizeof(T) elements) into smem.
// Must be called by all CK threads of the CTA. `phase` is the mbarrier parity of this use;
// the barrier completes a phase only when at least one slot is valid, which the return
// value reports (number of valid slots). Invalid slots are zero-filled. `ok` becomes false
// if the copies did not complete in time.
template <typename T, int D, int CK>
__device__ __forceinline__ int stage_chunk(const AttnArgs& a, int unit, const int32_t* idx_row, int t, int br,
                                           int ch, T* sK, T* sV, uint32_t* vmask, uint64_t* bar, uint32_t phase,
                                           bool& ok) {
    constexpr int RS = D + 16 / (int)sizeof(T);
    const int slot = threadIdx.x;
    const T* ks = nullptr;
    const T* vs = nullptr;
    const bool valid = resolve_slot<T, D, CK>(a, unit, idx_row, t, br, ch, slot, ks, vs);
    const unsigned bal = __ballot_sync(0xffffffffu, valid);
    if ((slot & 31) == 0) vmask[slot >> 5] = bal;
    const int nvalid = __syncthreads_count(valid);
    constexpr uint32_t kRowBytes = D * sizeof(T);
    if (slot == 0 && nvalid > 0) mbar_arrive_expect_tx(bar, (uint32_t)nvalid * 2 * kRowBytes);
    __syncthreads();
    if (valid) {
        bulk_g2s(sK + (size_t)slot * RS, ks, kRowBytes, bar);
        bulk_g2s(sV + (size_t)slot * RS, vs, kRowBytes, bar);
    } else {
        // zero the row so that p = 0 times the row stays 0
        uint4* kz = reinterpret_cast<uint4*>(sK + (size_t)slot * RS);
        uint4* vz = reinterpret_cast<uint4*>(sV + (size_t)slot * RS);
#pragma unroll
        for (int i = 0; i < (int)(kRowBytes / 16); ++i) {
            kz[i] = make_uint4(0, 0, 0, 0);
            vz[i] = make_uint4(0, 0, 0, 0);
        }
    }
    if (nvalid > 0 && !mbar_wait(bar, phase, a.err)) ok = false;
    ok = __syncthreads_and(ok) != 0;  // CTA-uniform, so no thread leaves a loop alone
    return nvalid;
}

// ------------------------------------------------------------------ bf16 tensor-core path
// One warp owns 32 consecutive key slots of the chunk and up to 16 query heads (rows of the
// m16 tile; rows >= G are zero). Per thread: rows r0 = lane/4 and r1 = r0 + 8.
template <int D>
struct WarpState {
    float m0, m1;       // running max (raw score units)
    float l0, l1;       // running sum of exp (this thread's columns only)
    float o[D / 8][4];  // unnormalised output accumulators
    __device__ void init() {
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.0f;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    }
};

// A fragments of the group's query heads (m16 x D, rows >= G zero).
template <int D>
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16* q, int G, uint32_t (&qa)[D / 16][4]) {
    const int lane = threadIdx.x & 31;
    const int r0 = lane >> 2, r1 = r0 + 8, c = 2 * (lane & 3);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t* q0 = reinterpret_cast<const uint32_t*>(q + (size_t)r0 * D + ks * 16 + c);
        const uint32_t* q1 = reinterpret_cast<const uint32_t*>(q + (size_t)r1 * D + ks * 16 + c);
        qa[ks][0] = r0 < G ? q0[0] : 0u;
        qa[ks][1] = r1 < G ? q1[0] : 0u;
        qa[ks][2] = r0 < G ? q0[4] : 0u;
        qa[ks][3] = r1 < G ? q1[4] : 0u;
    }
}

template <int D>
__device__ __forceinline__ void warp_chunk_mma(WarpState<D>& st, const uint32_t (&qa)[D / 16][4],
                                               const __nv_bfloat16* sK, const __nv_bfloat16* sV,
                                               const uint32_t* vmask, float sl2) {
    constexpr int RS = D + 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int key0 = warp * 32;
    const uint32_t vm = vmask[warp];
    if (vm == 0) return;  // no valid key in this warp's slots
    float s[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
    // S = Q K^T over the warp's 32 keys
    const int mi = lane >> 3;  // which 8x8 matrix this lane addresses
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            const int row = key0 + np * 16 + (lane & 7) + ((mi >> 1) << 3);
            const int col = ks * 16 + ((mi & 1) << 3);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, sK + (size_t)row * RS + col);
            mma_bf16_16816(s[2 * np], qa[ks], b0, b1);
            mma_bf16_16816(s[2 * np + 1], qa[ks], b2, b3);
        }
    }
    // mask invalid slots, row maxima
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int slot = nt * 8 + 2 * (lane & 3) + j;
            const bool ok = (vm >> slot) & 1u;
            s[nt][j] = ok ? s[nt][j] : -INFINITY;
            s[nt][2 + j] = ok ? s[nt][2 + j] : -INFINITY;
            mx0 = fmaxf(mx0, s[nt][j]);
            mx1 = fmaxf(mx1, s[nt][2 + j]);
        }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float nm0 = fmaxf(st.m0, mx0), nm1 = fmaxf(st.m1, mx1);
    // (a warp with at least one valid slot has finite maxima)
    const float al0 = exp2f((st.m0 - nm0) * sl2), al1 = exp2f((st.m1 - nm1) * sl2);
    st.m0 = nm0;
    st.m1 = nm1;
    float ps0 = 0.0f, ps1 = 0.0f;
    uint32_t pa[2][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const float p0 = exp2f((s[nt][0] - nm0) * sl2), p1 = exp2f((s[nt][1] - nm0) * sl2);
        const float p2 = exp2f((s[nt][2] - nm1) * sl2), p3 = exp2f((s[nt][3] - nm1) * sl2);
        ps0 += p0 + p1;
        ps1 += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
    st.l0 = st.l0 * al0 + ps0;
    st.l1 = st.l1 * al1 + ps1;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        st.o[nd][0] *= al0;
        st.o[nd][1] *= al0;
        st.o[nd][2] *= al1;
        st.o[nd][3] *= al1;
    }
    // O += P V over the warp's 32 keys (2 k-steps of 16)
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
            const int row = key0 + kk * 16 + (lane & 7) + ((mi & 1) << 3);
            const int col = np * 16 + ((mi >> 1) << 3);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(b0, b1, b2, b3, sV + (size_t)row * RS + col);
            mma_bf16_16816(st.o[2 * np], pa[kk], b0, b1);
            mma_bf16_16816(st.o[2 * np + 1], pa[kk], b2, b3);
        }
    }
}

// Combine the 4 warps' states of a CTA into one (m, l, o) per head row h < G:
// writes sm[h], sl[h] and so[h * D + c] (o relative to sm). `scratch` holds >= 4*16*D floats.
template <int D>
__device__ __forceinline__ void cta_combine(WarpState<D>& st, int G, float sl2, float* scratch, float* wm, float* wl,
                                            float* sm, float* sl, float* so) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r0 = lane >> 2, r1 = r0 + 8;
    float l0 = st.l0, l1 = st.l1;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if ((lane & 3) == 0) {
        wm[warp * 16 + r0] = st.m0;
        wm[warp * 16 + r1] = st.m1;
        wl[warp * 16 + r0] = l0;
        wl[warp * 16 + r1] = l1;
    }
    __syncthreads();
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        M0 = fmaxf(M0, wm[w * 16 + r0]);
        M1 = fmaxf(M1, wm[w * 16 + r1]);
    }
    const float f0 = st.m0 == -INFINITY ? 0.0f : exp2f((st.m0 - M0) * sl2);
    const float f1 = st.m1 == -INFINITY ? 0.0f : exp2f((st.m1 - M1) * sl2);
    float* mine = scratch + (size_t)warp * 16 * D;
    const int c = 2 * (lane & 3);
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        mine[r0 * D + nd * 8 + c] = st.o[nd][0] * f0;
        mine[r0 * D + nd * 8 + c + 1] = st.o[nd][1] * f0;
        mine[r1 * D + nd * 8 + c] = st.o[nd][2] * f1;
        mine[r1 * D + nd * 8 + c + 1] = st.o[nd][3] * f1;
    }
    __syncthreads();
    for (int h = threadIdx.x; h < G; h += blockDim.x) {
        float M = -INFINITY;
        for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * 16 + h]);
        float L = 0.0f;
        if (M != -INFINITY)
            for (int w = 0; w < 4; ++w)
                if (wm[w * 16 + h] != -INFINITY) L += wl[w * 16 + h] * exp2f((wm[w * 16 + h] - M) * sl2);
        sm[h] = M;
        sl[h] = L;
    }
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        so[e] = scratch[e] + scratch[16 * D + e] + scratch[2 * 16 * D + e] + scratch[3 * 16 * D + e];
    }
    __syncthreads();
}

}  // namespace cobs
