// Building blocks of the bf16 decode attention kernels: one warp computes the G <= 16 query
// heads of a (batch, KV-head) unit against a tile of 32 keys held in shared memory (K and V,
// 2-D TMA boxes of 64 columns with the 128-byte swizzle), as mma.sync m16n8k16 tiles with an
// online softmax in registers.
//
// Attention of the NSA paths (Janus issue #181: compression, selection, sliding window), each
// branch a softmax(q K^T / sqrt(d)) V of its own; COBS (gist.science explainer §2.3) changes
// only which blocks the selection path reads.
#pragma once

#include <math.h>

#include "common.cuh"

namespace cobs {

#ifndef COBS_DECODE_TK
#define COBS_DECODE_TK 32
#endif
constexpr int kTK = COBS_DECODE_TK;  // keys per tile (16 or 32)
static_assert(kTK == 16 || kTK == 32, "tile of 16 or 32 keys");

template <int D>
struct WState {
    float m0, m1, l0, l1;  // reference maxima (scaled log2 units) and row sums
    float o[D / 8][4];
    __device__ void init() {
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.0f;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    }
};

template <int D>
__device__ __forceinline__ void load_q(const __nv_bfloat16* q, int G, uint32_t (&qa)[D / 16][4], int lane) {
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

// 2^x on the special-function unit (approximate, flush-to-zero).
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Byte offset of 16-byte chunk `cc` (0..7) of row `r` in a 128-byte-swizzled 32-row box.
__device__ __forceinline__ uint32_t swz(int r, int cc) { return (uint32_t)(r * 128 + ((cc ^ (r & 7)) << 4)); }

// Byte offset of chunk `cc` of 64-column half `h` of row `r` in a K or V tile: with IL the two
// halves of a row are adjacent 128-byte segments (one 3-D box of [rows][2][64] columns), else
// each half is its own box of TK rows; both with the 128-byte swizzle of the segment index.
template <int TK, bool IL>
__device__ __forceinline__ uint32_t tile_off(int r, int h, int cc) {
    if (IL) {
        const int seg = 2 * r + h;
        return (uint32_t)(seg * 128 + ((cc ^ (seg & 7)) << 4));
    }
    return (uint32_t)(h * TK * 128) + swz(r, cc);
}

// One tile: S = Q K^T over TK keys, online softmax update, O += P V.
template <int D, int TK = kTK, bool IL = false>
__device__ __forceinline__ void tile_mma(WState<D>& st, const uint32_t (&qa)[D / 16][4], const unsigned char* sK,
                                         const unsigned char* sV, uint32_t vm, float sl2, int lane) {
    static_assert(TK == 16 || TK == 32, "tile of 16 or 32 keys");
    constexpr int NP = TK / 16;       // 16-key groups
    const int mi = lane >> 3;
    float s[2 * NP][4];
#pragma unroll
    for (int nt = 0; nt < 2 * NP; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < NP; ++np) {
            const int r = np * 16 + (lane & 7) + ((mi >> 1) << 3);
            const int cc = (ks & 3) * 2 + (mi & 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, sK + tile_off<TK, IL>(r, ks >> 2, cc));
            mma_bf16_16816(s[2 * np], qa[ks], b0, b1);
            mma_bf16_16816(s[2 * np + 1], qa[ks], b2, b3);
        }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2 * NP; ++nt) {
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
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 2));
    // Lazy rescale: the reference maxima st.m* (scaled log2 units) move only when a row's maximum
    // exceeds them by more than 8, so p = 2^(s sl2 - m) <= 2^8 and the accumulators are rescaled
    // rarely. The four threads of a quad hold the same row maxima and decide alike.
    mx0 *= sl2;
    mx1 *= sl2;
    const bool g0 = mx0 != -INFINITY && (st.m0 == -INFINITY || mx0 - st.m0 > 8.0f);
    const bool g1 = mx1 != -INFINITY && (st.m1 == -INFINITY || mx1 - st.m1 > 8.0f);
    if (__any_sync(kFull, g0 || g1)) {
        const float nm0 = g0 ? (st.m0 == -INFINITY ? mx0 : fmaxf(st.m0, mx0)) : st.m0;
        const float nm1 = g1 ? (st.m1 == -INFINITY ? mx1 : fmaxf(st.m1, mx1)) : st.m1;
        const float al0 = (g0 && st.m0 != -INFINITY) ? ex2f(st.m0 - nm0) : (g0 ? 0.0f : 1.0f);
        const float al1 = (g1 && st.m1 != -INFINITY) ? ex2f(st.m1 - nm1) : (g1 ? 0.0f : 1.0f);
        st.m0 = nm0;
        st.m1 = nm1;
        st.l0 *= al0;
        st.l1 *= al1;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) {
            st.o[nd][0] *= al0;
            st.o[nd][1] *= al0;
            st.o[nd][2] *= al1;
            st.o[nd][3] *= al1;
        }
    }
    const float nm0 = -st.m0, nm1 = -st.m1;
    const bool z0 = st.m0 == -INFINITY, z1 = st.m1 == -INFINITY;
    float ps0 = 0.0f, ps1 = 0.0f;
    uint32_t pa[NP][4];
#pragma unroll
    for (int nt = 0; nt < 2 * NP; ++nt) {
        const float p0 = z0 ? 0.0f : ex2f(fmaf(s[nt][0], sl2, nm0));
        const float p1 = z0 ? 0.0f : ex2f(fmaf(s[nt][1], sl2, nm0));
        const float p2 = z1 ? 0.0f : ex2f(fmaf(s[nt][2], sl2, nm1));
        const float p3 = z1 ? 0.0f : ex2f(fmaf(s[nt][3], sl2, nm1));
        ps0 += p0 + p1;
        ps1 += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
    st.l0 += ps0;
    st.l1 += ps1;
#pragma unroll
    for (int kk = 0; kk < NP; ++kk) {
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
            const int r = kk * 16 + (lane & 7) + ((mi & 1) << 3);
            const int cc = (np & 3) * 2 + (mi >> 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(b0, b1, b2, b3, sV + tile_off<TK, IL>(r, np >> 2, cc));
            mma_bf16_16816(st.o[2 * np], pa[kk], b0, b1);
            mma_bf16_16816(st.o[2 * np + 1], pa[kk], b2, b3);
        }
    }
}

// ----------------------------------------------------------------------------- keys as rows
// The same tile computed transposed, for groups of at most 8 heads: S^T = K Q^T with the keys as
// the 16 rows of each mma and the heads as its 8 columns, then O^T += V^T P^T with the head
// dimension as the rows. Half the mma and softmax work of the head-rows form at G <= 8, and half
// its accumulator registers. Thread t holds heads h0 = 2 (t % 4) and h0 + 1.
template <int D>
struct WStateT {
    float m[2], l[2];      // per held head: reference maximum (scaled log2 units), partial row sum
    float o[D / 16][4];    // O^T tile mt: (d mt 16 + t / 4, h0), (.., h0 + 1), (d + 8, h0), (d + 8, h0 + 1)
    __device__ void init() {
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.0f;
#pragma unroll
        for (int i = 0; i < D / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    }
};

// Q^T as the B operand of the score mma: for each 16-channel slice ks, thread t holds
// (q[t/4][ks 16 + 2 (t%4)], +1) and (.. + 8, + 9); heads >= G are zero.
template <int D>
__device__ __forceinline__ void load_qt(const __nv_bfloat16* q, int G, uint32_t (&qb)[D / 16][2], int lane) {
    const int h = lane >> 2, c = 2 * (lane & 3);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t* qr = reinterpret_cast<const uint32_t*>(q + (size_t)h * D + ks * 16 + c);
        qb[ks][0] = h < G ? qr[0] : 0u;
        qb[ks][1] = h < G ? qr[4] : 0u;
    }
}

template <int D, int TK, bool IL>
__device__ __forceinline__ void tile_mma_t(WStateT<D>& st, const uint32_t (&qb)[D / 16][2], const unsigned char* sK,
                                           const unsigned char* sV, uint32_t vm, float sl2, int lane) {
    static_assert(TK == 16 || TK == 32, "tile of 16 or 32 keys");
    constexpr int NP = TK / 16;  // 16-key row blocks
    const int mi = lane >> 3, g = lane >> 2;
    float s[NP][4];
#pragma unroll
    for (int p = 0; p < NP; ++p) s[p][0] = s[p][1] = s[p][2] = s[p][3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            // A = keys p 16 .. + 15 x channels ks 16 .. + 15 (row-major K)
            const int r = p * 16 + (lane & 7) + ((mi & 1) << 3);
            const int cc = (ks & 3) * 2 + (mi >> 1);
            uint32_t ak[4];
            ldmatrix_x4(ak[0], ak[1], ak[2], ak[3], sK + tile_off<TK, IL>(r, ks >> 2, cc));
            mma_bf16_16816(s[p], ak, qb[ks][0], qb[ks][1]);
        }
    }
    // mask invalid keys (row of c0/c1: key p 16 + g, of c2/c3: + 8); row maxima per held head
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const bool ok0 = (vm >> (p * 16 + g)) & 1u, ok1 = (vm >> (p * 16 + g + 8)) & 1u;
        s[p][0] = ok0 ? s[p][0] : -INFINITY;
        s[p][1] = ok0 ? s[p][1] : -INFINITY;
        s[p][2] = ok1 ? s[p][2] : -INFINITY;
        s[p][3] = ok1 ? s[p][3] : -INFINITY;
        mx0 = fmaxf(mx0, fmaxf(s[p][0], s[p][2]));
        mx1 = fmaxf(mx1, fmaxf(s[p][1], s[p][3]));
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
    }
    // lazy rescale: the reference maxima move only when a head's maximum exceeds them by more than
    // 8 (so p <= 2^8); the eight threads holding a head decide alike
    mx0 *= sl2;
    mx1 *= sl2;
    const bool g0 = mx0 != -INFINITY && (st.m[0] == -INFINITY || mx0 - st.m[0] > 8.0f);
    const bool g1 = mx1 != -INFINITY && (st.m[1] == -INFINITY || mx1 - st.m[1] > 8.0f);
    if (__any_sync(kFull, g0 || g1)) {
        const float nm0 = g0 ? (st.m[0] == -INFINITY ? mx0 : fmaxf(st.m[0], mx0)) : st.m[0];
        const float nm1 = g1 ? (st.m[1] == -INFINITY ? mx1 : fmaxf(st.m[1], mx1)) : st.m[1];
        const float al0 = (g0 && st.m[0] != -INFINITY) ? ex2f(st.m[0] - nm0) : (g0 ? 0.0f : 1.0f);
        const float al1 = (g1 && st.m[1] != -INFINITY) ? ex2f(st.m[1] - nm1) : (g1 ? 0.0f : 1.0f);
        st.m[0] = nm0;
        st.m[1] = nm1;
        st.l[0] *= al0;
        st.l[1] *= al1;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            st.o[mt][0] *= al0;
            st.o[mt][1] *= al1;
            st.o[mt][2] *= al0;
            st.o[mt][3] *= al1;
        }
    }
    const float nm0 = -st.m[0], nm1 = -st.m[1];
    const bool z0 = st.m[0] == -INFINITY, z1 = st.m[1] == -INFINITY;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const float p0 = z0 ? 0.0f : ex2f(fmaf(s[p][0], sl2, nm0));
        const float p1 = z1 ? 0.0f : ex2f(fmaf(s[p][1], sl2, nm1));
        const float p2 = z0 ? 0.0f : ex2f(fmaf(s[p][2], sl2, nm0));
        const float p3 = z1 ? 0.0f : ex2f(fmaf(s[p][3], sl2, nm1));
        st.l[0] += p0 + p2;
        st.l[1] += p1 + p3;
        // P^T of keys p 16 .. + 15 as the B operand: the two 8 x 8 blocks transposed in registers
        const uint32_t b0 = movmatrix_trans(pack_bf16(p0, p1));
        const uint32_t b1 = movmatrix_trans(pack_bf16(p2, p3));
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            // A = V^T: channels mt 16 .. + 15 x keys p 16 .. + 15 (transposed loads of row-major V)
            const int r = p * 16 + (lane & 7) + ((mi >> 1) << 3);
            const int cc = (mt & 3) * 2 + (mi & 1);
            uint32_t av[4];
            ldmatrix_x4_trans(av[0], av[1], av[2], av[3], sV + tile_off<TK, IL>(r, mt >> 2, cc));
            mma_bf16_16816(st.o[mt], av, b0, b1);
        }
    }
}

}  // namespace cobs
