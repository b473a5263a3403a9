// Building blocks of the cumulant-order block selection shared by the selector kernels:
// the canonical float32 group query and score arithmetic, and warp-wide top-k lists.
//
// COBS (gist.science explainer) §2.3 "Second-Order Scoring": score_b = q.mean_b +
// 1/2 q^T Sigma_b q with the per-channel variance; one selection per GQA group ranks blocks
// by the sum of its heads' scores,
//   S_{g,b} = (sum_c Qsum_c mu_{b,c}) * isd + c2 * (sum_c Q2_c var_{b,c}),
// Qsum = sum_h q_h, Q2 = sum_h q_h^2, isd = RN(1/sqrt(d)), c2 = RN(alpha/(2d)); skill card
// "Implementation steps" 3: keep the top-k blocks (score descending, ties to the lower index).
// Every sum runs in a fixed float32 order with one correctly rounded operation per step, so the
// selected indices are reproducible bit for bit.
#pragma once

#include <math.h>

#include "common.cuh"

namespace cobs {

constexpr int kInvalid = 0x7fffffff;
constexpr int kGroupBlocks = 32;

__device__ __forceinline__ bool better(float s1, int i1, float s2, int i2) {
    return s1 > s2 || (s1 == s2 && i1 < i2);
}

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

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Largest GQA group (query heads per KV head) the selectors handle; the host rejects larger.
constexpr int kMaxGroup = 16;

// NC consecutive elements (16-, 8- or 4-byte aligned vector loads) as float.
template <typename T, int NC>
__device__ __forceinline__ void load_chunk(const T* p, float (&x)[NC]) {
    if constexpr (sizeof(T) == 2) {
        static_assert(NC == 2 || NC == 4 || NC == 8, "chunk");
        uint32_t w[NC / 2];
        if constexpr (NC == 8) {
            const uint4 u = *reinterpret_cast<const uint4*>(p);
            w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
        } else if constexpr (NC == 4) {
            const uint2 u = *reinterpret_cast<const uint2*>(p);
            w[0] = u.x; w[1] = u.y;
        } else {
            w[0] = *reinterpret_cast<const uint32_t*>(p);
        }
#pragma unroll
        for (int i = 0; i < NC / 2; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
        static_assert(NC % 2 == 0, "chunk");
#pragma unroll
        for (int i = 0; i < NC; i += (NC % 4 == 0 ? 4 : 2)) {
            if constexpr (NC % 4 == 0) {
                const float4 v = *reinterpret_cast<const float4*>(p + i);
                x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2*>(p + i);
                x[i] = v.x; x[i + 1] = v.y;
            }
        }
    }
}

// Canonical group query of channels [c0, c0 + NC) of a group whose G head rows start at q
// (row stride D): every head's chunk is loaded at once, then Qsum_c = sum_h q_{h,c} (adds)
// and Q2_c = fma-sum of q_{h,c}^2 in ascending h.
template <typename T, int NC>
__device__ __forceinline__ void group_query_chunk(const T* q, int G, int D, int c0, bool valid, float* qs,
                                                  float* q2) {
    float x[kMaxGroup][NC];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        if (h < G && valid) {
            load_chunk<T, NC>(q + (size_t)h * D + c0, x[h]);
        } else {
#pragma unroll
            for (int j = 0; j < NC; ++j) x[h][j] = 0.0f;
        }
    }
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        float s = 0.0f, s2 = 0.0f;
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h < G) {
                s = __fadd_rn(s, x[h][j]);
                s2 = __fmaf_rn(x[h][j], x[h][j], s2);
            }
        }
        qs[j] = s;
        q2[j] = s2;
    }
}

// Canonical channel sums: four interleaved partial chains (chain j takes the channels
// c = j (mod 4) in ascending order from +0, one rounded fma per term), combined as
// (s0 + s1) + (s2 + s3). Lane = block; a group tile keeps four consecutive channels of a block
// in one 16-byte word, so one load feeds the four chains.
__device__ __forceinline__ float combine4(float s0, float s1, float s2, float s3) {
    return __fadd_rn(__fadd_rn(s0, s1), __fadd_rn(s2, s3));
}


// Q2tot = sum_c Q2_c by adds in ascending channel order from +0 (one thread).
template <int D>
__device__ __forceinline__ float q2_total(const float* q2) {
    float t = 0.0f;
    for (int c = 0; c < D; ++c) t = __fadd_rn(t, q2[c]);
    return t;
}

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


// Running best-first list of one warp (lane j = j-th best), with the k-th best as the bar
// a newcomer must beat. Groups with no lane above the bar cost one ballot.
struct RunList {
    float s;
    int i;
    float ts;
    int ti;
    __device__ void init() {
        s = -INFINITY;
        i = kInvalid;
        ts = -INFINITY;
        ti = kInvalid;
    }
    __device__ void bar(int k) {
        ts = __shfl_sync(kFull, s, k - 1);
        ti = __shfl_sync(kFull, i, k - 1);
    }
    // one candidate per lane (invalid lanes carry (-inf, kInvalid))
    __device__ void add(float sc, int bi, int k, int lane) {
        const unsigned up = __ballot_sync(kFull, bi != kInvalid && better(sc, bi, ts, ti));
        if (up == 0u) return;
        warp_sort_best_first(sc, bi, lane);
        warp_merge_best_first(s, i, sc, bi, lane);
        bar(k);
    }
};

// Continue the four canonical chains over NC4 consecutive channel quads: chain j adds
// fma(q_c, x_c, .) for the channels c = j (mod 4) in ascending order. x: [NC4][32][4]
// channel-interleaved values of the group's 32 blocks (lane = block); q: the NC4 * 4 matching
// query values. Feeding a group's channel quads in ascending order, in one call or several,
// gives the same chains.
template <int NC4>
__device__ __forceinline__ void score_chains(const float* x, const float* q, int lane, float (&c)[4]) {
    const float4* x4 = reinterpret_cast<const float4*>(x) + lane;
#pragma unroll 8
    for (int c4 = 0; c4 < NC4; ++c4) {
        const float4 m = x4[c4 * 32];
        const float4 qq = reinterpret_cast<const float4*>(q)[c4];
        c[0] = __fmaf_rn(qq.x, m.x, c[0]);
        c[1] = __fmaf_rn(qq.y, m.y, c[1]);
        c[2] = __fmaf_rn(qq.z, m.z, c[2]);
        c[3] = __fmaf_rn(qq.w, m.w, c[3]);
    }
}

// The mean half of the canonical score: a = (s0 + s1) + (s2 + s3), chain j summing
// fma(Qsum_c, mu_c, .) over the channels c = j (mod 4) in ascending order. mu: the group's
// [D/4][32][4] channel-interleaved means (lane = block).
template <int D>
__device__ __forceinline__ float score_mean_part(const float* mu, const float* qs, int lane) {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    score_chains<D / 4>(mu, qs, lane, c);
    return combine4(c[0], c[1], c[2], c[3]);
}

// The variance half: v = four-chain sum of fma(Q2_c, var_c, .) in the same order.
template <int D>
__device__ __forceinline__ float score_var_part(const float* var, const float* q2, int lane) {
    return score_mean_part<D>(var, q2, lane);
}

// S = fma(c2, v, a * isd).
__device__ __forceinline__ float score_combine(float a, float v, float isd, float c2) {
    return __fmaf_rn(c2, v, __fmul_rn(a, isd));
}

}  // namespace cobs
