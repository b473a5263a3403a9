// Decode attention at position T-1 for float32 (split-K over branch chunks, then a
// log-sum-exp merge that applies the gates; the bf16 path is decode_stream.cu), and the
// per-position prefill path (one CTA per position and group).
//
// NSA's three paths (Janus issue #181) — compression (CMP), selection (SLC), sliding
// window (WIN) — mixed by per-head gates; COBS (gist.science explainer, §2.3) changes only
// how SLC picks its blocks. Only the selected blocks, the window and the compressed tokens
// are read from HBM ("Problemstellung": decode is bound by KV-cache reads).
#include <algorithm>
#include <mutex>

#include "attn.cuh"
#include "dims.h"

namespace cobs {
namespace {

constexpr int kCK = 128;  // keys per chunk (bf16 path)
constexpr int kCKf = 64;  // keys per chunk (float32 path)

__host__ __device__ __forceinline__ int part_stride(int D) { return D + 4; }  // m, l, pad, pad, o[D]

// chunk id -> (branch, chunk within branch) for the decode enumeration SLC | WIN | CMP
__device__ __forceinline__ void decode_chunk(const AttnArgs& a, int id, int& br, int& ch) {
    if (id < a.nS) {
        br = kSLC;
        ch = id;
    } else if (id < a.nS + a.nW) {
        br = kWIN;
        ch = id - a.nS;
    } else {
        br = kCMP;
        ch = id - a.nS - a.nW;
    }
}

// ---------------------------------------------------------------- float32 chunk kernel (CUDA cores)
template <int D>
__global__ void __launch_bounds__(kCKf) decode_chunk_f32(AttnArgs a) {
    constexpr int RS = D + 4;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float* sK = reinterpret_cast<float*>(smem_raw);
    float* sV = sK + kCKf * RS;
    float* sq = sV + kCKf * RS;   // [16][D]
    float* sp = sq + 16 * D;      // [16][kCKf] scores / probabilities
    __shared__ uint32_t vmask[kCKf / 32];
    __shared__ float sm[16], sl[16];
    __shared__ __align__(8) uint64_t bar;

    const int unit = blockIdx.y;
    const int b = unit / a.Hkv, g = unit % a.Hkv;
    const int t = a.T - 1;
    const int G = a.G;
    int br, ch;
    decode_chunk(a, blockIdx.x, br, ch);
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    const float* q = static_cast<const float*>(a.Q) + ((size_t)b * a.Hq + (size_t)g * G) * D;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) sq[e] = q[e];
    const int32_t* idx_row = a.idx + (size_t)unit * a.k;
    bool ok = true;
    stage_chunk<float, D, kCKf>(a, unit, idx_row, t, br, ch, sK, sV, vmask, &bar, 0, ok);
    const float scale = 1.0f / sqrtf((float)D);
    // scores
    for (int e = threadIdx.x; e < G * kCKf; e += blockDim.x) {
        const int h = e / kCKf, s = e % kCKf;
        const bool valid = ok && ((vmask[s >> 5] >> (s & 31)) & 1u);
        float acc = 0.0f;
        for (int c = 0; c < D; ++c) acc = fmaf(sq[h * D + c], sK[s * RS + c], acc);
        sp[e] = valid ? acc * scale : -INFINITY;
    }
    __syncthreads();
    for (int h = threadIdx.x; h < G; h += blockDim.x) {
        float M = -INFINITY;
        for (int s = 0; s < kCKf; ++s) M = fmaxf(M, sp[h * kCKf + s]);
        float L = 0.0f;
        for (int s = 0; s < kCKf; ++s) {
            const float p = M == -INFINITY ? 0.0f : expf(sp[h * kCKf + s] - M);
            sp[h * kCKf + s] = p;
            L += p;
        }
        sm[h] = M;
        sl[h] = L;
    }
    __syncthreads();
    float* rec = a.part + ((size_t)unit * a.nchunks + blockIdx.x) * G * part_stride(D);
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, c = e % D;
        float acc = 0.0f;
        for (int s = 0; s < kCKf; ++s) acc = fmaf(sp[h * kCKf + s], sV[s * RS + c], acc);
        rec[h * part_stride(D) + 4 + c] = acc;
    }
    for (int h = threadIdx.x; h < G; h += blockDim.x) {
        // float32 path records natural-log maxima; the merge uses the same convention (ln2 scale)
        rec[h * part_stride(D) + 0] = sm[h];
        rec[h * part_stride(D) + 1] = sl[h];
    }
}

// ---------------------------------------------------------------- merge + gates
// grid (G, units), 4 warps: warps split the chunks of each branch, lanes split channels.
// mscale converts a recorded maximum difference to log2 units: sl2 for bf16 records
// (raw scores), log2(e) for float32 records (scaled scores).
template <typename T, int D>
__global__ void __launch_bounds__(128) decode_merge(AttnArgs a, float mscale) {
    __shared__ float wM[4], wL[4];
    __shared__ float wO[4][D];
    const int h = blockIdx.x, unit = blockIdx.y;
    const int b = unit / a.Hkv, g = unit % a.Hkv;
    const int hq = g * a.G + h;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* gate = a.gates + ((size_t)b * a.Hq + hq) * 3;
    float out[4] = {0.f, 0.f, 0.f, 0.f};
    const int c0 = lane * 4;
    const int ps = part_stride(D);
    const float* base = a.part + (size_t)unit * a.nchunks * a.G * ps;
    for (int br = 0; br < 3; ++br) {
        const int cs = br == kSLC ? 0 : (br == kWIN ? a.nS : a.nS + a.nW);
        const int ce = br == kSLC ? a.nS : (br == kWIN ? a.nS + a.nW : a.nchunks);
        float M = -INFINITY, L = 0.0f, acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int c = cs + warp; c < ce; c += 4) {
            const float* rec = base + ((size_t)c * a.G + h) * ps;
            const float m = __ldcg(rec), l = __ldcg(rec + 1);
            if (m == -INFINITY) continue;
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c0 < D) o = __ldcg(reinterpret_cast<const float4*>(rec + 4 + c0));
            const float nM = fmaxf(M, m);
            const float fa = M == -INFINITY ? 0.0f : exp2f((M - nM) * mscale);
            const float fb = exp2f((m - nM) * mscale);
            L = L * fa + l * fb;
            acc[0] = acc[0] * fa + o.x * fb;
            acc[1] = acc[1] * fa + o.y * fb;
            acc[2] = acc[2] * fa + o.z * fb;
            acc[3] = acc[3] * fa + o.w * fb;
            M = nM;
        }
        if (lane == 0) {
            wM[warp] = M;
            wL[warp] = L;
        }
        if (c0 < D) {
            wO[warp][c0 + 0] = acc[0];
            wO[warp][c0 + 1] = acc[1];
            wO[warp][c0 + 2] = acc[2];
            wO[warp][c0 + 3] = acc[3];
        }
        __syncthreads();
        if (warp == 0) {
            float GM = -INFINITY;
            for (int w = 0; w < 4; ++w) GM = fmaxf(GM, wM[w]);
            float GL = 0.0f, go[4] = {0.f, 0.f, 0.f, 0.f};
            if (GM != -INFINITY) {
                for (int w = 0; w < 4; ++w) {
                    if (wM[w] == -INFINITY) continue;
                    const float f = exp2f((wM[w] - GM) * mscale);
                    GL += wL[w] * f;
                    if (c0 < D)
                        for (int j = 0; j < 4; ++j) go[j] += wO[w][c0 + j] * f;
                }
            }
            const float gw = gate[gate_slot(br)];
            if (GL > 0.0f)
                for (int j = 0; j < 4; ++j) out[j] += gw * (go[j] / GL);
        }
        __syncthreads();
    }
    if (warp == 0 && c0 < D) {
        T* o = static_cast<T*>(a.O) + ((size_t)b * a.Hq + hq) * D + c0;
        for (int j = 0; j < 4; ++j) Elem<T>::store(o + j, out[j]);
    }
}

// ---------------------------------------------------------------- prefill (one CTA per position and group)
// grid (T, B * Hkv). Branches run one after another; within a branch the chunks are
// folded with an online softmax; the gated branch outputs accumulate in shared memory.
template <int D>
__global__ void __launch_bounds__(kCK) prefill_pos_bf16(AttnArgs a) {
    constexpr int RS = D + 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem_raw);
    __nv_bfloat16* sV = sK + kCK * RS;
    float* scratch = reinterpret_cast<float*>(smem_raw);       // [4][16][D], over sK/sV
    float* acc = reinterpret_cast<float*>(sV + kCK * RS);      // [16][D] gated output
    float* so = acc + 16 * D;                                   // [16][D]
    __shared__ uint32_t vmask[kCK / 32];
    __shared__ float wm[64], wl[64], sm[16], sl[16];
    __shared__ __align__(8) uint64_t bar;

    const int t = blockIdx.x;
    const int unit = blockIdx.y;
    const int b = unit / a.Hkv, g = unit % a.Hkv;
    const int G = a.G;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) acc[e] = 0.0f;
    const size_t qrow = ((size_t)b * a.T + t) * a.Hq + (size_t)g * G;
    uint32_t qa[D / 16][4];
    load_q_frags<D>(static_cast<const __nv_bfloat16*>(a.Q) + qrow * D, G, qa);
    const int32_t* idx_row = a.idx + (((size_t)b * a.T + t) * a.Hkv + g) * a.k;
    uint32_t phase = 0;
    bool ok = true;
    for (int br = 0; br < 3; ++br) {
        WarpState<D> st;
        st.init();
        const int nch = branch_chunks<kCK>(a, br, t);
        for (int ch = 0; ch < nch; ++ch) {
            if (!ok) break;
            if (stage_chunk<__nv_bfloat16, D, kCK>(a, unit, idx_row, t, br, ch, sK, sV, vmask, &bar, phase, ok) > 0)
                phase ^= 1u;
            if (ok) warp_chunk_mma<D>(st, qa, sK, sV, vmask, a.sl2);
            __syncthreads();
            fence_proxy_async();
        }
        cta_combine<D>(st, G, a.sl2, scratch, wm, wl, sm, sl, so);
        for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
            const int h = e / D;
            const float gw = a.gates[(qrow + h) * 3 + gate_slot(br)];
            if (sl[h] > 0.0f) acc[e] += gw * (so[e] / sl[h]);
        }
        __syncthreads();
    }
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.O) + qrow * D;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) o[e] = __float2bfloat16_rn(acc[e]);
}

template <int D>
__global__ void __launch_bounds__(kCKf) prefill_pos_f32(AttnArgs a) {
    constexpr int RS = D + 4;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float* sK = reinterpret_cast<float*>(smem_raw);
    float* sV = sK + kCKf * RS;
    float* sq = sV + kCKf * RS;   // [16][D]
    float* sp = sq + 16 * D;      // [16][kCKf]
    float* acc = sp + 16 * kCKf;  // [16][D] gated output
    float* ob = acc + 16 * D;     // [16][D] branch accumulator
    __shared__ uint32_t vmask[kCKf / 32];
    __shared__ float sM[16], sL[16], sF[16];
    __shared__ __align__(8) uint64_t bar;

    const int t = blockIdx.x;
    const int unit = blockIdx.y;
    const int b = unit / a.Hkv, g = unit % a.Hkv;
    const int G = a.G;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    const size_t qrow = ((size_t)b * a.T + t) * a.Hq + (size_t)g * G;
    const float* q = static_cast<const float*>(a.Q) + qrow * D;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        sq[e] = q[e];
        acc[e] = 0.0f;
    }
    const int32_t* idx_row = a.idx + (((size_t)b * a.T + t) * a.Hkv + g) * a.k;
    const float scale = 1.0f / sqrtf((float)D);
    uint32_t phase = 0;
    bool ok = true;
    for (int br = 0; br < 3; ++br) {
        for (int e = threadIdx.x; e < G * D; e += blockDim.x) ob[e] = 0.0f;
        for (int h = threadIdx.x; h < G; h += blockDim.x) {
            sM[h] = -INFINITY;
            sL[h] = 0.0f;
        }
        __syncthreads();
        const int nch = branch_chunks<kCKf>(a, br, t);
        for (int ch = 0; ch < nch; ++ch) {
            if (!ok) break;
            if (stage_chunk<float, D, kCKf>(a, unit, idx_row, t, br, ch, sK, sV, vmask, &bar, phase, ok) > 0)
                phase ^= 1u;
            for (int e = threadIdx.x; e < G * kCKf; e += blockDim.x) {
                const int h = e / kCKf, s = e % kCKf;
                const bool valid = ok && ((vmask[s >> 5] >> (s & 31)) & 1u);
                float x = 0.0f;
                for (int c = 0; c < D; ++c) x = fmaf(sq[h * D + c], sK[s * RS + c], x);
                sp[e] = valid ? x * scale : -INFINITY;
            }
            __syncthreads();
            for (int h = threadIdx.x; h < G; h += blockDim.x) {
                float M = sM[h];
                for (int s = 0; s < kCKf; ++s) M = fmaxf(M, sp[h * kCKf + s]);
                const float f = (sM[h] == -INFINITY) ? 0.0f : expf(sM[h] - M);
                float L = sL[h] * f;
                for (int s = 0; s < kCKf; ++s) {
                    const float p = M == -INFINITY ? 0.0f : expf(sp[h * kCKf + s] - M);
                    sp[h * kCKf + s] = p;
                    L += p;
                }
                sM[h] = M;
                sL[h] = L;
                sF[h] = f;
            }
            __syncthreads();
            for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
                const int h = e / D, c = e % D;
                float x = ob[e] * sF[h];
                for (int s = 0; s < kCKf; ++s) x = fmaf(sp[h * kCKf + s], sV[s * RS + c], x);
                ob[e] = x;
            }
            __syncthreads();
            fence_proxy_async();
        }
        for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
            const int h = e / D;
            const float gw = a.gates[(qrow + h) * 3 + gate_slot(br)];
            if (sL[h] > 0.0f) acc[e] += gw * (ob[e] / sL[h]);
        }
        __syncthreads();
    }
    float* o = static_cast<float*>(a.O) + qrow * D;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) o[e] = acc[e];
}

AttnArgs make_args(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc, const void* Vc,
                   const int32_t* idx, const float* gates, void* O, void* ws, int* err, int Tq, int CK) {
    AttnArgs a;
    a.Q = Q; a.K = K; a.V = V; a.Kc = Kc; a.Vc = Vc; a.idx = idx; a.gates = gates; a.O = O;
    a.part = static_cast<float*>(ws);
    a.err = err;
    a.B = m.B; a.Hq = m.Hq; a.Hkv = m.Hkv; a.G = m.G; a.T = m.T; a.L = m.L; a.lc = m.lc; a.sc = m.sc;
    a.k = m.k; a.W = m.W; a.nB = m.nB; a.nC = m.nC; a.Tq = Tq;
    const int t = m.T - 1;
    const int CB = CK / 64;
    a.nS = (m.k + CB - 1) / CB;
    a.nW = (std::min(m.W, t + 1) + CK - 1) / CK;
    const int ncv = t < m.lc - 1 ? 0 : std::min(m.nC, (t - m.lc + 1) / m.sc + 1);
    a.nCk = (ncv + CK - 1) / CK;
    a.nchunks = a.nS + a.nW + a.nCk;
    a.sl2 = 1.4426950408889634f / sqrtf((float)m.d);
    return a;
}

template <int D>
size_t decode_smem_f32() { return (size_t)2 * kCKf * (D + 4) * 4 + (size_t)16 * D * 4 + (size_t)16 * kCKf * 4; }

template <int D>
cudaError_t launch_decode_d(const Dims& m, AttnArgs a, cudaStream_t s) {
    const dim3 grid(a.nchunks, m.units());
    const size_t smem = decode_smem_f32<D>();
    cudaError_t e = cudaFuncSetAttribute(decode_chunk_f32<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    decode_chunk_f32<D><<<grid, kCKf, smem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch();
    decode_merge<float, D><<<dim3(m.G, m.units()), 128, 0, s>>>(a, 1.4426950408889634f);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_prefill_d(const Dims& m, AttnArgs a, cudaStream_t s) {
    const dim3 grid(m.T, m.units());
    cudaError_t e;
    if (m.dtype == COBS_BF16) {
        const size_t smem = (size_t)2 * kCK * (D + 8) * 2 + (size_t)2 * 16 * D * 4;
        e = cudaFuncSetAttribute(prefill_pos_bf16<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        count_launch();
        prefill_pos_bf16<D><<<grid, kCK, smem, s>>>(a);
        return cudaGetLastError();
    }
    const size_t smem = (size_t)2 * kCKf * (D + 4) * 4 + (size_t)3 * 16 * D * 4 + (size_t)16 * kCKf * 4;
    e = cudaFuncSetAttribute(prefill_pos_f32<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    prefill_pos_f32<D><<<grid, kCKf, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(const Dims& m) {
    if (m.dtype == COBS_BF16) return decode_stream_workspace_bytes(m);
    AttnArgs a = make_args(m, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                           nullptr, 1, kCKf);
    return (size_t)m.units() * a.nchunks * m.G * part_stride(m.d) * sizeof(float);
}

cudaError_t launch_decode(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                          const void* Vc, const int32_t* idx, const float* gates, void* O, void* ws,
                          cudaStream_t s, int* err, bool after_select) {
    if (m.dtype == COBS_BF16)
        return launch_decode_stream(m, Q, K, V, Kc, Vc, idx, gates, O, ws, after_select, s, err);
    AttnArgs a = make_args(m, Q, K, V, Kc, Vc, idx, gates, O, ws, err, 1, kCKf);
    return m.d == 128 ? launch_decode_d<128>(m, a, s) : launch_decode_d<64>(m, a, s);
}

// ---------------------------------------------------------------- allocation-free decode variant
// Scratch of cobs_sparse_attn_decode_noalloc: the split-K partial records live in this fixed
// array instead of a caller-provided workspace. Every device that loads the library holds it
// until the process exits. Calls share it, so calls that overlap on the GPU race; nothing in it
// needs clearing, because a call writes every record before it reads it.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kNoAllocMaxDevices] = {nullptr};

// The array's name is only a host-side stand-in: its device address is looked up once per
// device, with that device current.
cudaError_t noalloc_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}
}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t launch_decode_noalloc(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                                  const void* Vc, const int32_t* idx, const float* gates, void* O, cudaStream_t s,
                                  int* err) {
    void* scratch = nullptr;
    cudaError_t e = noalloc_scratch_address(&scratch);
    if (e != cudaSuccess) return e;
    return launch_decode(m, Q, K, V, Kc, Vc, idx, gates, O, scratch, s, err);
}

size_t prefill_workspace_bytes(const Dims&) { return 0; }

cudaError_t launch_prefill(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                           const void* Vc, const int32_t* idx, const float* gates, void* O, void* ws,
                           cudaStream_t s, int* err) {
    // tensor-core tiles for bf16, d = 128, 16 heads per group; the per-position kernel otherwise
    const cudaError_t tc = launch_prefill_tc(m, Q, K, V, Kc, Vc, idx, gates, O, s, err);
    if (tc != cudaErrorNotSupported) return tc;
    const int CK = m.dtype == COBS_BF16 ? kCK : kCKf;
    AttnArgs a = make_args(m, Q, K, V, Kc, Vc, idx, gates, O, ws, err, m.T, CK);
    return m.d == 128 ? launch_prefill_d<128>(m, a, s) : launch_prefill_d<64>(m, a, s);
}

}  // namespace cobs
