// C ABI of the COBS library: host-side validation and launches on the caller's stream.
// The library allocates nothing; every buffer and the workspace belong to the caller.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <atomic>
#include <mutex>
#include <string>

#include "common.cuh"
#include "dims.h"

namespace {

thread_local std::string g_last_error;

cobs_status fail(cobs_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

cobs_status cuda_fail(cudaError_t e, const char* where) {
    return fail(COBS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Device error flag: one int per device that loads this library. Host code cannot use
// the symbol's name as a device address, so the address is looked up once per device.
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
std::mutex g_flag_mutex;
int* g_flag_addr[kMaxDevices] = {nullptr};

cobs_status device_flag(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(COBS_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
    std::lock_guard<std::mutex> lock(g_flag_mutex);
    if (g_flag_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_error);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        g_flag_addr[dev] = static_cast<int*>(p);
    }
    *out = g_flag_addr[dev];
    return COBS_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The query-subspace summaries (float32 or FP4 coordinates) take a basis.
bool uses_basis(const cobs_params* p) {
    return p->variance == COBS_VAR_SUBSPACE || p->variance == COBS_VAR_SUBSPACE_FP4;
}

cobs_status validate(const cobs_params* p) {
    if (p == nullptr) return fail(COBS_ERR_INVALID_ARG, "params is NULL");
    if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->T < 1)
        return fail(COBS_ERR_INVALID_ARG, "B, Hq, Hkv and T must be >= 1 (got %d, %d, %d, %d)", p->B, p->Hq,
                    p->Hkv, p->T);
    if (p->Hq % p->Hkv != 0) return fail(COBS_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", p->Hq, p->Hkv);
    if (p->Hq / p->Hkv > 16) return fail(COBS_ERR_UNSUPPORTED, "GQA group size %d > 16", p->Hq / p->Hkv);
    if (p->d != 64 && p->d != 128) return fail(COBS_ERR_UNSUPPORTED, "head dimension %d (supported: 64, 128)", p->d);
    if (p->block != 64) return fail(COBS_ERR_UNSUPPORTED, "selection block %d (supported: 64)", p->block);
    if (p->topk < 1) return fail(COBS_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", p->topk);
    if (p->topk > 32) return fail(COBS_ERR_UNSUPPORTED, "topk %d > 32", p->topk);
    if (p->window < p->block)
        return fail(COBS_ERR_INVALID_ARG, "window (%d) must be >= block (%d) so that the partial block is covered",
                    p->window, p->block);
    if (p->cmp_stride < 1 || p->cmp_block < p->cmp_stride)
        return fail(COBS_ERR_INVALID_ARG, "need 1 <= cmp_stride <= cmp_block (got %d, %d)", p->cmp_stride,
                    p->cmp_block);
    if (p->dtype != COBS_F32 && p->dtype != COBS_BF16) return fail(COBS_ERR_INVALID_ARG, "dtype %d", p->dtype);
    if (p->variance < COBS_VAR_CHANNEL || p->variance > COBS_VAR_SUBSPACE_FP4)
        return fail(COBS_ERR_INVALID_ARG, "variance %d (a cobs_variance value)", p->variance);
    if (p->variance >= COBS_VAR_LOWRANK && (p->rank < 1 || p->rank > 8))
        return fail(COBS_ERR_UNSUPPORTED, "rank %d (supported: 1 .. 8)", p->rank);
    if (uses_basis(p)) {
        if (p->sub < 4 || p->sub > p->d || p->sub % 4 != 0)
            return fail(COBS_ERR_UNSUPPORTED, "subspace dimension %d (a multiple of 4 in 4 .. d)", p->sub);
    }
    if (!isfinite(p->alpha)) return fail(COBS_ERR_INVALID_ARG, "alpha is not finite");
    if ((long long)p->B * p->Hkv > 65535) return fail(COBS_ERR_UNSUPPORTED, "B * Hkv > 65535");
    // K / V rows (and the compressed rows, fewer) are addressed by int32 row coordinates in the
    // TMA tensor maps and tile descriptors
    if ((long long)p->B * p->Hkv * p->T > INT32_MAX)
        return fail(COBS_ERR_UNSUPPORTED, "B * Hkv * T = %lld rows exceeds 2^31 - 1",
                    (long long)p->B * p->Hkv * p->T);
    return COBS_OK;
}

// Prefill calls address query rows [B, T, Hq] with int32 coordinates as well.
cobs_status validate_prefill_rows(const cobs_params* p) {
    if ((long long)p->B * p->Hq * p->T > INT32_MAX)
        return fail(COBS_ERR_UNSUPPORTED, "B * Hq * T = %lld query rows exceeds 2^31 - 1",
                    (long long)p->B * p->Hq * p->T);
    return COBS_OK;
}

cobs_status check_ptr(const void* ptr, const char* name, bool may_be_null = false) {
    if (ptr == nullptr) {
        if (may_be_null) return COBS_OK;
        return fail(COBS_ERR_INVALID_ARG, "%s is NULL", name);
    }
    if (!aligned16(ptr)) return fail(COBS_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return COBS_OK;
}

#define COBS_TRY(x)                      \
    do {                                 \
        cobs_status _s = (x);            \
        if (_s != COBS_OK) return _s;    \
    } while (0)

}  // namespace

namespace cobs {
static std::atomic<long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

void score_constants(int d, float alpha, float* isd, float* c2) {
    *isd = (float)(1.0 / sqrt((double)d));
    *c2 = (float)((double)alpha * 0.5 / (double)d);
}
}  // namespace cobs

namespace {
size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Decode step workspace: the selection workspace followed by the decode-attention workspace.
size_t step_workspace_bytes(const cobs::Dims& m) {
    return al256(cobs::select_workspace_bytes(m, 0)) + cobs::decode_workspace_bytes(m);
}
}  // namespace

extern "C" {

int32_t cobs_version(void) { return 102; }

int64_t cobs_launch_count(int32_t reset) {
    return reset ? cobs::g_launches.exchange(0) : cobs::g_launches.load();
}

const char* cobs_status_string(cobs_status s) {
    switch (s) {
        case COBS_OK: return "ok";
        case COBS_ERR_INVALID_ARG: return "invalid argument";
        case COBS_ERR_UNSUPPORTED: return "unsupported shape or option";
        case COBS_ERR_CUDA: return "CUDA error";
        case COBS_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

const char* cobs_last_error(void) { return g_last_error.c_str(); }

size_t cobs_summaries_elems(const cobs_params* p) {
    if (p == nullptr || validate(p) != COBS_OK) return 0;
    const cobs::Dims m = cobs::make_dims(*p);
    return (size_t)m.units() * m.summ_unit_floats();
}

size_t cobs_workspace_bytes(const cobs_params* p, int32_t which) {
    if (p == nullptr || validate(p) != COBS_OK) return 0;
    const cobs::Dims m = cobs::make_dims(*p);
    switch (which) {
        case COBS_WS_SELECT: {
            const size_t a = cobs::select_workspace_bytes(m, 0), b = cobs::select_workspace_bytes(m, 1);
            return a > b ? a : b;
        }
        case COBS_WS_DECODE: return cobs::decode_workspace_bytes(m);
        case COBS_WS_PREFILL: return cobs::prefill_workspace_bytes(m);
        case COBS_WS_STEP: return step_workspace_bytes(m);
        case COBS_WS_STEP_FUSED: return cobs::decode_step_workspace_bytes(m);  // 0: shape not taken
        case COBS_WS_BASIS: return cobs::basis_workspace_bytes(m);
    }
    return 0;
}

int32_t cobs_device_error(int32_t reset) {
    int* flag = nullptr;
    if (device_flag(&flag) != COBS_OK) return -1;
    int v = 0;
    if (cudaMemcpy(&v, flag, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
    if (reset) {
        const int zero = 0;
        if (cudaMemcpy(flag, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return -1;
    }
    return v;
}

cobs_status cobs_build_summaries(const cobs_params* p, const void* K, const void* V, const float* Pk,
                                 const float* Pv, int32_t t_begin, float* summaries, void* Kc, void* Vc,
                                 cobs_stream_t stream) {
    COBS_TRY(validate(p));
    COBS_TRY(check_ptr(K, "K"));
    COBS_TRY(check_ptr(V, "V"));
    COBS_TRY(check_ptr(Pk, "Pk", true));
    COBS_TRY(check_ptr(Pv, "Pv", true));
    COBS_TRY(check_ptr(summaries, "summaries"));
    if (uses_basis(p)) COBS_TRY(check_ptr(p->basis, "basis"));
    const cobs::Dims m = cobs::make_dims(*p);
    if (m.nC > 0) {
        COBS_TRY(check_ptr(Kc, "Kc"));
        COBS_TRY(check_ptr(Vc, "Vc"));
    }
    if (t_begin < 0 || t_begin > p->T) return fail(COBS_ERR_INVALID_ARG, "t_begin %d outside [0, T]", t_begin);
    int* flag = nullptr;
    COBS_TRY(device_flag(&flag));
    cudaError_t e = cobs::launch_summaries(m, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, (cudaStream_t)stream, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_build_summaries launch");
    return COBS_OK;
}

cobs_status cobs_select(const cobs_params* p, const void* Q, const float* summaries, int32_t prefill, int32_t* idx,
                        void* workspace, size_t ws_bytes, cobs_stream_t stream) {
    COBS_TRY(validate(p));
    COBS_TRY(check_ptr(Q, "Q"));
    COBS_TRY(check_ptr(summaries, "summaries"));
    COBS_TRY(check_ptr(idx, "idx"));
    if (prefill != 0 && prefill != 1) return fail(COBS_ERR_INVALID_ARG, "prefill must be 0 or 1");
    if (prefill) COBS_TRY(validate_prefill_rows(p));
    if (uses_basis(p) && !prefill) COBS_TRY(check_ptr(p->basis, "basis"));
    if (prefill && p->variance >= COBS_VAR_LOWRANK)
        return fail(COBS_ERR_UNSUPPORTED, "prefill selection with low-rank summaries");
    const cobs::Dims m = cobs::make_dims(*p);
    const size_t need = cobs::select_workspace_bytes(m, prefill);
    if (need > 0) {
        COBS_TRY(check_ptr(workspace, "workspace"));
        if (ws_bytes < need) return fail(COBS_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    }
    int* flag = nullptr;
    COBS_TRY(device_flag(&flag));
    cudaError_t e = cobs::launch_select(m, Q, summaries, prefill, idx, workspace, (cudaStream_t)stream, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_select launch");
    return COBS_OK;
}

static cobs_status attn_common(const cobs_params* p, const void* Q, const void* K, const void* V, const void* Kc,
                               const void* Vc, const int32_t* idx, const float* gates, void* O) {
    COBS_TRY(validate(p));
    COBS_TRY(check_ptr(Q, "Q"));
    COBS_TRY(check_ptr(K, "K"));
    COBS_TRY(check_ptr(V, "V"));
    COBS_TRY(check_ptr(idx, "idx"));
    COBS_TRY(check_ptr(gates, "gates"));
    COBS_TRY(check_ptr(O, "O"));
    const cobs::Dims m = cobs::make_dims(*p);
    if (m.nC > 0) {
        COBS_TRY(check_ptr(Kc, "Kc"));
        COBS_TRY(check_ptr(Vc, "Vc"));
    }
    return COBS_OK;
}

cobs_status cobs_sparse_attn_decode(const cobs_params* p, const void* Q, const void* K, const void* V,
                                    const void* Kc, const void* Vc, const int32_t* idx, const float* gates, void* O,
                                    void* workspace, size_t ws_bytes, cobs_stream_t stream) {
    COBS_TRY(attn_common(p, Q, K, V, Kc, Vc, idx, gates, O));
    const cobs::Dims m = cobs::make_dims(*p);
    const size_t need = cobs::decode_workspace_bytes(m);
    if (need > 0) {
        COBS_TRY(check_ptr(workspace, "workspace"));
        if (ws_bytes < need) return fail(COBS_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    }
    int* flag = nullptr;
    COBS_TRY(device_flag(&flag));
    cudaError_t e = cobs::launch_decode(m, Q, K, V, Kc, Vc, idx, gates, O, workspace, (cudaStream_t)stream, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_sparse_attn_decode launch");
    return COBS_OK;
}

// Checks shared by the two decode-step entry points.
static cobs_status step_common(const cobs_params* p, const void* Q, const void* K, const void* V, const float* Pk,
                               const float* Pv, int32_t t_begin, float* summaries, void* Kc, void* Vc,
                               int32_t* idx, const float* gates, void* O, void* workspace) {
    COBS_TRY(attn_common(p, Q, K, V, Kc, Vc, idx, gates, O));
    COBS_TRY(check_ptr(Pk, "Pk", true));
    COBS_TRY(check_ptr(Pv, "Pv", true));
    COBS_TRY(check_ptr(summaries, "summaries"));
    if (uses_basis(p)) COBS_TRY(check_ptr(p->basis, "basis"));
    if (t_begin < 0 || t_begin > p->T) return fail(COBS_ERR_INVALID_ARG, "t_begin %d outside [0, T]", t_begin);
    COBS_TRY(check_ptr(workspace, "workspace"));
    return COBS_OK;
}

cobs_status cobs_decode_step(const cobs_params* p, const void* Q, const void* K, const void* V, const float* Pk,
                             const float* Pv, int32_t t_begin, float* summaries, void* Kc, void* Vc, int32_t* idx,
                             const float* gates, void* O, void* workspace, size_t ws_bytes, cobs_stream_t stream) {
    COBS_TRY(step_common(p, Q, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, idx, gates, O, workspace));
    const cobs::Dims m = cobs::make_dims(*p);
    const size_t need = step_workspace_bytes(m);
    if (ws_bytes < need) return fail(COBS_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    int* flag = nullptr;
    COBS_TRY(device_flag(&flag));
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cobs::launch_summaries(m, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, s, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_decode_step: summary update launch");
    unsigned char* w = static_cast<unsigned char*>(workspace);
    e = cobs::launch_select(m, Q, summaries, 0, idx, w, s, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_decode_step: selection launch");
    // the attention grid follows the selection grids as their programmatic dependent
    e = cobs::launch_decode(m, Q, K, V, Kc, Vc, idx, gates, O, w + al256(cobs::select_workspace_bytes(m, 0)), s, flag,
                            true);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_decode_step: attention launch");
    return COBS_OK;
}

cobs_status cobs_decode_step_fused(const cobs_params* p, const void* Q, const void* K, const void* V,
                                   const float* Pk, const float* Pv, int32_t t_begin, float* summaries, void* Kc,
                                   void* Vc, int32_t* idx, const float* gates, void* O, void* workspace,
                                   size_t ws_bytes, cobs_stream_t stream) {
    COBS_TRY(step_common(p, Q, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, idx, gates, O, workspace));
    const cobs::Dims m = cobs::make_dims(*p);
    if (!cobs::decode_step_supported(m))
        return fail(COBS_ERR_UNSUPPORTED,
                    "cobs_decode_step_fused takes bf16, d in {64, 128}, block 64 and the per-channel or isotropic "
                    "summaries (with its rings and index tables in shared memory); use cobs_decode_step");
    const size_t need = cobs::decode_step_workspace_bytes(m);
    if (ws_bytes < need) return fail(COBS_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    int* flag = nullptr;
    COBS_TRY(device_flag(&flag));
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cobs::launch_summaries(m, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, s, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_decode_step_fused: summary update launch");
    e = cobs::launch_decode_step(m, Q, summaries, K, V, Kc, Vc, idx, gates, O, workspace, s, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_decode_step_fused launch");
    return COBS_OK;
}

cobs_status cobs_sparse_attn_decode_noalloc(const cobs_params* p, const void* Q, const void* K, const void* V,
                                            const void* Kc, const void* Vc, const int32_t* idx, const float* gates,
                                            void* O, cobs_stream_t stream) {
    COBS_TRY(attn_common(p, Q, K, V, Kc, Vc, idx, gates, O));
    const cobs::Dims m = cobs::make_dims(*p);
    const size_t need = cobs::decode_workspace_bytes(m);
    const size_t have = cobs::noalloc_scratch_bytes();
    if (need > have)
        return fail(COBS_ERR_WORKSPACE,
                    "this problem needs %zu bytes of decode scratch, more than the %zu bytes built into the library; "
                    "call cobs_sparse_attn_decode with a workspace instead",
                    need, have);
    int* flag = nullptr;
    COBS_TRY(device_flag(&flag));
    cudaError_t e = cobs::launch_decode_noalloc(m, Q, K, V, Kc, Vc, idx, gates, O, (cudaStream_t)stream, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_sparse_attn_decode_noalloc launch");
    return COBS_OK;
}

cobs_status cobs_sparse_attn_prefill(const cobs_params* p, const void* Q, const void* K, const void* V,
                                     const void* Kc, const void* Vc, const int32_t* idx, const float* gates,
                                     void* O, void* workspace, size_t ws_bytes, cobs_stream_t stream) {
    COBS_TRY(attn_common(p, Q, K, V, Kc, Vc, idx, gates, O));
    COBS_TRY(validate_prefill_rows(p));
    const cobs::Dims m = cobs::make_dims(*p);
    const size_t need = cobs::prefill_workspace_bytes(m);
    if (need > 0) {
        COBS_TRY(check_ptr(workspace, "workspace"));
        if (ws_bytes < need) return fail(COBS_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    }
    int* flag = nullptr;
    COBS_TRY(device_flag(&flag));
    cudaError_t e = cobs::launch_prefill(m, Q, K, V, Kc, Vc, idx, gates, O, workspace, (cudaStream_t)stream, flag);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_sparse_attn_prefill launch");
    return COBS_OK;
}

cobs_status cobs_block_log_mass(const cobs_params* p, const void* Q, const void* K, float* out,
                                cobs_stream_t stream) {
    COBS_TRY(validate(p));
    COBS_TRY(check_ptr(Q, "Q"));
    COBS_TRY(check_ptr(K, "K"));
    COBS_TRY(check_ptr(out, "out"));
    const cobs::Dims m = cobs::make_dims(*p);
    if (m.G > 16) return fail(COBS_ERR_UNSUPPORTED, "cobs_block_log_mass supports at most 16 query heads per group");
    cudaError_t e = cobs::launch_block_log_mass(m, Q, K, out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_block_log_mass launch");
    return COBS_OK;
}

cobs_status cobs_query_basis(const cobs_params* p, const void* Q, int64_t n, float* basis, float* eigenvalues,
                             void* workspace, size_t ws_bytes, cobs_stream_t stream) {
    COBS_TRY(validate(p));
    if (p->sub < 4 || p->sub > p->d || p->sub % 4 != 0)
        return fail(COBS_ERR_UNSUPPORTED, "subspace dimension %d (a multiple of 4 in 4 .. d)", p->sub);
    if (n < 1) return fail(COBS_ERR_INVALID_ARG, "n = %lld query rows (at least one)", (long long)n);
    COBS_TRY(check_ptr(Q, "Q"));
    COBS_TRY(check_ptr(basis, "basis"));
    COBS_TRY(check_ptr(eigenvalues, "eigenvalues", true));
    COBS_TRY(check_ptr(workspace, "workspace"));
    const cobs::Dims m = cobs::make_dims(*p);
    cobs::Dims mb = m;
    mb.sub = p->sub;  // the basis width, whatever the params' summary form
    const size_t need = cobs::basis_workspace_bytes(mb);
    if (ws_bytes < need) return fail(COBS_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    cudaError_t e = cobs::launch_query_basis(mb, Q, (long long)n, basis, eigenvalues, workspace, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cobs_query_basis launch");
    return COBS_OK;
}

}  // extern "C"
