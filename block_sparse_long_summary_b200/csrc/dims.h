// Host-side derived sizes shared by the launchers (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/cobs.h"

namespace cobs {

struct Dims {
    int B, Hq, Hkv, G, d, T, L, lc, sc, k, W;
    int nB;       // complete selection blocks, T / L
    int nG;       // 32-block summary groups, ceil(nB / 32) (at least 1)
    int nC;       // compressed tokens, (T - lc) / sc + 1 (0 if T < lc)
    float alpha;
    int dtype;    // cobs_dtype
    int iso;      // summaries keep one variance scalar per block (COBS_VAR_ISOTROPIC)
    int lr;       // eigenpairs per block (COBS_VAR_LOWRANK / _FP4), else 0
    int fp4;      // low-rank summaries stored as FP4 eigenvectors (or coordinates) and a bf16 mean
    int sub;      // COBS_VAR_SUBSPACE(_FP4): eigenvectors kept as sub coordinates in the basis, else 0
    const float* basis;  // COBS_VAR_SUBSPACE(_FP4): [d][sub] float32 device array
    int units() const { return B * Hkv; }
    // floats of one 32-block summary group: means and per-channel variances, means and one
    // scalar per block, or means, lr eigenvectors and lr eigenvalues per block
    // FP4 codes per vector and block: d, or sub rounded up to a multiple of 32
    int code_width() const { return sub ? (sub + 31) / 32 * 32 : d; }
    size_t group_floats() const {
        if (lr && fp4) return (size_t)8 * (2 * d + lr * code_width() / 2 + 8 * lr);
        if (lr && sub) return (size_t)32 * (d + lr * sub + lr);
        if (lr) return (size_t)32 * (d + lr * d + lr);
        return iso ? (size_t)(d + 1) * 32 : (size_t)2 * d * 32;
    }
    size_t summ_unit_floats() const { return (size_t)nG * group_floats(); }
};

inline Dims make_dims(const cobs_params& p) {
    Dims m;
    m.B = p.B; m.Hq = p.Hq; m.Hkv = p.Hkv; m.G = p.Hkv ? p.Hq / p.Hkv : 0; m.d = p.d; m.T = p.T;
    m.L = p.block; m.lc = p.cmp_block; m.sc = p.cmp_stride; m.k = p.topk; m.W = p.window;
    m.nB = p.block > 0 ? p.T / p.block : 0;
    m.nG = m.nB > 0 ? (m.nB + 31) / 32 : 1;
    m.nC = (p.cmp_stride > 0 && p.T >= p.cmp_block) ? (p.T - p.cmp_block) / p.cmp_stride + 1 : 0;
    m.alpha = p.alpha; m.dtype = p.dtype; m.iso = p.variance == COBS_VAR_ISOTROPIC;
    m.lr = p.variance >= COBS_VAR_LOWRANK ? p.rank : 0;
    m.fp4 = p.variance == COBS_VAR_LOWRANK_FP4 || p.variance == COBS_VAR_SUBSPACE_FP4;
    const bool subspace = p.variance == COBS_VAR_SUBSPACE || p.variance == COBS_VAR_SUBSPACE_FP4;
    m.sub = subspace ? p.sub : 0;
    m.basis = subspace ? p.basis : nullptr;
    return m;
}

// Count one kernel launch (read through cobs_launch_count).
void count_launch(int n = 1);

// Score constants of the canonical selector: isd = RN32(1/sqrt(d)) (through double),
// c2 = RN32(alpha * 0.5 / d).
void score_constants(int d, float alpha, float* isd, float* c2);

// ---- launchers (return cudaSuccess or the launch error) ----
cudaError_t launch_summaries(const Dims& m, const void* K, const void* V, const float* Pk,
                             const float* Pv, int t_begin, float* summ, void* Kc, void* Vc,
                             cudaStream_t s, int* err);

size_t select_workspace_bytes(const Dims& m, int prefill);
cudaError_t launch_select(const Dims& m, const void* Q, const float* summ, int prefill, int32_t* idx,
                          void* ws, cudaStream_t s, int* err);

size_t decode_workspace_bytes(const Dims& m);
size_t decode_stream_workspace_bytes(const Dims& m);
// after_select: launched as a programmatic dependent of the selection grids just before it in the
// stream (the decode step); it then reads K, V, Kc and Vc before they complete and idx after.
cudaError_t launch_decode_stream(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                                 const void* Vc, const int32_t* idx, const float* gates, void* O, void* ws,
                                 bool after_select, cudaStream_t s, int* err);
cudaError_t launch_decode(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                          const void* Vc, const int32_t* idx, const float* gates, void* O, void* ws,
                          cudaStream_t s, int* err, bool after_select = false);

// Decode with the library's fixed device scratch in place of a workspace (no allocation).
size_t noalloc_scratch_bytes();
cudaError_t launch_decode_noalloc(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                                  const void* Vc, const int32_t* idx, const float* gates, void* O, cudaStream_t s,
                                  int* err);

// Fused decode step (selection + decode attention in one persistent kernel): bf16, d in {64, 128},
// the per-channel or isotropic summaries.
bool decode_step_supported(const Dims& m);
size_t decode_step_workspace_bytes(const Dims& m);
cudaError_t launch_decode_step(const Dims& m, const void* Q, const float* summ, const void* K, const void* V,
                               const void* Kc, const void* Vc, int32_t* idx, const float* gates, void* O, void* ws,
                               cudaStream_t s, int* err);

size_t prefill_workspace_bytes(const Dims& m);
// tcgen05 prefill (bf16, d = 128, G = 16); cudaErrorNotSupported for other shapes.
cudaError_t launch_prefill_tc(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                              const void* Vc, const int32_t* idx, const float* gates, void* O, cudaStream_t s,
                              int* err);
cudaError_t launch_prefill(const Dims& m, const void* Q, const void* K, const void* V, const void* Kc,
                           const void* Vc, const int32_t* idx, const float* gates, void* O, void* ws,
                           cudaStream_t s, int* err);

// Query-subspace basis from n query rows [n][d]: the eigenvectors of their second moment for the
// m.sub largest eigenvalues, basis [d][m.sub] float32 (evals [m.sub], may be null).
size_t basis_workspace_bytes(const Dims& m);
cudaError_t launch_query_basis(const Dims& m, const void* Q, long long n, float* basis, float* evals, void* ws,
                               cudaStream_t s);

// Evaluation only: ln of the exact attention mass of every complete block, out [B, Hq, nB] f32
// (cudaErrorNotSupported if G > 16).
cudaError_t launch_block_log_mass(const Dims& m, const void* Q, const void* K, float* out, cudaStream_t s);

}  // namespace cobs
