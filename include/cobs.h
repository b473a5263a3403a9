/*
 * cobs.h — C ABI of the B200 (sm_100a) library for block-sparse attention with
 * cumulant-order block selection (COBS).
 *
 * Method sources (cited per call below):
 *   [COBS]    "COBS: Cumulant Order Block Sparse Attention", gist.science explainer of
 *             arXiv 2607.09052: §2.1 attention mass, §2.2 cumulant expansion,
 *             §2.3 second-order scoring on the NSA branches.
 *   [SKILL]   "cumulant-order-block-sparse-attention" skill card: "Method",
 *             "Implementation steps".
 *   [NSA-181] deepseek-ai/Janus issue #181 ("four dimensions regarding importance and
 *             connection strength"): compression / selection / sliding-window paths and
 *             their gates.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument except `p` is DEVICE memory owned by the caller; `p` is host
 *   memory read during the call only. The library never allocates, frees or keeps
 *   pointers past the call, and never synchronises: work is enqueued on `stream`
 *   (NULL = legacy default stream) and the call returns at once.
 * - Arguments are validated on the host before anything is launched. An invalid
 *   argument returns COBS_ERR_INVALID_ARG (or COBS_ERR_UNSUPPORTED for a valid
 *   but unsupported shape) and enqueues nothing; cobs_last_error() then holds a
 *   message. A failed launch returns COBS_ERR_CUDA. Kernels never trap: an
 *   out-of-range block index met on the device is skipped and recorded in a device
 *   flag read by cobs_device_error().
 * - Tensor layouts (row-major, contiguous, element type per `dtype`: bfloat16 or
 *   float32; indices int32; gates and summaries float32):
 *     K, V         [B, Hkv, T, d]
 *     Q, O decode  [B, Hq, d]            (the query at position T-1)
 *     Q, O prefill [B, T, Hq, d]
 *     gates        decode [B, Hq, 3], prefill [B, T, Hq, 3]: (g_cmp, g_slc, g_win),
 *                  already passed through the sigmoid
 *     Kc, Vc       [B, Hkv, nC, d], nC = (T - cmp_block) / cmp_stride + 1 (0 if T < cmp_block)
 *     idx          decode [B, Hkv, topk], prefill [B, T, Hkv, topk]
 *     summaries    variance = COBS_VAR_CHANNEL: [B, Hkv, nG, 2, d/4, 32, 4] float32,
 *                  nG = ceil(nB / 32), nB = T / block: block b of a unit lives in group b/32,
 *                  lane b%32; entry [..., 0, c/4, b%32, c%4] is the key mean mu_{b,c},
 *                  [..., 1, ...] the key variance var_{b,c}.
 *                  variance = COBS_VAR_ISOTROPIC: [B, Hkv, nG, (d/4 * 32 * 4) + 32] float32:
 *                  the means as above, then sigma2_b of the group's 32 blocks.
 *                  variance = COBS_VAR_LOWRANK (rank R): [B, Hkv, nG, (1 + R) * (d/4 * 32 * 4) + R * 32]
 *                  float32: the means as above, then eigenvector j < R of the group's blocks in
 *                  the same [d/4, 32, 4] interleaving, then the R eigenvalues [R, 32].
 *                  variance = COBS_VAR_LOWRANK_FP4 (rank R): per group of 32 blocks, bytes
 *                  [d/8, 32, 8] bf16 means, then for j < R [d/32, 32, 16] bytes of E2M1 codes
 *                  (byte i of a lane's 16-byte word: channel 2i in the low nibble, 2i + 1 in the
 *                  high one), then [R, 32] float32 scales, then [R, 32] float32 eigenvalues
 *                  (8 (2d + R d / 2 + 8 R) float32 elements per group).
 *                  variance = COBS_VAR_SUBSPACE (rank R, sub s): [B, Hkv, nG, 32 (d + R s + R)]
 *                  float32: the means as above, then the s coordinates of eigenvector j < R in a
 *                  [s/4, 32, 4] interleaving, then the R eigenvalues [R, 32].
 *                  variance = COBS_VAR_SUBSPACE_FP4 (rank R, sub s; sp = s rounded up to a
 *                  multiple of 32): the COBS_VAR_LOWRANK_FP4 layout with the codes of the s
 *                  coordinates of projected eigenvector j in [sp/32, 32, 16] bytes (coordinates
 *                  s .. sp - 1 have code 0): 8 (2d + R sp / 2 + 8 R) float32 elements per group.
 *                  (32 consecutive blocks are interleaved channel-by-channel so that one
 *                  group is one contiguous copy and lane b%32 reads its block's channels.)
 * - GQA: query head h belongs to KV head h / (Hq / Hkv).
 * - Supported: d in {64, 128}; block = 64; 1 <= topk <= 32; window >= block;
 *   Hq % Hkv == 0 and Hq / Hkv <= 16; cmp_block = 32, cmp_stride = 16 for bf16
 *   (any cmp_block >= cmp_stride >= 1 for float32); T >= 1.
 */
#ifndef COBS_H_
#define COBS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cobs_stream_t; /* identical to cudaStream_t */

typedef enum {
    COBS_OK = 0,
    COBS_ERR_INVALID_ARG = -1,
    COBS_ERR_UNSUPPORTED = -2,
    COBS_ERR_CUDA = -3,
    COBS_ERR_WORKSPACE = -4
} cobs_status;

typedef enum { COBS_F32 = 0, COBS_BF16 = 1 } cobs_dtype;

typedef enum {
    COBS_WS_SELECT = 0,
    COBS_WS_DECODE = 1,
    COBS_WS_PREFILL = 2,
    COBS_WS_STEP = 3,      /* cobs_decode_step */
    COBS_WS_STEP_FUSED = 4, /* cobs_decode_step_fused (0 bytes: a shape it does not take) */
    COBS_WS_BASIS = 5       /* cobs_query_basis */
} cobs_workspace_kind;

/* Second-order statistic kept per block ([COBS] §2.2/§2.3: the block covariance Sigma_b, compressed):
 *   COBS_VAR_CHANNEL    the per-channel population variance var_{b,c} (the diagonal of Sigma_b);
 *                       score term alpha/2 * sum_c q_c^2 var_{b,c} / d.
 *   COBS_VAR_ISOTROPIC  one scalar per block ([SKILL] "Pitfalls": one or two scalars per block):
 *                       Sigma_b ~ sigma2_b I with sigma2_b = (1/d) sum_c var_{b,c};
 *                       score term alpha/2 * sigma2_b |q|^2 / d. Summaries are about half the bytes.
 *   COBS_VAR_LOWRANK    the `rank` leading eigenpairs (lambda_j, u_j) of Sigma_b ([COBS] §2.2/§2.3,
 *                       low-rank compression of the covariance); score term
 *                       alpha/2 * sum_j lambda_j (q . u_j)^2 / d. The eigenpairs come from a fixed
 *                       float32 subspace iteration (24 steps, modified Gram-Schmidt), so they are
 *                       reproducible bit for bit. Decode selection only (prefill selection with
 *                       these summaries returns COBS_ERR_UNSUPPORTED).
 *   COBS_VAR_LOWRANK_FP4  the same eigenpairs with each eigenvector in FP4 (E2M1, one float32
 *                       scale max|u|/6 per vector, round to nearest with ties to even, saturating)
 *                       and the mean in bf16 ([COBS] §2.3); the score uses the dequantized values.
 *                       About a fifth of the float32 low-rank bytes. Decode selection only.
 *   COBS_VAR_SUBSPACE   the COBS_VAR_LOWRANK eigenpairs with each eigenvector kept as its `sub`
 *                       coordinates u~_j = P^T u_j in the query subspace spanned by the columns of
 *                       `basis` ([COBS] §2.3, projection onto the query subspace: r d -> r s numbers
 *                       per block); the query heads are projected the same way, q~ = P^T q (float32,
 *                       four-chain sums over the d channels), and the score term is
 *                       alpha/2 * sum_j lambda_j (q~ . u~_j)^2 / d. Exact for queries inside span(P)
 *                       when P has orthonormal columns. Decode selection only.
 *   COBS_VAR_SUBSPACE_FP4  the three compressions of [COBS] §2.3 together (the form its §4.1 reports
 *                       as "Subspace, r=4, FP4"): the COBS_VAR_SUBSPACE coordinates of each
 *                       eigenvector in FP4 (E2M1, one float32 scale max|u~|/6 per vector, the
 *                       COBS_VAR_LOWRANK_FP4 rounding) and the mean in bf16; the score uses the
 *                       dequantized values. Decode selection only. */
typedef enum {
    COBS_VAR_CHANNEL = 0,
    COBS_VAR_ISOTROPIC = 1,
    COBS_VAR_LOWRANK = 2,
    COBS_VAR_LOWRANK_FP4 = 3,
    COBS_VAR_SUBSPACE = 4,
    COBS_VAR_SUBSPACE_FP4 = 5
} cobs_variance;

/* Problem statement ([COBS] §2.3, [SKILL] "Method"): block size, compression block and
 * stride, top-k, window and alpha. */
typedef struct {
    int32_t B;          /* batch */
    int32_t Hq;         /* query heads */
    int32_t Hkv;        /* key/value heads (GQA groups) */
    int32_t d;          /* head dimension */
    int32_t T;          /* context length (decode: the query sits at T-1) */
    int32_t block;      /* selection block L */
    int32_t cmp_block;  /* compression block l_c */
    int32_t cmp_stride; /* compression stride s_c */
    int32_t topk;       /* selected blocks per GQA group */
    int32_t window;     /* sliding window W */
    float alpha;        /* weight of the second-order (variance) term */
    int32_t dtype;      /* cobs_dtype of Q, K, V, Kc, Vc, O */
    int32_t variance;   /* cobs_variance: the second-order statistic of the summaries */
    int32_t rank;       /* eigenpairs per block for the low-rank forms (1 .. 8); ignored otherwise */
    int32_t sub;        /* COBS_VAR_SUBSPACE(_FP4): subspace dimension s (a multiple of 4, 4 .. d); else ignored */
    const float* basis; /* COBS_VAR_SUBSPACE(_FP4): device array [d][sub] float32, the basis P of the query
                           subspace (orthonormal columns expected, not checked), read by
                           cobs_build_summaries and cobs_select and owned by the caller; else ignored */
} cobs_params;

/*
 * Block summaries and compressed tokens: one pass over K and V.
 * [COBS] §2.2/§2.3: per block, the key mean mu_b (kappa_1) and the second-order
 * statistic, here the per-channel population variance var_b (the diagonal of the
 * block covariance kappa_2); [NSA-181] compression path: compressed token i is
 * P · mean(rows cmp_stride*i .. cmp_stride*i + cmp_block - 1), for K with P_k and for V
 * with P_v ([SKILL] step 4: the compression branch itself is unchanged).
 *   Pk, Pv     [d, d] float32 device matrices (out = P @ pooled), or NULL for identity.
 *   t_begin    positions < t_begin are already summarised: only blocks and compressed
 *              tokens whose last row is >= t_begin are (re)written. 0 = full build;
 *              T - 1 = the update after appending the token at T - 1.
 *   summaries, Kc, Vc: outputs (layouts above). Summaries are float32 in a fixed
 *              summation order (row order), so they are reproducible bit for bit.
 */
cobs_status cobs_build_summaries(const cobs_params* p, const void* K, const void* V,
                                 const float* Pk, const float* Pv, int32_t t_begin,
                                 float* summaries, void* Kc, void* Vc, cobs_stream_t stream);

/*
 * Block selection ([COBS] §2.3 second-order score; [SKILL] step 3 and "Method": top-k).
 * For each GQA group g and candidate block b:
 *   S_{g,b} = (sum_c Qsum_c mu_{b,c}) * RN(1/sqrt(d)) + RN(alpha/(2d)) * (sum_c Q2_c var_{b,c}),
 *   or, with COBS_VAR_ISOTROPIC summaries, ... + RN(alpha/(2d)) * RN((sum_c Q2_c) * sigma2_b)
 *   (sum_c Q2_c by adds in ascending c), or, with COBS_VAR_LOWRANK summaries,
 *   ... + RN(alpha/(2d)) * sum_j lambda_j * (sum_{h in g} (q_h . u_j)^2) (fma, ascending j and h);
 *   every channel sum runs as four partial chains (channels c = j mod 4) combined as
 *   (s0 + s1) + (s2 + s3),
 *   Qsum = sum_{h in g} q_h, Q2 = sum_{h in g} q_h*q_h   (= sum_h [q_h.mu_b/sqrt(d)
 *   + alpha/2 * sum_c q_{h,c}^2 var_{b,c}/d]), evaluated in float32 with fused multiply-adds
 *   in ascending head and channel order. Candidates are the complete blocks
 *   b < (t + 1) / block at query position t. The topk best by (score descending, block
 *   ascending) are written in ascending block order, padded with -1.
 *   prefill = 0: Q [B, Hq, d] at t = T - 1, idx [B, Hkv, topk].
 *   prefill = 1: Q [B, T, Hq, d] at every t, idx [B, T, Hkv, topk].
 *   workspace: >= cobs_workspace_bytes(p, COBS_WS_SELECT) bytes of scratch (decode: the
 *              partial top-k lists of contexts split across CTAs; no initial contents needed).
 *              Calls that share one workspace must not run concurrently.
 */
cobs_status cobs_select(const cobs_params* p, const void* Q, const float* summaries,
                        int32_t prefill, int32_t* idx, void* workspace, size_t ws_bytes,
                        cobs_stream_t stream);

/*
 * Decode attention at position T - 1 ([NSA-181] three paths; [COBS] §2.3):
 *   o_h = g_cmp softmax_cmp + g_slc softmax_slc + g_win softmax_win, each branch a
 *   softmax(q K^T / sqrt(d)) V of its own over the compressed tokens (all nC), the tokens
 *   of the selected blocks idx (entries -1 skipped) and the tokens max(0, T-W) .. T-1.
 *   An empty branch contributes zero.
 *   workspace: >= cobs_workspace_bytes(p, COBS_WS_DECODE) bytes of scratch for the split-K
 *              partial results; no initial contents are needed (every partial is written
 *              before it is read). Calls that share one workspace must not run concurrently.
 */
cobs_status cobs_sparse_attn_decode(const cobs_params* p, const void* Q, const void* K,
                                    const void* V, const void* Kc, const void* Vc,
                                    const int32_t* idx, const float* gates, void* O,
                                    void* workspace, size_t ws_bytes, cobs_stream_t stream);

/*
 * One decode step, enqueued as one unit: the summary update of cobs_build_summaries from t_begin,
 * then the block selection of cobs_select (prefill = 0), then cobs_sparse_attn_decode, with the
 * arguments, layouts and results of those three calls ([COBS] §2.2/§2.3 summaries and
 * second-order selection; [NSA-181] the three paths and their gates). idx and O are written as
 * the separate calls write them (the same indices bit for bit, the same attention up to float32
 * summation order).
 * The attention grid is launched as a programmatic dependent of the selection grids: its window
 * and compressed-token tiles, which do not depend on idx, stream while the selection finishes,
 * and it reads idx only after the selection grids have completed.
 *   workspace: >= cobs_workspace_bytes(p, COBS_WS_STEP) bytes; no initial contents are needed.
 *              Calls that share one workspace must not run concurrently.
 * Errors: those of the three calls.
 */
cobs_status cobs_decode_step(const cobs_params* p, const void* Q, const void* K, const void* V,
                             const float* Pk, const float* Pv, int32_t t_begin, float* summaries,
                             void* Kc, void* Vc, int32_t* idx, const float* gates, void* O,
                             void* workspace, size_t ws_bytes, cobs_stream_t stream);

/*
 * The same decode step with the selection and the attention in one persistent kernel (one CTA per
 * SM, cooperative launch): the summaries, the window and compressed tokens and the selected blocks
 * are read back to back, and a unit's selected blocks are read as soon as its selection is
 * complete; after a grid barrier every CTA folds a share of the split-K partial results. Results
 * are those of cobs_decode_step. It is an alternative schedule of the same work: on the seeded
 * decode workloads it measures slower than cobs_decode_step.
 * Takes bf16, d in {64, 128}, block 64 and the COBS_VAR_CHANNEL or COBS_VAR_ISOTROPIC summaries
 * (when its per-CTA tables fit in shared memory); other shapes return COBS_ERR_UNSUPPORTED.
 *   workspace: >= cobs_workspace_bytes(p, COBS_WS_STEP_FUSED) bytes (sized for the current
 *              device's SM count), ZERO-FILLED before its first use and again before it is used
 *              with other params or after a call that set the device error flag; a completed call
 *              leaves it ready for the next one. Calls that share one workspace must not run
 *              concurrently.
 * Errors: those of cobs_decode_step. A wait on another CTA's result is bounded: if it gives up
 * (kernel resources held by other work for more than about 0.1 s), the device error flag is set.
 */
cobs_status cobs_decode_step_fused(const cobs_params* p, const void* Q, const void* K,
                                   const void* V, const float* Pk, const float* Pv,
                                   int32_t t_begin, float* summaries, void* Kc, void* Vc,
                                   int32_t* idx, const float* gates, void* O, void* workspace,
                                   size_t ws_bytes, cobs_stream_t stream);

/*
 * Decode attention without a workspace. The paper has no counterpart to this call: it exists
 * for callers that cannot hand the library any device memory of its own, such as a host
 * program whose allocations all go through a pool it has already carved up, or a plug-in
 * whose host forbids device allocations after start-up. It computes exactly what
 * cobs_sparse_attn_decode computes, with the split-K partial results kept in a scratch array
 * built into the library (8 MiB, one per device that loads the library, held until the
 * process exits) and no allocation of any kind.
 *   - Problems whose partials need more than 8 MiB (cobs_workspace_bytes(p, COBS_WS_DECODE))
 *     are rejected with COBS_ERR_WORKSPACE before anything is launched.
 *   - The first call on each device looks up the scratch array's device address (with that
 *     device current); make that first call before any stream capture begins.
 *   - Every call on a device shares the one array and it keeps the last call's contents
 *     (nothing in it needs clearing). Calls whose kernels overlap on the GPU, for example
 *     on two streams without ordering between them, race on it: order them.
 * Other arguments, layouts and errors are those of cobs_sparse_attn_decode.
 */
cobs_status cobs_sparse_attn_decode_noalloc(const cobs_params* p, const void* Q, const void* K,
                                            const void* V, const void* Kc, const void* Vc,
                                            const int32_t* idx, const float* gates, void* O,
                                            cobs_stream_t stream);

/*
 * Causal prefill attention: the decode computation at every position t = 0 .. T-1, with
 * the window tokens max(0, t-W+1) .. t, the compressed tokens i with
 * cmp_stride*i + cmp_block - 1 <= t, and the selected blocks idx[b, t, g, :].
 *   Q, gates, O, idx in their prefill layouts.
 *   workspace: >= cobs_workspace_bytes(p, COBS_WS_PREFILL) bytes (may be 0).
 */
cobs_status cobs_sparse_attn_prefill(const cobs_params* p, const void* Q, const void* K,
                                     const void* V, const void* Kc, const void* Vc,
                                     const int32_t* idx, const float* gates, void* O,
                                     void* workspace, size_t ws_bytes, cobs_stream_t stream);

/*
 * The query subspace for COBS_VAR_SUBSPACE(_FP4) from a sample of queries ([COBS] §2.3: the
 * covariance is kept in the subspace spanned by the top eigenvectors of the queries' second
 * moment). M = (1/n) sum_i q_i q_i^T over the n rows of Q [n, d] (storage type of p->dtype; any
 * query vectors, for example a prefill's Q [B, T, Hq, d] as n = B T Hq rows), accumulated in
 * float32 per range of rows and summed over the ranges in double; then a cyclic Jacobi
 * eigendecomposition of M in float32 on the GPU.
 *   basis       [d, p->sub] float32 (row-major, the layout of cobs_params.basis): the
 *               eigenvectors of the p->sub largest eigenvalues as orthonormal columns, in
 *               descending eigenvalue order, each with its largest-magnitude entry positive.
 *   eigenvalues [p->sub] float32 in the same order, or NULL.
 *   workspace   >= cobs_workspace_bytes(p, COBS_WS_BASIS) bytes (sized for the current
 *               device's SM count); no initial contents are needed.
 * Only p->d, p->dtype and p->sub are used (the rest must still validate). Errors:
 * COBS_ERR_UNSUPPORTED unless p->sub is a multiple of 4 in 4 .. d; COBS_ERR_INVALID_ARG for
 * n < 1 or NULL / misaligned pointers; COBS_ERR_WORKSPACE. Eigenvectors of eigenvalues that
 * (nearly) coincide are any orthonormal basis of their eigenspace; the spanned subspace is
 * well defined when the p->sub-th and (p->sub + 1)-th eigenvalues are apart.
 */
cobs_status cobs_query_basis(const cobs_params* p, const void* Q, int64_t n, float* basis,
                             float* eigenvalues, void* workspace, size_t ws_bytes,
                             cobs_stream_t stream);

/*
 * Evaluation only (no step of the decode or prefill path calls it): the log of the exact
 * attention mass of every complete key block for the decode query at T - 1 ([COBS] §2.1,
 * "attention mass" and the oracle sparse attention OSA that keeps the blocks of largest mass),
 *   out[b, h, j] = ln sum_{r = 64 j}^{64 j + 63} exp(q_{b,h} . k_{b,h/G,r} / sqrt(d)),
 * for j < T / 64, in float32 (fused multiply-adds in ascending channel order, then
 * max + ln(sum exp(s - max)) over the block's 64 keys).
 *   Q [B, Hq, d] and K [B, Hkv, T, d] in the storage type of p->dtype; out [B, Hq, T / 64]
 *   float32, caller-owned device memory. Nothing is written when T < 64.
 *   Errors: the validation of the other calls; COBS_ERR_UNSUPPORTED when Hq / Hkv > 16.
 */
cobs_status cobs_block_log_mass(const cobs_params* p, const void* Q, const void* K, float* out,
                                cobs_stream_t stream);

/* Bytes of workspace a call needs (0 for an invalid p). */
size_t cobs_workspace_bytes(const cobs_params* p, int32_t which);

/* Number of float32 elements of the summaries tensor. */
size_t cobs_summaries_elems(const cobs_params* p);

/* Static text for a status code. */
const char* cobs_status_string(cobs_status s);

/* Message of the last failed call on this host thread ("" if none). */
const char* cobs_last_error(void);

/*
 * Device error flag of the current device: 0 if no kernel met an out-of-range index or
 * gave up a bounded wait since the last reset, else a nonzero code. Synchronises the
 * current device. reset != 0 clears the flag.
 */
int32_t cobs_device_error(int32_t reset);

/* Kernel launches this library has issued in this process (all host threads); reset != 0
 * sets the count back to zero after reading it. */
int64_t cobs_launch_count(int32_t reset);

/* ABI version (major * 100 + minor). */
int32_t cobs_version(void);

#ifdef __cplusplus
}
#endif
#endif /* COBS_H_ */
