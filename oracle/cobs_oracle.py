"""ORACLE (test infrastructure): float64 restatement of COBS block-sparse attention.

Sources, cited per function below:

* [COBS] "COBS: Cumulant Order Block Sparse Attention" — gist.science explainer of
  arXiv 2607.09052: §2.1 (attention mass, oracle sparse attention), §2.2 (cumulant
  expansion of the log mass), §2.3 (second-order scoring on the NSA architecture, NoPE).
* [SKILL] "cumulant-order-block-sparse-attention" skill card: "Method" and
  "Implementation steps" (score = first-order term + alpha * cumulant term, top-k,
  the other branches unchanged).
* [NSA-181] deepseek-ai/Janus issue #181, "four dimensions regarding importance and
  connection strength": the three NSA paths (compression, selection, sliding window)
  and their gate weights.

Readings of points the pages leave open (each one is also listed in the design notes):
the log mass carries the usual 1/sqrt(d) logit scale; the second-order statistic is
the per-channel population variance of the keys (the diagonal of the block covariance);
the constant ln L is dropped (it is the same for every complete block); the group score
is the sum of its heads' scores; candidates are the complete blocks at or before the
query position; an empty branch contributes zero; gates arrive post-sigmoid in the
order (compressed, selected, window). For the compressed covariance forms of [COBS] §2.3:
the low-rank eigenpairs come from a fixed float32 subspace iteration (pinned against
numpy's eigh); FP4 keeps one float32 scale max|u|/6 per eigenvector; the query-subspace
basis is given by the caller, and both the eigenvectors and the query heads are projected
on it; the three together (the form §4.1 reports) quantize the projected coordinates with
the same FP4 rule and keep the mean in bf16.

Nothing here is blocked, fused or reordered: each function follows the definition it
cites, with numpy's matmul, sum and sort as the only library steps.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_C_SRC = os.path.join(_HERE, "canonical_fp32.c")
_C_LIB = os.path.join(_HERE, "libcobs_oracle.so")
_clib = None


# ----------------------------------------------------------------------------------
# float32 canonical selector (C)
# ----------------------------------------------------------------------------------

def build(force: bool = False) -> str:
    """Compile the float32 canonical selector (plain C, gcc)."""
    if force or not os.path.exists(_C_LIB) or os.path.getmtime(_C_LIB) < os.path.getmtime(_C_SRC):
        tmp = _C_LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _C_SRC, "-lm"])
        os.replace(tmp, _C_LIB)
    return _C_LIB


def _c():
    global _clib
    if _clib is None:
        build()
        lib = ctypes.CDLL(_C_LIB)
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        lib.cobs_oracle_summaries_f32.argtypes = [vp, i64, i32, i32, vp]
        lib.cobs_oracle_summaries_f32.restype = None
        lib.cobs_oracle_group_query_f32.argtypes = [vp, i32, i32, vp, vp]
        lib.cobs_oracle_group_query_f32.restype = None
        lib.cobs_oracle_score_constants.argtypes = [i32, f32, ctypes.POINTER(f32), ctypes.POINTER(f32)]
        lib.cobs_oracle_score_constants.restype = None
        lib.cobs_oracle_scores_f32.argtypes = [vp, vp, vp, i64, i64, i32, f32, f32, vp]
        lib.cobs_oracle_scores_f32.restype = None
        lib.cobs_oracle_iso_summaries_f32.argtypes = [vp, i64, i32, vp]
        lib.cobs_oracle_iso_summaries_f32.restype = None
        lib.cobs_oracle_iso_scores_f32.argtypes = [vp, vp, vp, i64, i64, i32, f32, f32, vp]
        lib.cobs_oracle_iso_scores_f32.restype = None
        lib.cobs_oracle_lowrank_f32.argtypes = [vp, vp, i64, i32, i32, i32, vp, vp]
        lib.cobs_oracle_lowrank_f32.restype = None
        lib.cobs_oracle_lowrank_scores_f32.argtypes = [vp, vp, i32, vp, vp, vp, i64, i32, i32, f32, f32, vp]
        lib.cobs_oracle_lowrank_scores_f32.restype = None
        lib.cobs_oracle_lowrank_fp4_f32.argtypes = [vp, vp, i64, i32, i32, vp, vp, vp, vp]
        lib.cobs_oracle_lowrank_fp4_f32.restype = None
        lib.cobs_oracle_e2m1_code.argtypes = [f32]
        lib.cobs_oracle_e2m1_code.restype = i32
        lib.cobs_oracle_bf16_rn.argtypes = [f32]
        lib.cobs_oracle_bf16_rn.restype = f32
        lib.cobs_oracle_subspace_project.argtypes = [vp, vp, i64, i32, i32, vp]
        lib.cobs_oracle_subspace_project.restype = None
        lib.cobs_oracle_subspace_scores.argtypes = [vp, vp, i32, vp, vp, vp, i64, i32, i32, i32, vp, f32, f32, vp]
        lib.cobs_oracle_subspace_scores.restype = None
        lib.cobs_oracle_fp4_vectors.argtypes = [vp, i64, i32, vp, vp, vp]
        lib.cobs_oracle_fp4_vectors.restype = None
        lib.cobs_oracle_subspace_fp4_f32.argtypes = [vp, vp, i64, i32, i32, i32, vp, vp, vp, vp]
        lib.cobs_oracle_subspace_fp4_f32.restype = None
        _clib = lib
    return _clib


def _f32c(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def canonical_summaries(K32: np.ndarray, L: int) -> np.ndarray:
    """float32 block summaries [nB, 2, d] (mean, variance) of key rows K32 [T, d].

    [COBS] §2.2: kappa_1 is the block mean of the keys; kappa_2 is their covariance,
    here its diagonal (per-channel population variance). Canonical float32 order: see
    canonical_fp32.c.
    """
    K32 = _f32c(K32)
    T, d = K32.shape
    nB = T // L
    out = np.zeros((nB, 2, d), np.float32)
    if nB:
        _c().cobs_oracle_summaries_f32(K32.ctypes.data, T, d, L, out.ctypes.data)
    return out


def canonical_group_query(q32: np.ndarray):
    """Sum and sum of squares over the query heads of one GQA group, float32 canonical.

    q32: [..., G, d] -> (qsum, q2) each [..., d].
    """
    q32 = _f32c(q32)
    G, d = q32.shape[-2:]
    lead = q32.shape[:-2]
    flat = q32.reshape(-1, G, d)
    qs = np.empty((flat.shape[0], d), np.float32)
    q2 = np.empty((flat.shape[0], d), np.float32)
    lib = _c()
    for i in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[i])
        a = np.empty(d, np.float32)
        b = np.empty(d, np.float32)
        lib.cobs_oracle_group_query_f32(row.ctypes.data, G, d, a.ctypes.data, b.ctypes.data)
        qs[i], q2[i] = a, b
    return qs.reshape(lead + (d,)), q2.reshape(lead + (d,))


def score_constants(d: int, alpha: float):
    """(isd, c2) = (RN32(1/sqrt(d)), RN32(alpha/(2d))) as float32."""
    isd, c2 = ctypes.c_float(), ctypes.c_float()
    _c().cobs_oracle_score_constants(d, ctypes.c_float(alpha), ctypes.byref(isd), ctypes.byref(c2))
    return np.float32(isd.value), np.float32(c2.value)


def canonical_scores(qsum: np.ndarray, q2: np.ndarray, summ: np.ndarray, alpha: float) -> np.ndarray:
    """float32 group scores S [nq, nB] of group queries against block summaries.

    [COBS] §2.3 second-order score q.k_b + 1/2 q^T Sigma_b q, with the logit scale and
    the diagonal covariance; [SKILL] "Implementation steps" 3: first-order term plus
    alpha times the cumulant term. Summed over the heads of the group.
    """
    qsum = _f32c(qsum).reshape(-1, summ.shape[-1])
    q2 = _f32c(q2).reshape(-1, summ.shape[-1])
    summ = _f32c(summ)
    nq, d = qsum.shape
    nb = summ.shape[0]
    isd, c2 = score_constants(d, alpha)
    S = np.empty((nq, nb), np.float32)
    if nq and nb:
        _c().cobs_oracle_scores_f32(qsum.ctypes.data, q2.ctypes.data, summ.ctypes.data, nq, nb, d,
                                    float(isd), float(c2), S.ctypes.data)
    return S


def canonical_summaries_iso(K32: np.ndarray, L: int) -> np.ndarray:
    """float32 isotropic block summaries [nB, d + 1]: the block mean, then the mean over channels
    of the per-channel population variance (one second-order scalar per block).

    [COBS] §2.2/§2.3 (the block covariance kappa_2 = Sigma_b, compressed); [SKILL] "Pitfalls"
    (one or two scalars per block): Sigma_b taken as sigma2_b I, sigma2_b = tr(Sigma_b) / d.
    Canonical float32 order: see canonical_fp32.c.
    """
    summ = canonical_summaries(K32, L)
    nB, _, d = summ.shape
    out = np.zeros((nB, d + 1), np.float32)
    if nB:
        _c().cobs_oracle_iso_summaries_f32(summ.ctypes.data, nB, d, out.ctypes.data)
    return out


def canonical_scores_iso(qsum: np.ndarray, q2: np.ndarray, summ_iso: np.ndarray, alpha: float) -> np.ndarray:
    """float32 group scores S [nq, nB] with isotropic summaries [nB, d + 1]:
    (sum_c Qsum_c mu_c) isd + c2 (sum_c Q2_c) sigma2_b. Canonical order: see canonical_fp32.c."""
    d = summ_iso.shape[-1] - 1
    qsum = _f32c(qsum).reshape(-1, d)
    q2 = _f32c(q2).reshape(-1, d)
    summ_iso = _f32c(summ_iso)
    nq, nb = qsum.shape[0], summ_iso.shape[0]
    isd, c2 = score_constants(d, alpha)
    S = np.empty((nq, nb), np.float32)
    if nq and nb:
        _c().cobs_oracle_iso_scores_f32(qsum.ctypes.data, q2.ctypes.data, summ_iso.ctypes.data, nq, nb, d,
                                        float(isd), float(c2), S.ctypes.data)
    return S


class LowRank(tuple):
    """Low-rank block summaries: (mu [nB, d], u [nB, R, d], lam [nB, R]), float32."""


def canonical_summaries_lowrank(K32: np.ndarray, L: int, R: int) -> LowRank:
    """float32 low-rank summaries: the block mean and the R leading eigenpairs of the block
    covariance from the fixed float32 solver of canonical_fp32.c.

    [COBS] §2.2/§2.3: the second cumulant kappa_2 = Sigma_b kept as its leading eigenpairs
    (the low-rank compression of the block covariance).
    """
    K32 = _f32c(K32)
    T, d = K32.shape
    nB = T // L
    mu = np.ascontiguousarray(canonical_summaries(K32, L)[:, 0, :])
    u = np.zeros((nB, R, d), np.float32)
    lam = np.zeros((nB, R), np.float32)
    if nB:
        _c().cobs_oracle_lowrank_f32(K32.ctypes.data, mu.ctypes.data, nB, d, L, R, u.ctypes.data, lam.ctypes.data)
    return LowRank((mu, u, lam))


class LowRankFP4(tuple):
    """FP4 low-rank summaries: (mu_q [nB, d] bf16 values as float32, codes [nB, R, d] uint8,
    scales [nB, R] float32, lam [nB, R] float32, u_q [nB, R, d] the dequantized vectors)."""

    def dequantized(self) -> LowRank:
        mu_q, _, _, lam, u_q = self
        return LowRank((mu_q, u_q, lam))


def e2m1_code(x: float) -> int:
    """E2M1 (FP4) code of x: nearest magnitude of {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even
    index, saturating; sign in bit 3 (canonical_fp32.c)."""
    return int(_c().cobs_oracle_e2m1_code(float(x)))


def canonical_summaries_lowrank_fp4(K32: np.ndarray, L: int, R: int) -> LowRankFP4:
    """The low-rank summaries with the mean rounded to bf16 and each eigenvector stored in E2M1
    with one float32 scale (max |u| / 6) ([COBS] §2.3: FP4 eigenvectors, BF16 mean)."""
    mu, u, lam = canonical_summaries_lowrank(K32, L, R)
    nB, d = mu.shape
    mu_q = np.zeros_like(mu)
    codes = np.zeros((nB, R, d), np.uint8)
    scales = np.zeros((nB, R), np.float32)
    u_q = np.zeros_like(u)
    if nB:
        _c().cobs_oracle_lowrank_fp4_f32(mu.ctypes.data, np.ascontiguousarray(u).ctypes.data, nB, d, R,
                                         mu_q.ctypes.data, codes.ctypes.data, scales.ctypes.data, u_q.ctypes.data)
    return LowRankFP4((mu_q, codes, scales, lam, u_q))


class Subspace(tuple):
    """Query-subspace low-rank summaries: (mu [nB, d], ut [nB, R, s] = P^T u_j, lam [nB, R], P [d, s])."""


def canonical_summaries_subspace(K32: np.ndarray, L: int, R: int, P: np.ndarray) -> Subspace:
    """The low-rank summaries with each eigenvector kept as its s coordinates in the query
    subspace spanned by the orthonormal columns of P ([COBS] §2.3: query-subspace projection,
    r d -> r s numbers per block). Canonical float32 order: canonical_fp32.c."""
    mu, u, lam = canonical_summaries_lowrank(K32, L, R)
    P = _f32c(P)
    d, sdim = P.shape
    nB = mu.shape[0]
    ut = np.zeros((nB, R, sdim), np.float32)
    if nB:
        _c().cobs_oracle_subspace_project(P.ctypes.data, np.ascontiguousarray(u).ctypes.data, nB * R, d, sdim,
                                          ut.ctypes.data)
    return Subspace((mu, ut, lam, P))


def fp4_vectors(x: np.ndarray):
    """E2M1 form of the rows of x [n, len] (one scale per row, canonical_fp32.c): (codes uint8,
    scales float32 [n], dequantized float32 [n, len])."""
    x = _f32c(x)
    n, ln = x.shape
    codes = np.zeros((n, ln), np.uint8)
    scales = np.zeros(n, np.float32)
    xq = np.zeros((n, ln), np.float32)
    if n:
        _c().cobs_oracle_fp4_vectors(x.ctypes.data, n, ln, codes.ctypes.data, scales.ctypes.data, xq.ctypes.data)
    return codes, scales, xq


class SubspaceFP4(tuple):
    """Query-subspace summaries with FP4 coordinates: (mu_q [nB, d] bf16 values as float32, codes
    [nB, R, s] uint8, scales [nB, R] float32, lam [nB, R] float32, ut_q [nB, R, s] the dequantized
    coordinates, P [d, s])."""

    def dequantized(self) -> Subspace:
        mu_q, _, _, lam, ut_q, P = self
        return Subspace((mu_q, ut_q, lam, P))


def canonical_summaries_subspace_fp4(K32: np.ndarray, L: int, R: int, P: np.ndarray) -> SubspaceFP4:
    """The query-subspace summaries with the mean rounded to bf16 and each projected eigenvector's
    s coordinates stored in E2M1 with one float32 scale (max |u~| / 6): the three compressions of
    [COBS] §2.3 together, the form [COBS] §4.1 reports as "Subspace, r=4, FP4"."""
    mu, ut, lam, P = canonical_summaries_subspace(K32, L, R, P)
    nB, d = mu.shape
    sdim = ut.shape[2]
    mu_q = np.zeros_like(mu)
    codes = np.zeros((nB, R, sdim), np.uint8)
    scales = np.zeros((nB, R), np.float32)
    ut_q = np.zeros_like(ut)
    if nB:
        _c().cobs_oracle_subspace_fp4_f32(mu.ctypes.data, np.ascontiguousarray(ut).ctypes.data, nB, d, sdim, R,
                                          mu_q.ctypes.data, codes.ctypes.data, scales.ctypes.data, ut_q.ctypes.data)
    return SubspaceFP4((mu_q, codes, scales, lam, ut_q, P))


def canonical_scores_subspace(q_group32: np.ndarray, summ: Subspace, alpha: float) -> np.ndarray:
    """float32 group scores [nB] with query-subspace summaries (canonical_fp32.c)."""
    mu, ut, lam, P = summ
    q = _f32c(q_group32)
    G, d = q.shape
    qs, _ = canonical_group_query(q)
    isd, c2 = score_constants(d, alpha)
    S = np.empty(mu.shape[0], np.float32)
    if mu.shape[0]:
        _c().cobs_oracle_subspace_scores(q.ctypes.data, _f32c(qs).ctypes.data, G, _f32c(mu).ctypes.data,
                                         _f32c(ut).ctypes.data, _f32c(lam).ctypes.data, mu.shape[0], d,
                                         ut.shape[2], ut.shape[1], _f32c(P).ctypes.data, float(isd), float(c2),
                                         S.ctypes.data)
    return S


def canonical_scores_lowrank(q_group32: np.ndarray, summ: LowRank, alpha: float) -> np.ndarray:
    """float32 group scores [nB] of one group's query heads [G, d] against low-rank summaries:
    (sum_c Qsum_c mu_c) isd + c2 sum_j lam_j sum_h (q_h . u_j)^2. Canonical order: canonical_fp32.c."""
    mu, u, lam = summ
    q = _f32c(q_group32)
    G, d = q.shape
    qs, _ = canonical_group_query(q)
    qs = _f32c(qs)
    isd, c2 = score_constants(d, alpha)
    S = np.empty(mu.shape[0], np.float32)
    if mu.shape[0]:
        _c().cobs_oracle_lowrank_scores_f32(q.ctypes.data, qs.ctypes.data, G, _f32c(mu).ctypes.data,
                                            _f32c(u).ctypes.data, _f32c(lam).ctypes.data, mu.shape[0], d,
                                            u.shape[1], float(isd), float(c2), S.ctypes.data)
    return S


# ----------------------------------------------------------------------------------
# float64 steps
# ----------------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even), returned as float64."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def block_summaries(K: np.ndarray, L: int):
    """Block mean mu [nB, d] and per-channel population variance var [nB, d], float64.

    [COBS] §2.2: kappa_1 = block mean of the keys, kappa_2 = block covariance of the keys
    (here its diagonal: var_{b,c} = (1/L) sum_r (k_{r,c} - mu_{b,c})^2). Complete blocks only.
    """
    T, d = K.shape
    nB = T // L
    mu = np.zeros((nB, d))
    var = np.zeros((nB, d))
    for b in range(nB):
        rows = K[b * L:(b + 1) * L]
        mu[b] = rows.sum(axis=0) / L
        var[b] = ((rows - mu[b]) ** 2).sum(axis=0) / L
    return mu, var


def compressed_tokens(X: np.ndarray, P, lc: int, sc: int, dtype: str) -> np.ndarray:
    """Compressed tokens [nC, d]: P @ (mean of rows sc*i .. sc*i+lc-1), i < nC.

    [NSA-181] Compression Path (CMP): blocks aggregated into coarse tokens; [SKILL]
    "Implementation steps" 4: the compression branch is unchanged by COBS. The aggregation
    is a mean-pool followed by a linear map P (identity when P is None); bf16 workloads
    store the compressed tokens in bf16.
    """
    T, d = X.shape
    nC = (T - lc) // sc + 1 if T >= lc else 0
    out = np.zeros((nC, d))
    for i in range(nC):
        m = X[sc * i:sc * i + lc].sum(axis=0) / lc
        out[i] = m if P is None else np.asarray(P, np.float64) @ m
    return round_bf16(out) if dtype == "bf16" else out


def head_scores(q: np.ndarray, mu: np.ndarray, var: np.ndarray, alpha: float) -> np.ndarray:
    """Per-head score of every block: q.mu_b/sqrt(d) + alpha * 1/2 * sum_c q_c^2 var_{b,c} / d.

    [COBS] §2.2 truncated after the second cumulant with logits q.k/sqrt(d): the linear
    term is q^T kappa_1 / sqrt(d) and the quadratic term 1/2 q^T kappa_2 q / d; ln L dropped.
    """
    d = q.shape[-1]
    first = (mu @ q) / np.sqrt(d)
    second = 0.5 * (var @ (q * q)) / d
    return first + alpha * second


def group_scores(qs: np.ndarray, mu: np.ndarray, var: np.ndarray, alpha: float) -> np.ndarray:
    """Group score of every block: sum of head_scores over the G query heads qs [G, d].

    Reading: one selection per GQA group (shared by its heads) ranks blocks by the sum
    of the heads' log-mass estimates.
    """
    return sum(head_scores(q, mu, var, alpha) for q in qs)


def head_scores_iso(q: np.ndarray, mu: np.ndarray, sigma2: np.ndarray, alpha: float) -> np.ndarray:
    """Isotropic per-head score: q.mu_b/sqrt(d) + alpha * 1/2 * sigma2_b |q|^2 / d.

    The second cumulant 1/2 q^T Sigma_b q / d of [COBS] §2.2 with Sigma_b = sigma2_b I
    ([SKILL] "Pitfalls": one scalar per block), sigma2_b = mean over channels of var_{b,c}.
    """
    d = q.shape[-1]
    return (mu @ q) / np.sqrt(d) + alpha * 0.5 * sigma2 * float(q @ q) / d


def group_scores_iso(qs: np.ndarray, mu: np.ndarray, sigma2: np.ndarray, alpha: float) -> np.ndarray:
    """Sum of head_scores_iso over the G query heads qs [G, d] (the group-sum reading)."""
    return sum(head_scores_iso(q, mu, sigma2, alpha) for q in qs)


def block_eigenpairs(K: np.ndarray, L: int, R: int):
    """Block mean mu [nB, d] and the R leading eigenpairs (u [nB, R, d], lam [nB, R]) of the
    population covariance Sigma_b = (1/L) sum_r (k_r - mu_b)(k_r - mu_b)^T, float64 (numpy eigh).

    [COBS] §2.2/§2.3: kappa_2 = Sigma_b, compressed to its leading eigenpairs.
    """
    T, d = K.shape
    nB = T // L
    mu = np.zeros((nB, d))
    u = np.zeros((nB, R, d))
    lam = np.zeros((nB, R))
    for b in range(nB):
        rows = K[b * L:(b + 1) * L]
        mu[b] = rows.sum(axis=0) / L
        Y = rows - mu[b]
        w, vecs = np.linalg.eigh(Y.T @ Y / L)
        order = np.argsort(-w, kind="stable")[:R]
        lam[b] = w[order]
        u[b] = vecs[:, order].T
    return mu, u, lam


def query_basis(Q: np.ndarray, s: int):
    """The query subspace of [COBS] §2.3: the eigenvectors of the queries' second moment
    M = (1/n) sum_i q_i q_i^T (rows of Q [n, d], float64) for its s largest eigenvalues, as the
    columns of P [d, s] in descending eigenvalue order (numpy's eigh), each column's sign fixed so
    that its largest-magnitude entry (the first such on ties) is positive. Returns (P, eigenvalues
    [s]).

    The pages say the subspace is spanned by the top eigenvectors of the query second moment but
    not how it is estimated: reading, the second moment of the sample of queries the caller
    passes (for example a prefill's queries)."""
    Q = np.asarray(Q, np.float64)
    n, d = Q.shape
    M = Q.T @ Q / n
    w, V = np.linalg.eigh(M)
    order = np.argsort(-w, kind="stable")[:s]
    P = V[:, order].copy()
    for k in range(s):
        i = int(np.argmax(np.abs(P[:, k])))
        if P[i, k] < 0:
            P[:, k] = -P[:, k]
    return P, w[order]


def head_scores_lowrank(q: np.ndarray, mu: np.ndarray, u: np.ndarray, lam: np.ndarray, alpha: float) -> np.ndarray:
    """Low-rank per-head score: q.mu_b/sqrt(d) + alpha * 1/2 * sum_j lam_j (q . u_j)^2 / d
    (the second cumulant 1/2 q^T Sigma_b q / d with Sigma_b ~ sum_j lam_j u_j u_j^T)."""
    d = q.shape[-1]
    return (mu @ q) / np.sqrt(d) + alpha * 0.5 * ((u @ q) ** 2 * lam).sum(axis=-1) / d


def group_scores_subspace(qs: np.ndarray, mu, u, lam, P, alpha: float) -> np.ndarray:
    """Query-subspace per-group score: sum_h [q_h.mu/sqrt(d) + alpha/2 sum_j lam_j ((P^T q_h).(P^T u_j))^2 / d]."""
    return group_scores_subspace_coords(qs, mu, u @ P, lam, P, alpha)


def group_scores_subspace_coords(qs: np.ndarray, mu, ut, lam, P, alpha: float) -> np.ndarray:
    """The same score from the eigenvectors' subspace coordinates ut [nB, R, s] as stored (for
    the FP4 form: the dequantized coordinates and the bf16 mean), float64."""
    d = qs.shape[-1]
    out = 0.0
    for q in qs:
        qp = P.T @ q
        out = out + (mu @ q) / np.sqrt(d) + alpha * 0.5 * ((ut @ qp) ** 2 * lam).sum(axis=-1) / d
    return out


def group_scores_lowrank(qs: np.ndarray, mu, u, lam, alpha: float) -> np.ndarray:
    """Sum of head_scores_lowrank over the G query heads qs [G, d] (the group-sum reading)."""
    return sum(head_scores_lowrank(q, mu, u, lam, alpha) for q in qs)


def n_candidates(t: int, L: int) -> int:
    """Candidate blocks for a query at position t: the complete blocks b with (b+1)L-1 <= t."""
    return (t + 1) // L


def top_k(S: np.ndarray, ncand: int, k: int) -> np.ndarray:
    """k best candidates by (score descending, block index ascending), returned ascending, -1 padded.

    [SKILL] "Method": retrieve the top-k blocks by the estimated mass.
    """
    cand = np.asarray(S[:ncand])
    order = np.argsort(-cand, kind="stable")   # stable: equal scores keep ascending index
    chosen = np.sort(order[:min(k, ncand)])
    out = np.full(k, -1, np.int32)
    out[:len(chosen)] = chosen
    return out


def attend(q: np.ndarray, Ks: np.ndarray, Vs: np.ndarray) -> np.ndarray:
    """softmax(q K^T / sqrt(d)) V over the given keys; zero vector when there are none."""
    d = q.shape[-1]
    if Ks.shape[0] == 0:
        return np.zeros(Vs.shape[-1])
    s = (Ks @ q) / np.sqrt(d)
    p = np.exp(s - s.max())
    return (p @ Vs) / p.sum()


def branch_tokens(t: int, idx: np.ndarray, L: int, W: int, lc: int, sc: int, nC: int):
    """Key index sets of the three branches for a query at position t.

    [NSA-181]: Selection Path (SLC) = tokens of the selected blocks; Sliding Window (WIN) =
    the W most recent tokens up to t; Compression Path (CMP) = compressed tokens whose
    source rows all lie at or before t.
    """
    slc = np.concatenate([np.arange(b * L, (b + 1) * L) for b in idx if b >= 0] or [np.zeros(0, int)])
    win = np.arange(max(0, t - W + 1), t + 1)
    ncv = 0 if t < lc - 1 else min(nC, (t - lc + 1) // sc + 1)
    cmp_ = np.arange(ncv)
    return slc.astype(int), win, cmp_


def position_output(qs, gates, K, V, Kc, Vc, idx, t, L, W, lc, sc) -> np.ndarray:
    """Outputs [G, d] of the G heads of one group at position t.

    o_h = g_cmp o_cmp + g_slc o_slc + g_win o_win ([NSA-181] gate weights; [COBS] §2.3: COBS
    keeps NSA's compression, selection and sliding-window branches).
    """
    slc, win, cmp_ = branch_tokens(t, idx, L, W, lc, sc, Kc.shape[0])
    out = np.zeros((qs.shape[0], V.shape[1]))
    for h, q in enumerate(qs):
        o_cmp = attend(q, Kc[cmp_], Vc[cmp_])
        o_slc = attend(q, K[slc], V[slc])
        o_win = attend(q, K[win], V[win])
        g = np.asarray(gates[h], np.float64)
        out[h] = g[0] * o_cmp + g[1] * o_slc + g[2] * o_win
    return out


def exact_log_mass(q: np.ndarray, K: np.ndarray, L: int) -> np.ndarray:
    """ln m_b = ln sum_{r in b} exp(q.k_r/sqrt(d)) for every complete block ([COBS] §2.1)."""
    d = q.shape[-1]
    nB = K.shape[0] // L
    s = (K[:nB * L] @ q).reshape(nB, L) / np.sqrt(d)
    mx = s.max(axis=1)
    return mx + np.log(np.exp(s - mx[:, None]).sum(axis=1))


def exact_group_score(qs: np.ndarray, K: np.ndarray, L: int) -> np.ndarray:
    """sum_h (ln m_{h,b} - ln L): the exact counterpart of group_scores."""
    return sum(exact_log_mass(q, K, L) - np.log(L) for q in qs)


def osa_top_k(qs, K, L, ncand, k) -> np.ndarray:
    """Oracle sparse attention selection: top-k by exact mass ([COBS] §2.1)."""
    return top_k(exact_group_score(qs, K, L), ncand, k)


def near_tie_gap(S64: np.ndarray, sel32: np.ndarray, ncand: int, k: int):
    """How far apart, in float64, the blocks are on which the float32 selection differs from
    the float64 one: None when both pick the same set, else the relative gap
    (max S64 over the float64-only picks - min S64 over the float32-only picks) / max(1, max |S64|).

    The float32 decision and the float64 ranking of the same definition ([COBS] §2.3 score,
    [SKILL] "Method" top-k) can differ only where float64 scores lie within float32 rounding of
    each other, so this gap is of the order of the float32 unit roundoff (about 1e-7) times the
    magnitude of the summed terms.
    """
    sel64 = top_k(S64, ncand, k)
    a = set(int(x) for x in sel64 if x >= 0)
    b = set(int(x) for x in sel32 if x >= 0)
    if a == b:
        return None
    S = np.asarray(S64[:ncand], np.float64)
    only64, only32 = sorted(a - b), sorted(b - a)
    hi = max(S[i] for i in only64) if only64 else -np.inf
    lo = min(S[i] for i in only32) if only32 else np.inf
    gap = max(0.0, hi - lo) if only64 and only32 else np.inf
    return float(gap / max(1.0, float(np.abs(S).max())))


def recall(sel: np.ndarray, ref: np.ndarray) -> float:
    a = set(int(x) for x in sel if x >= 0)
    b = set(int(x) for x in ref if x >= 0)
    return len(a & b) / max(1, len(b))


# ----------------------------------------------------------------------------------
# whole-path drivers
# ----------------------------------------------------------------------------------

def unit_cache(w, Kst: np.ndarray, Vst: np.ndarray, Pk, Pv):
    """Per-unit cache state: canonical float32 summaries and float64 compressed K/V.

    Kst, Vst: one unit's [T, d] keys/values in storage form (uint16 bf16 bits or float32).
    """
    K = _to_f64(Kst, w.dtype)
    V = _to_f64(Vst, w.dtype)
    summ = canonical_summaries(K.astype(np.float32), w.block)
    Kc = compressed_tokens(K, Pk, w.cmp_block, w.cmp_stride, w.dtype)
    Vc = compressed_tokens(V, Pv, w.cmp_block, w.cmp_stride, w.dtype)
    return K, V, summ, Kc, Vc


def select_decode(w, q_group32: np.ndarray, summ: np.ndarray):
    """Selected blocks [k] for the decode query at position T-1 of one (batch, group).

    summ: canonical summaries [nB, 2, d] (per-channel variance), [nB, d + 1] (isotropic) or a
    LowRank triple (mean, eigenvectors, eigenvalues)."""
    if isinstance(summ, SubspaceFP4):
        summ = summ.dequantized()
    if isinstance(summ, Subspace):
        S = canonical_scores_subspace(q_group32, summ, w.alpha)
        return top_k(S, n_candidates(w.T - 1, w.block), w.topk), S
    if isinstance(summ, LowRankFP4):
        summ = summ.dequantized()
    if isinstance(summ, LowRank):
        S = canonical_scores_lowrank(q_group32, summ, w.alpha)
        return top_k(S, n_candidates(w.T - 1, w.block), w.topk), S
    qs, q2 = canonical_group_query(q_group32)
    if summ.ndim == 2:
        S = canonical_scores_iso(qs[None], q2[None], summ, w.alpha)[0]
    else:
        S = canonical_scores(qs[None], q2[None], summ, w.alpha)[0]
    return top_k(S, n_candidates(w.T - 1, w.block), w.topk), S


def decode(w, K_all, V_all, Q, gates, Pk, Pv, units=None, variance="channel", rank=4, basis=None):
    """Decode at position T-1 for every (batch, KV head) unit (or the listed units).

    variance: "channel" (per-channel variance summaries), "isotropic" (one scalar per block),
    "lowrank" / "lowrank_fp4" (the rank leading eigenpairs of each block's covariance) or
    "subspace" (those eigenpairs with the eigenvectors as coordinates in basis [d, s]) or
    "subspace_fp4" (those coordinates in E2M1 with one scale per vector, the mean in bf16).

    Returns dict with idx [B, Hkv, k], O [B, Hq, d] (float64; rows of unlisted units are NaN),
    summ, Kc, Vc per computed unit, and near-tie reports (b, h, relative gap) for the units where
    the float64 ranking of the group score disagrees with the float32 canonical one (near_tie_gap).
    """
    G, t = w.G, w.T - 1
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)] if units is None else units
    idx = np.full((w.B, w.Hkv, w.topk), -1, np.int32)
    O = np.full((w.B, w.Hq, w.d), np.nan)
    cache = {}
    near_ties = []
    Qf = _to_f64(Q, w.dtype)
    for (b, h) in units:
        K, V, summ, Kc, Vc = unit_cache(w, K_all[b, h], V_all[b, h], Pk, Pv)
        cache[(b, h)] = (summ, Kc, Vc)
        qs = Qf[b, h * G:(h + 1) * G]
        if variance == "isotropic":
            sel_summ = canonical_summaries_iso(K.astype(np.float32), w.block)
        elif variance == "lowrank":
            sel_summ = canonical_summaries_lowrank(K.astype(np.float32), w.block, rank)
        elif variance == "lowrank_fp4":
            sel_summ = canonical_summaries_lowrank_fp4(K.astype(np.float32), w.block, rank)
        elif variance == "subspace":
            sel_summ = canonical_summaries_subspace(K.astype(np.float32), w.block, rank, basis)
        elif variance == "subspace_fp4":
            sel_summ = canonical_summaries_subspace_fp4(K.astype(np.float32), w.block, rank, basis)
        else:
            sel_summ = summ
        sel, _ = select_decode(w, qs.astype(np.float32), sel_summ)
        idx[b, h] = sel
        mu, var = block_summaries(K, w.block)
        if variance == "isotropic":
            S64 = group_scores_iso(qs, mu, var.mean(axis=1), w.alpha)
        elif variance in ("lowrank", "lowrank_fp4"):
            S64 = group_scores_lowrank(qs, *block_eigenpairs(K, w.block, rank), w.alpha)
        elif variance == "subspace":
            S64 = group_scores_subspace(qs, *block_eigenpairs(K, w.block, rank), np.asarray(basis, np.float64),
                                        w.alpha)
        elif variance == "subspace_fp4":  # the float64 score of the stored (quantized) form
            mu_q, _, _, lam_q, ut_q, _ = sel_summ
            S64 = group_scores_subspace_coords(qs, mu_q.astype(np.float64), ut_q.astype(np.float64),
                                               lam_q.astype(np.float64), np.asarray(basis, np.float64), w.alpha)
        else:
            S64 = group_scores(qs, mu, var, w.alpha)
        gap = near_tie_gap(S64, sel, n_candidates(t, w.block), w.topk)
        if gap is not None:
            near_ties.append((b, h, gap))
        O[b, h * G:(h + 1) * G] = position_output(qs, gates[b, h * G:(h + 1) * G], K, V, Kc, Vc, sel,
                                                  t, w.block, w.window, w.cmp_block, w.cmp_stride)
    return {"idx": idx, "O": O, "cache": cache, "near_ties": near_ties}


def select_prefill_unit(w, Qst_bh: np.ndarray, summ: np.ndarray, positions=None) -> np.ndarray:
    """Selected blocks [P, k] at every listed position (default all T) of one (batch, group).

    Qst_bh: the group's queries [T or P, G, d] in storage form, aligned with ``positions``.
    summ: canonical summaries [nB, 2, d] (per-channel variance) or [nB, d + 1] (isotropic).
    """
    pos = np.arange(w.T) if positions is None else np.asarray(positions)
    q32 = _to_f64(Qst_bh, w.dtype).astype(np.float32)
    qs, q2 = canonical_group_query(q32)
    nb_max = n_candidates(int(pos.max()), w.block) if len(pos) else 0
    scores = canonical_scores_iso if summ.ndim == 2 else canonical_scores
    S = scores(qs, q2, summ[:nb_max], w.alpha) if nb_max else np.zeros((len(pos), 0), np.float32)
    out = np.empty((len(pos), w.topk), np.int32)
    for i, t in enumerate(pos):
        out[i] = top_k(S[i], n_candidates(int(t), w.block), w.topk)
    return out


def prefill_positions(w, K_all, V_all, Qsub, gates_sub, Pk, Pv, positions, b=0):
    """Prefill outputs [P, Hq, d] and idx [P, Hkv, k] at the listed positions of batch row b.

    Qsub [P, Hq, d] and gates_sub [P, Hq, 3] hold the queries and gates of those positions.
    """
    G = w.G
    positions = np.asarray(positions)
    O = np.zeros((len(positions), w.Hq, w.d))
    idx = np.zeros((len(positions), w.Hkv, w.topk), np.int32)
    Qf = _to_f64(Qsub, w.dtype)
    for h in range(w.Hkv):
        K, V, summ, Kc, Vc = unit_cache(w, K_all[b, h], V_all[b, h], Pk, Pv)
        sel = select_prefill_unit(w, Qsub[:, h * G:(h + 1) * G], summ, positions)
        idx[:, h] = sel
        for i, t in enumerate(positions):
            O[i, h * G:(h + 1) * G] = position_output(Qf[i, h * G:(h + 1) * G], gates_sub[i, h * G:(h + 1) * G],
                                                      K, V, Kc, Vc, sel[i], int(t), w.block, w.window,
                                                      w.cmp_block, w.cmp_stride)
    return O, idx


def _to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of stored tensors (uint16 bfloat16 bit patterns or float32)."""
    if dtype == "bf16":
        u = np.ascontiguousarray(x, np.uint16).astype(np.uint32) << 16
        return u.view(np.float32).astype(np.float64)
    return np.asarray(x, np.float32).astype(np.float64)
