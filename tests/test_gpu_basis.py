"""GPU parity of the query-subspace basis estimated from queries (cobs_query_basis) against the
oracle's float64 eigendecomposition of the same queries' second moment. The float32 Jacobi solver
reaches the same subspace (projectors P P^T within 2e-4), eigenvalues (relative 1e-4) and
orthonormal columns; well-separated columns match the oracle's column for column, sign included."""
import numpy as np
import pytest
import torch

import synth
from oracle import cobs_oracle as O
from gpu_common import cobs, dev, params_of

pytestmark = pytest.mark.gpu


def _planted(rng, n, d, s0, scales, noise):
    P0, _ = np.linalg.qr(rng.standard_normal((d, s0)))
    return ((rng.standard_normal((n, s0)) * scales) @ P0.T + noise * rng.standard_normal((n, d))).astype(np.float32)


def _check(Qrows, w, s, dtype, proj_tol=2e-4):
    C = cobs()
    p = params_of(w.replace(dtype=dtype))
    p.sub = s
    p.variance = "subspace"
    stored = Qrows if dtype == "f32" else synth.f32_to_bf16(Qrows)   # the storage form both sides read
    tQ = dev(stored, dtype)
    Q64 = synth.to_f64(stored, dtype)
    basis, evals = C.query_basis(p, tQ)
    torch.cuda.synchronize()
    P = basis.double().cpu().numpy()
    lam = evals.double().cpu().numpy()
    Pr, lr = O.query_basis(Q64, s)
    assert np.abs(P.T @ P - np.eye(s)).max() < 1e-5
    assert np.allclose(lam, lr, rtol=1e-4, atol=1e-6 * abs(lr[0]))
    assert np.abs(P @ P.T - Pr @ Pr.T).max() < proj_tol
    # columns whose eigenvalue is well apart from its neighbours: the same vector, same sign
    gaps = np.minimum(np.abs(np.diff(np.r_[np.inf, lr])), np.abs(np.diff(np.r_[lr, -np.inf])))
    for k in range(s):
        if gaps[k] > 0.05 * abs(lr[0]):
            assert np.abs(P[:, k] - Pr[:, k]).max() < 1e-3, k
    return P, lam


@pytest.mark.parametrize("d,s,dtype", [(128, 84, "bf16"), (128, 16, "f32"), (64, 32, "bf16"), (64, 4, "f32")])
def test_query_basis_matches_oracle_on_a_planted_subspace(d, s, dtype):
    rng = np.random.default_rng(91 + d + s)
    s0 = min(s, 12)
    Q = _planted(rng, 20000, d, s0, np.linspace(3.0, 1.0, s0), 0.2)
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=1, Hq=4, T=1024, d=d)
    _check(Q, w, s, dtype)


def test_query_basis_of_an_exactly_diagonal_second_moment():
    """Rows +-c_k u_k (float32): the basis is the u_k of the largest c_k."""
    rng = np.random.default_rng(97)
    d, s = 128, 84
    U, _ = np.linalg.qr(rng.standard_normal((d, d)))
    c = np.linspace(3.0, 0.5, d)
    rows = np.concatenate([c[:, None] * U.T, -c[:, None] * U.T]).astype(np.float32)
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=1, Hq=4, T=1024)
    P, lam = _check(rows, w, s, "f32")
    Uf = U.astype(np.float32).astype(np.float64)
    for k in range(s):
        u = Uf[:, k] * np.sign(Uf[np.argmax(np.abs(Uf[:, k])), k])
        assert np.abs(P[:, k] - u).max() < 1e-4, k


def test_query_basis_from_prefill_queries_drives_the_subspace_selection():
    """The basis estimated on the GPU from a prefill's queries feeds the subspace summaries: the
    stored coordinates are those the oracle computes with that same basis (the basis is an input of
    the summary step), bit for bit."""
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=4096)
    P0 = synth.subspace_basis(w, 84)
    Qpre = synth.queries_decode_subspace(w.replace(B=64), P0)   # [64, Hq, d] sample of queries
    p = params_of(w)
    p.sub, p.variance = 84, "subspace"
    basis, _ = C.query_basis(p, dev(Qpre, w.dtype))
    torch.cuda.synchronize()
    Pg = basis.cpu().numpy()
    Pr, _ = O.query_basis(synth.to_f64(Qpre, w.dtype).reshape(-1, w.d), 84)
    assert np.abs(Pg.astype(np.float64) @ Pg.T - Pr @ Pr.T).max() < 2e-3
    from gpu_common import inputs_decode, run_decode, summaries_blocks
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p2, buf = run_decode(w, K, V, Q, g, Pk, Pv, variance="subspace", rank=4, basis=Pg)
    assert C.device_error() == 0
    _, ut_g, _ = summaries_blocks(buf.summaries, p2)
    for h in range(w.Hkv):
        ref = O.canonical_summaries_subspace(synth.to_f64(K[0, h], w.dtype).astype(np.float32), w.block, 4, Pg)
        assert np.array_equal(ut_g[0, h], ref[1])


def test_query_basis_argument_errors():
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=1, Hq=4, T=1024)
    p = params_of(w)
    p.variance = "subspace"   # the binding passes sub for the subspace forms
    Q = torch.zeros((64, w.d), dtype=torch.bfloat16, device="cuda")
    basis = torch.empty((w.d, 84), dtype=torch.float32, device="cuda")
    ws = torch.empty(C.workspace_bytes(p, C.COBS_WS_BASIS), dtype=torch.uint8, device="cuda")
    p.sub = 82
    with pytest.raises(C.CobsError) as ei:
        C.cobs_query_basis(p, Q, 64, basis, None, ws)
    assert ei.value.status == -2
    p.sub = 84
    with pytest.raises(C.CobsError) as ei:
        C.cobs_query_basis(p, Q, 0, basis, None, ws)
    assert ei.value.status == -1
    with pytest.raises(C.CobsError) as ei:
        C.cobs_query_basis(p, Q, 64, basis, None, ws[:1024])
    assert ei.value.status == -4
