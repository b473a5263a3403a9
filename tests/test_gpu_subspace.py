"""GPU parity of the query-subspace low-rank selector (each block's leading covariance
eigenvectors kept as coordinates in a query subspace, the query heads projected on the same
basis) against the oracle: means, projected eigenvectors, eigenvalues and selected blocks bit for
bit, outputs within tolerance."""
import numpy as np
import pytest
import torch

import synth
from oracle import cobs_oracle as O
from gpu_common import TOL, cobs, dev, f64, inputs_decode, params_of, run_decode, summaries_blocks

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over,R,s", [
    ("tiny", dict(), 4, 16),                                             # float32, d = 64
    ("decode32k", dict(B=2, Hkv=2, Hq=8, T=4096), 4, 84),                 # bf16, d = 128, G = 4, s = 84
    ("decode32k", dict(B=1, Hkv=1, Hq=16, T=2048 + 37), 3, 32),           # G = 16, odd rank, ragged tail
    ("decode32k", dict(B=1, Hkv=2, Hq=2, d=64, T=3000, topk=32), 8, 64),  # d = 64, G = 1, rank 8, s = d
])
def test_subspace_decode_matches_oracle(name, over, R, s):
    w = synth.WORKLOADS[name].replace(**over)
    K, V, _, g, Pk, Pv = inputs_decode(w)
    P = synth.subspace_basis(w, s)
    Q = synth.queries_decode_subspace(w, P)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv, variance="subspace", rank=R, basis=P)
    assert cobs().device_error() == 0
    mu_g, ut_g, lam_g = summaries_blocks(buf.summaries, p)
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    Qf = synth.to_f64(Q, w.dtype)
    G = w.G
    for b in range(w.B):
        for h in range(w.Hkv):
            ref = O.canonical_summaries_subspace(synth.to_f64(K[b, h], w.dtype).astype(np.float32), w.block, R, P)
            assert np.array_equal(mu_g[b, h], ref[0]), f"means differ at {(b, h)}"
            assert np.array_equal(ut_g[b, h], ref[1]), f"projected eigenvectors differ at {(b, h)}"
            assert np.array_equal(lam_g[b, h], ref[2]), f"eigenvalues differ at {(b, h)}"
            qs = Qf[b, h * G:(h + 1) * G]
            sel, _ = O.select_decode(w, qs.astype(np.float32), ref)
            assert np.array_equal(idx_g[b, h], sel), f"idx {(b, h)}: {idx_g[b, h]} vs {sel}"
            Kf, Vf, _, Kc, Vc = O.unit_cache(w, K[b, h], V[b, h], Pk, Pv)
            out = O.position_output(qs, g[b, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, sel, w.T - 1, w.block, w.window,
                                    w.cmp_block, w.cmp_stride)
            assert np.abs(O_g[b, h * G:(h + 1) * G] - out).max() <= TOL[w.dtype]


def test_subspace_with_identity_basis_selects_as_low_rank():
    """P = I: the projected summaries are the low-rank eigenvectors and the selection is the
    low-rank selection, block for block."""
    w = synth.WORKLOADS["decode32k"].replace(B=2, Hkv=2, Hq=8, T=4096)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    I = np.eye(w.d, dtype=np.float32)
    p_s, buf_s = run_decode(w, K, V, Q, g, Pk, Pv, variance="subspace", rank=4, basis=I)
    _, buf_l = run_decode(w, K, V, Q, g, Pk, Pv, variance="lowrank", rank=4)
    assert torch.equal(buf_s.idx, buf_l.idx)
    assert torch.equal(buf_s.summaries, buf_l.summaries)   # same layout when s = d
    assert torch.equal(buf_s.O, buf_l.O)


@pytest.mark.parametrize("back", [1, 64])
def test_subspace_incremental_update_matches_full_build(back):
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=4096)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    P = synth.subspace_basis(w, 84)
    p = params_of(w, "subspace", 4, P)
    tK, tV, tPk, tPv = dev(K, w.dtype), dev(V, w.dtype), dev(Pk, "f32"), dev(Pv, "f32")
    full = C.alloc(p, prefill=False)
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, 0, full.summaries, full.Kc, full.Vc)
    inc = C.alloc(p, prefill=False)
    inc.summaries.copy_(full.summaries)
    nb = w.T // 64
    view = inc.summaries.view(p.B, p.Hkv, -1, 32 * (p.d + 4 * 84 + 4))
    view[:, :, (nb - 1) // 32] = float("nan")
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, w.T - back, inc.summaries, inc.Kc, inc.Vc)
    torch.cuda.synchronize()
    for a, b in zip(summaries_blocks(inc.summaries, p), summaries_blocks(full.summaries, p)):
        assert np.array_equal(a[:, :, nb - 1], b[:, :, nb - 1])


def test_subspace_argument_errors():
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=1, Hq=4, T=1024)
    P = synth.subspace_basis(w, 84)
    p = params_of(w, "subspace", 4, P)
    buf = C.alloc(p, prefill=False)
    Q = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    bad = params_of(w, "subspace", 4, P)
    bad.basis = None                       # NULL basis: rejected before any launch
    with pytest.raises(C.CobsError) as ei:
        C.cobs_select(bad, Q, buf.summaries, 0, buf.idx, buf.ws_select)
    assert ei.value.status == -1
    odd = params_of(w, "subspace", 4, synth.subspace_basis(w, 82))   # s not a multiple of 4
    with pytest.raises(C.CobsError) as ei:
        C.cobs_select(odd, Q, buf.summaries, 0, buf.idx, buf.ws_select)
    assert ei.value.status == -2
    with pytest.raises(C.CobsError) as ei:  # prefill selection is decode-only for the low-rank forms
        C.cobs_select(p, torch.zeros((w.B, w.T, w.Hq, w.d), dtype=torch.bfloat16, device="cuda"), buf.summaries,
                      1, buf.idx, buf.ws_select)
    assert ei.value.status == -2


# ---------------------------------------------------------------- FP4 coordinates, bf16 means

def _check_subspace_fp4(w, K, V, Q, g, Pk, Pv, p, buf, P, R, units, out_units):
    mu_g, codes_g, scales_g, lam_g = summaries_blocks(buf.summaries, p)
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    Qf = synth.to_f64(Q, w.dtype)
    G = w.G
    for (b, h) in units:
        ref = O.canonical_summaries_subspace_fp4(synth.to_f64(K[b, h], w.dtype).astype(np.float32), w.block, R, P)
        assert np.array_equal(mu_g[b, h], ref[0]), f"bf16 means differ at {(b, h)}"
        assert np.array_equal(codes_g[b, h], ref[1]), f"codes differ at {(b, h)}"
        assert np.array_equal(scales_g[b, h], ref[2]), f"scales differ at {(b, h)}"
        assert np.array_equal(lam_g[b, h], ref[3]), f"eigenvalues differ at {(b, h)}"
        qs = Qf[b, h * G:(h + 1) * G]
        sel, _ = O.select_decode(w, qs.astype(np.float32), ref)
        assert np.array_equal(idx_g[b, h], sel), f"idx {(b, h)}: {idx_g[b, h]} vs {sel}"
        if (b, h) in out_units:
            Kf, Vf, _, Kc, Vc = O.unit_cache(w, K[b, h], V[b, h], Pk, Pv)
            out = O.position_output(qs, g[b, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, sel, w.T - 1, w.block, w.window,
                                    w.cmp_block, w.cmp_stride)
            assert np.abs(O_g[b, h * G:(h + 1) * G] - out).max() <= TOL[w.dtype]


@pytest.mark.parametrize("name,over,R,s", [
    ("tiny", dict(), 4, 16),                                             # float32, d = 64
    ("decode32k", dict(B=2, Hkv=2, Hq=8, T=4096), 4, 84),                 # bf16, s = 84 (codes padded to 96)
    ("decode32k", dict(B=1, Hkv=1, Hq=16, T=2048 + 37), 3, 32),           # G = 16, odd rank, ragged tail
    ("decode32k", dict(B=1, Hkv=2, Hq=2, d=64, T=3000, topk=32), 8, 64),  # d = 64, G = 1, rank 8, s = d
    ("decode32k", dict(B=1, Hkv=1, Hq=4, T=4096), 2, 4),                  # the smallest subspace
])
def test_subspace_fp4_decode_matches_oracle(name, over, R, s):
    w = synth.WORKLOADS[name].replace(**over)
    K, V, _, g, Pk, Pv = inputs_decode(w)
    P = synth.subspace_basis(w, s)
    Q = synth.queries_decode_subspace(w, P)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv, variance="subspace_fp4", rank=R, basis=P)
    assert cobs().device_error() == 0
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    _check_subspace_fp4(w, K, V, Q, g, Pk, Pv, p, buf, P, R, units, units)


def test_subspace_fp4_with_identity_basis_selects_as_fp4_low_rank():
    """P = I: the FP4 coordinates are the FP4 eigenvectors, the same bytes and the same selection."""
    w = synth.WORKLOADS["decode32k"].replace(B=2, Hkv=2, Hq=8, T=4096)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    I = np.eye(w.d, dtype=np.float32)
    _, buf_s = run_decode(w, K, V, Q, g, Pk, Pv, variance="subspace_fp4", rank=4, basis=I)
    _, buf_l = run_decode(w, K, V, Q, g, Pk, Pv, variance="lowrank_fp4", rank=4)
    # same layout when s = d; compared as bits (the packed bf16 / FP4 words are not all finite floats)
    assert torch.equal(buf_s.summaries.view(torch.int32), buf_l.summaries.view(torch.int32))
    assert torch.equal(buf_s.idx, buf_l.idx)
    assert torch.equal(buf_s.O, buf_l.O)


@pytest.mark.parametrize("back", [1, 64])
def test_subspace_fp4_incremental_update_matches_full_build(back):
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=4096)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    P = synth.subspace_basis(w, 84)
    p = params_of(w, "subspace_fp4", 4, P)
    tK, tV, tPk, tPv = dev(K, w.dtype), dev(V, w.dtype), dev(Pk, "f32"), dev(Pv, "f32")
    full = C.alloc(p, prefill=False)
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, 0, full.summaries, full.Kc, full.Vc)
    inc = C.alloc(p, prefill=False)
    inc.summaries.copy_(full.summaries)
    nb = w.T // 64
    gf = 8 * (2 * p.d + 4 * 96 // 2 + 8 * 4)
    view = inc.summaries.view(p.B, p.Hkv, -1, gf)
    view[:, :, (nb - 1) // 32] = float("nan")
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, w.T - back, inc.summaries, inc.Kc, inc.Vc)
    torch.cuda.synchronize()
    # the poisoned lanes of the other blocks in the group stay poisoned: compare the last block only
    for a, b in zip(summaries_blocks(inc.summaries, p, check_padding=False), summaries_blocks(full.summaries, p)):
        assert np.array_equal(a[:, :, nb - 1], b[:, :, nb - 1])
