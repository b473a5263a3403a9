"""GPU parity of the decode path (summaries, selection, decode attention) against the oracle.

Bars: summaries and selected block indices bit-exact (both sides use the same float32
arithmetic in the same order); compressed tokens within one storage ulp; outputs within
max-abs 1e-4 (float32) or 2e-2 (bf16).
"""
import numpy as np
import pytest

import synth
from oracle import cobs_oracle as O
from gpu_common import TOL, cobs, dev, f64, inputs_decode, kc_close, params_of, run_decode, summaries_blocks

pytestmark = pytest.mark.gpu


def _check_units(w, K, V, Q, gates, Pk, Pv, p, buf, units, check_out=True):
    G = w.G
    summ = summaries_blocks(buf.summaries, p)
    Kc_g, Vc_g = f64(buf.Kc), f64(buf.Vc)
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    Qf = synth.to_f64(Q, w.dtype)
    worst = 0.0
    for (b, h) in units:
        Kf, Vf, summ_o, Kc_o, Vc_o = O.unit_cache(w, K[b, h], V[b, h], Pk, Pv)
        assert np.array_equal(summ[b, h], summ_o), f"summaries differ at unit {(b, h)}"
        if w.nC:
            assert kc_close(Kc_g[b, h, :w.nC], Kc_o, w.dtype).all(), f"Kc unit {(b, h)}"
            assert kc_close(Vc_g[b, h, :w.nC], Vc_o, w.dtype).all(), f"Vc unit {(b, h)}"
        qs = Qf[b, h * G:(h + 1) * G]
        sel, _ = O.select_decode(w, qs.astype(np.float32), summ_o)
        assert np.array_equal(idx_g[b, h], sel), f"idx unit {(b, h)}: {idx_g[b, h]} vs {sel}"
        # the float32 decision against the float64 ranking of the same score
        mu, var = O.block_summaries(Kf, w.block)
        gap = O.near_tie_gap(O.group_scores(qs, mu, var, w.alpha), sel, O.n_candidates(w.T - 1, w.block), w.topk)
        assert gap is None or gap < 1e-5, f"unit {(b, h)}: float32 and float64 selections differ by {gap}"
        if check_out:
            ref = O.position_output(qs, gates[b, h * G:(h + 1) * G], Kf, Vf, Kc_o, Vc_o, sel, w.T - 1, w.block,
                                    w.window, w.cmp_block, w.cmp_stride)
            err = np.abs(O_g[b, h * G:(h + 1) * G] - ref).max()
            worst = max(worst, err)
            assert err <= TOL[w.dtype], f"unit {(b, h)} max-abs {err}"
    return worst


def test_tiny_fp32_decode():
    w = synth.WORKLOADS["tiny"]
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv)
    assert cobs().device_error() == 0
    _check_units(w, K, V, Q, g, Pk, Pv, p, buf, [(0, 0)])


@pytest.mark.parametrize("name,over", [
    ("decode32k", dict(B=2, Hkv=2, Hq=8)),
    ("decode32k", dict(B=1, Hkv=1, Hq=16, T=4096 + 37)),          # ragged tail, G = 16
    ("decode32k", dict(B=1, Hkv=2, Hq=2, T=2000, topk=32)),       # G = 1, k > nB
    ("decode32k", dict(B=1, Hkv=1, Hq=4, T=700, window=1024)),    # W > T
    ("decode32k", dict(B=1, Hkv=1, Hq=4, T=40, topk=4, window=64)),  # no complete block
    ("decode32k", dict(B=1, Hkv=1, Hq=4, T=20, topk=4, window=64)),  # no compressed token either
    ("decode32k", dict(B=2, Hkv=1, Hq=8, d=64, T=3000)),          # d = 64 bf16
    ("tiny", dict(T=1000 + 23, Hq=3, Hkv=1, d=128)),               # float32, ragged, d = 128
    ("tiny", dict(T=5000, Hq=8, Hkv=2, topk=7, window=300)),        # float32, odd k
])
@pytest.mark.parametrize("path", ["step", "calls"])
def test_decode_shapes(name, over, path):
    w = synth.WORKLOADS[name].replace(**over)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv, path=path)
    assert cobs().device_error() == 0
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    _check_units(w, K, V, Q, g, Pk, Pv, p, buf, units)


def test_decode32k_full_size():
    """The 32k decode workload: every unit's summaries and indices, outputs of sampled units."""
    w = synth.WORKLOADS["decode32k"]
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv)
    assert cobs().device_error() == 0
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    sampled = {(0, 0), (3, 5), (7, 7), (5, 2)}
    _check_units(w, K, V, Q, g, Pk, Pv, p, buf, [u for u in units if u not in sampled], check_out=False)
    _check_units(w, K, V, Q, g, Pk, Pv, p, buf, sorted(sampled))


def test_decode128k_full_size():
    w = synth.WORKLOADS["decode128k"]
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv)
    assert cobs().device_error() == 0
    _check_units(w, K, V, Q, g, Pk, Pv, p, buf, [(0, h) for h in range(w.Hkv)])


def test_incremental_update_matches_full_build():
    """t_begin = T-1 rewrites exactly the block and compressed token completed by the last row."""
    import torch
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=8192)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p = params_of(w)
    full = C.alloc(p, prefill=False)
    tK, tV, tPk, tPv = dev(K, w.dtype), dev(V, w.dtype), dev(Pk, "f32"), dev(Pv, "f32")
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, 0, full.summaries, full.Kc, full.Vc)
    inc = C.alloc(p, prefill=False)
    inc.summaries.copy_(full.summaries)
    inc.Kc.copy_(full.Kc)
    inc.Vc.copy_(full.Vc)
    nb = w.T // 64
    sb = summaries_blocks(inc.summaries, p).copy()
    # poison the last block's summary and the last compressed token, then update
    flat = inc.summaries.view(p.B, p.Hkv, -1)
    grp = (nb - 1) // 32
    lane = (nb - 1) % 32
    view = flat.view(p.B, p.Hkv, -1, 2, p.d // 4, 32, 4)
    view[:, :, grp, :, :, lane, :] = float("nan")
    inc.Kc[:, :, -1] = 7.0
    inc.Vc[:, :, -1] = 7.0
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, w.T - 1, inc.summaries, inc.Kc, inc.Vc)
    torch.cuda.synchronize()
    assert np.array_equal(summaries_blocks(inc.summaries, p), sb)
    # rows before the last compressed token are untouched; the rewritten one matches the full
    # build within one bf16 ulp (the two paths round their float32 projections separately)
    assert torch.equal(inc.Kc[:, :, :-1], full.Kc[:, :, :-1]) and torch.equal(inc.Vc[:, :, :-1], full.Vc[:, :, :-1])
    for a_, b_ in ((inc.Kc, full.Kc), (inc.Vc, full.Vc)):
        assert kc_close(f64(a_[:, :, -1]), f64(b_[:, :, -1]), "bf16").all()


def test_bad_index_sets_device_flag_without_fault():
    """An out-of-range selected block is skipped and reported through the device error flag."""
    import torch
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=1, Hq=4, T=4096)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv)
    assert C.device_error() == 0
    bad = buf.idx.clone()
    bad[0, 0, 0] = w.T // 64 + 5
    C.device_error(reset=True)
    C.cobs_sparse_attn_decode(p, dev(Q, w.dtype), dev(K, w.dtype), dev(V, w.dtype), buf.Kc, buf.Vc, bad,
                              torch.from_numpy(g).cuda(), buf.O, buf.ws_attn)
    torch.cuda.synchronize()
    assert C.device_error(reset=True) == 1
    assert torch.isfinite(buf.O.float()).all()
