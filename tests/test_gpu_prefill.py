"""GPU parity of the causal prefill path (per-position selection and attention) against the oracle.

Selected indices are compared bit for bit at every position; outputs at every position for
small cases and at sampled positions (the first 128, every 97th, the last 64) for the 32k
prefill workload.
"""
import numpy as np
import pytest

import synth
from oracle import cobs_oracle as O
from gpu_common import TOL, cobs, f64, run_decode, run_prefill

pytestmark = pytest.mark.gpu


def _inputs(w, positions=None):
    K, V = synth.kv_cache(w)
    return K, V, synth.queries_prefill(w), synth.gates_prefill(w), *synth.projections(w)


def _check(w, K, V, Q, gates, Pk, Pv, buf, positions, b=0, check_idx_all=True):
    G = w.G
    idx_g = buf.idx.cpu().numpy()      # [B, T, Hkv, k]
    O_g = f64(buf.O)                   # [B, T, Hq, d]
    if check_idx_all:
        for h in range(w.Hkv):
            Kf = synth.to_f64(K[b, h], w.dtype)
            summ = O.canonical_summaries(Kf.astype(np.float32), w.block)
            ref = O.select_prefill_unit(w, Q[b, :, h * G:(h + 1) * G], summ)
            bad = np.nonzero(~np.all(idx_g[b, :, h] == ref, axis=1))[0]
            assert len(bad) == 0, f"group {h}: idx differs at positions {bad[:10]}"
    pos = np.asarray(positions)
    Oref, idx_ref = O.prefill_positions(w, K, V, Q[b, pos], gates[b, pos], Pk, Pv, pos, b=b)
    assert np.array_equal(idx_g[b, pos], idx_ref)
    # the float32 decisions against the float64 ranking of the same score at the checked positions
    Qf = synth.to_f64(Q[b], w.dtype)
    for h in range(w.Hkv):
        mu, var = O.block_summaries(synth.to_f64(K[b, h], w.dtype), w.block)
        for i, t in enumerate(pos):
            S64 = O.group_scores(Qf[t, h * G:(h + 1) * G], mu, var, w.alpha)
            gap = O.near_tie_gap(S64, idx_ref[i, h], O.n_candidates(int(t), w.block), w.topk)
            assert gap is None or gap < 1e-5, f"position {t} group {h}: float32/float64 gap {gap}"
    err = np.abs(O_g[b, pos] - Oref).max()
    assert err <= TOL[w.dtype], f"max-abs {err}"
    return err


@pytest.mark.parametrize("over", [
    dict(B=1, Hq=16, Hkv=1, T=1024 + 37, topk=4, window=128),
    dict(B=2, Hq=8, Hkv=2, T=700, topk=16, window=64),
    dict(B=1, Hq=4, Hkv=1, T=300, topk=2, window=512, d=64),
])
def test_prefill_small_bf16(over):
    w = synth.WORKLOADS["prefill32k"].replace(**over)
    K, V, Q, g, Pk, Pv = _inputs(w)
    p, buf = run_prefill(w, K, V, Q, g, Pk, Pv)
    assert cobs().device_error() == 0
    for b in range(w.B):
        _check(w, K, V, Q, g, Pk, Pv, buf, np.arange(w.T), b=b)


def test_prefill_fp32_and_last_row_equals_decode():
    w = synth.WORKLOADS["tiny"].replace(Hq=4, Hkv=2, T=600, mode="prefill")
    K, V, Q, g, Pk, Pv = _inputs(w)
    p, buf = run_prefill(w, K, V, Q, g, Pk, Pv)
    assert cobs().device_error() == 0
    _check(w, K, V, Q, g, Pk, Pv, buf, np.arange(w.T))
    # the decode path at the same context gives the last prefill row
    wd = w.replace(mode="decode")
    pd, bd = run_decode(wd, K, V, synth.queries_decode(wd), synth.gates_decode(wd), Pk, Pv)
    assert np.array_equal(bd.idx.cpu().numpy(), buf.idx.cpu().numpy()[:, -1])
    assert np.abs(f64(bd.O) - f64(buf.O)[:, -1]).max() <= 1e-5


def test_prefill32k_full_size():
    w = synth.WORKLOADS["prefill32k"]
    K, V, Q, g, Pk, Pv = _inputs(w)
    p, buf = run_prefill(w, K, V, Q, g, Pk, Pv)
    assert cobs().device_error() == 0
    pos = np.unique(np.concatenate([np.arange(128), np.arange(0, w.T, 97), np.arange(w.T - 64, w.T)]))
    _check(w, K, V, Q, g, Pk, Pv, buf, pos)
