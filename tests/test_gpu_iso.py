"""GPU parity of the isotropic scalar-variance selector (one second-order scalar per block)
against the oracle: summaries (means and the block scalar) and selected blocks bit for bit,
outputs within the bf16 / float32 tolerance, for decode, the decode-step update, prefill and
a long context."""
import numpy as np
import pytest
import torch

import synth
from oracle import cobs_oracle as O
from gpu_common import TOL, cobs, dev, f64, inputs_decode, params_of, run_decode, run_prefill, summaries_blocks

pytestmark = pytest.mark.gpu


def _unit_ref(w, Kst):
    return O.canonical_summaries_iso(synth.to_f64(Kst, w.dtype).astype(np.float32), w.block)


@pytest.mark.parametrize("name,over", [
    ("tiny", dict()),                                              # float32, d = 64
    ("decode32k", dict(B=2, Hkv=2, Hq=8, T=8192)),                 # bf16, d = 128, fused build
    ("decode32k", dict(B=1, Hkv=1, Hq=16, T=4096 + 37)),           # G = 16, ragged tail
    ("decode32k", dict(B=1, Hkv=2, Hq=4, d=64, T=3000, topk=32)),  # d = 64, k > candidates
])
def test_iso_decode_matches_oracle(name, over):
    w = synth.WORKLOADS[name].replace(**over)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv, variance="isotropic")
    assert cobs().device_error() == 0
    summ_g = summaries_blocks(buf.summaries, p)
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    Qf = synth.to_f64(Q, w.dtype)
    G = w.G
    for b in range(w.B):
        for h in range(w.Hkv):
            ref = _unit_ref(w, K[b, h])
            assert np.array_equal(summ_g[b, h], ref), f"iso summaries differ at {(b, h)}"
            qs = Qf[b, h * G:(h + 1) * G]
            sel, _ = O.select_decode(w, qs.astype(np.float32), ref)
            assert np.array_equal(idx_g[b, h], sel), f"idx {(b, h)}: {idx_g[b, h]} vs {sel}"
            Kf, Vf, _, Kc, Vc = O.unit_cache(w, K[b, h], V[b, h], Pk, Pv)
            out = O.position_output(qs, g[b, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, sel, w.T - 1, w.block, w.window,
                                    w.cmp_block, w.cmp_stride)
            assert np.abs(O_g[b, h * G:(h + 1) * G] - out).max() <= TOL[w.dtype]


def test_iso_incremental_update_matches_full_build():
    """t_begin = T-1 rewrites the completed block's means and scalar exactly as a full build."""
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=8192)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p = params_of(w, "isotropic")
    tK, tV, tPk, tPv = dev(K, w.dtype), dev(V, w.dtype), dev(Pk, "f32"), dev(Pv, "f32")
    full = C.alloc(p, prefill=False)
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, 0, full.summaries, full.Kc, full.Vc)
    inc = C.alloc(p, prefill=False)
    inc.summaries.copy_(full.summaries)
    inc.Kc.copy_(full.Kc)
    inc.Vc.copy_(full.Vc)
    # poison the last block (its means and its scalar), then update
    nb = w.T // 64
    gf = (p.d + 1) * 32
    view = inc.summaries.view(p.B, p.Hkv, -1, gf)
    grp, lane = (nb - 1) // 32, (nb - 1) % 32
    mu = view[:, :, grp, :p.d * 32].view(p.B, p.Hkv, p.d // 4, 32, 4)
    mu[:, :, :, lane, :] = float("nan")
    view[:, :, grp, p.d * 32 + lane] = float("nan")
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, w.T - 1, inc.summaries, inc.Kc, inc.Vc)
    torch.cuda.synchronize()
    assert torch.equal(inc.summaries, full.summaries)


@pytest.mark.parametrize("name,over", [
    ("prefill32k", dict(B=1, Hq=16, Hkv=1, T=1024 + 37, topk=4, window=128)),
    ("tiny", dict(Hq=4, Hkv=2, T=600, mode="prefill")),
])
def test_iso_prefill_matches_oracle(name, over):
    w = synth.WORKLOADS[name].replace(**over)
    K, V = synth.kv_cache(w)
    Q, g = synth.queries_prefill(w), synth.gates_prefill(w)
    Pk, Pv = synth.projections(w)
    p, buf = run_prefill(w, K, V, Q, g, Pk, Pv, variance="isotropic")
    assert cobs().device_error() == 0
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    G = w.G
    for h in range(w.Hkv):
        ref_s = _unit_ref(w, K[0, h])
        ref = O.select_prefill_unit(w, Q[0, :, h * G:(h + 1) * G], ref_s)
        bad = np.nonzero(~np.all(idx_g[0, :, h] == ref, axis=1))[0]
        assert len(bad) == 0, f"group {h}: idx differs at positions {bad[:10]}"
        Kf, Vf, _, Kc, Vc = O.unit_cache(w, K[0, h], V[0, h], Pk, Pv)
        Qf = synth.to_f64(Q[0], w.dtype)
        for t in list(range(0, w.T, 97)) + [w.T - 1]:
            out = O.position_output(Qf[t, h * G:(h + 1) * G], g[0, t, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, ref[t], t,
                                    w.block, w.window, w.cmp_block, w.cmp_stride)
            assert np.abs(O_g[0, t, h * G:(h + 1) * G] - out).max() <= TOL[w.dtype], t


def test_iso_long_context_sampled_units():
    """131072 keys (64 summary groups per unit, the selection split across CTAs)."""
    C = cobs()
    w = synth.WORKLOADS["sweep"].replace(T=131072, B=2)
    p = params_of(w, "isotropic")
    K = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.bfloat16, device="cuda")
    sampled = [(0, 0), (1, w.Hkv - 1)]
    host = {u: synth.keys_unit(w, *u) for u in sampled}
    for b in range(w.B):
        for h in range(w.Hkv):
            if (b, h) in host:
                K[b, h].copy_(dev(host[(b, h)], "bf16"))
            else:
                synth.keys_unit_on_device(w, b, h, K[b, h])
    Pk, Pv = synth.projections(w)
    buf = C.alloc(p, prefill=False)
    C.device_error(reset=True)
    C.cobs_build_summaries(p, K, K, dev(Pk, "f32"), dev(Pv, "f32"), 0, buf.summaries, buf.Kc, buf.Vc)
    Q = synth.queries_decode(w)
    C.cobs_select(p, dev(Q, "bf16"), buf.summaries, 0, buf.idx, buf.ws_select)
    torch.cuda.synchronize()
    assert C.device_error() == 0
    summ_g = summaries_blocks(buf.summaries, p)
    idx = buf.idx.cpu().numpy()
    Qf = synth.to_f64(Q, "bf16")
    for (b, h) in sampled:
        ref = _unit_ref(w, host[(b, h)])
        assert np.array_equal(summ_g[b, h], ref)
        sel, _ = O.select_decode(w, Qf[b, h * w.G:(h + 1) * w.G].astype(np.float32), ref)
        assert np.array_equal(idx[b, h], sel)
