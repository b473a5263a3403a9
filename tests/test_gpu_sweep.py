"""GPU parity of the selector at the sweep's context lengths (8k, 128k, 1M keys).

The key cache of the non-sampled units is drawn on the device (same streams, device libm); the
sampled units are drawn on the host, uploaded, and compared bit for bit (summaries and selected
blocks) with the oracle.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import cobs_oracle as O
from gpu_common import cobs, dev, params_of, summaries_blocks

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [8192, 131072, 1048576])
def test_selector_sweep_sampled_units(T):
    C = cobs()
    w = synth.WORKLOADS["sweep"].replace(T=T, B=2)
    p = params_of(w)
    K = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.bfloat16, device="cuda")
    sampled = [(0, 0), (1, w.Hkv - 1)]
    host_keys = {u: synth.keys_unit(w, *u) for u in sampled}
    for b in range(w.B):
        for h in range(w.Hkv):
            if (b, h) in sampled:
                K[b, h].copy_(dev(host_keys[(b, h)], "bf16"))
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
    idx = buf.idx.cpu().numpy()
    summ_g = summaries_blocks(buf.summaries, p)
    Qf = synth.to_f64(Q, "bf16")
    for (b, h) in sampled:
        summ = O.canonical_summaries(synth.to_f32(host_keys[(b, h)], "bf16"), w.block)
        assert np.array_equal(summ_g[b, h], summ), f"summaries differ at {(b, h)}"
        sel, _ = O.select_decode(w, Qf[b, h * w.G:(h + 1) * w.G].astype(np.float32), summ)
        assert np.array_equal(idx[b, h], sel), f"idx differ at {(b, h)}: {idx[b, h]} vs {sel}"
    # every unit's list is a valid selection: distinct, ascending, in range
    for b in range(w.B):
        for h in range(w.Hkv):
            v = idx[b, h]
            assert np.all(np.diff(v) > 0) and v.min() >= 0 and v.max() < w.nB


@pytest.mark.parametrize("name,over", [
    ("tiny", dict()),                                   # float32, d = 64, G = 3
    ("decode32k", dict(B=2, Hkv=2, Hq=8, T=4096 + 50)),  # bf16, d = 128, G = 4, ragged tail
    ("decode32k", dict(B=1, Hkv=1, Hq=16, T=2048)),      # G = 16
    ("decode32k", dict(B=1, Hkv=1, Hq=4, T=40)),         # no complete block: nothing written
])
def test_block_log_mass_matches_oracle(name, over):
    """ln of the exact block mass (evaluation call) against the oracle's float64 value."""
    C = cobs()
    w = synth.WORKLOADS[name].replace(**over)
    p = params_of(w)
    K, _ = synth.kv_cache(w)
    Q = synth.queries_decode(w)
    nB = w.T // w.block
    out = torch.full((w.B, w.Hq, max(1, nB)), 7.0, dtype=torch.float32, device="cuda")
    C.cobs_block_log_mass(p, dev(Q, w.dtype), dev(K, w.dtype), out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    if nB == 0:
        assert np.all(got == 7.0)
        return
    Qf = synth.to_f64(Q, w.dtype)
    for b in range(w.B):
        for h in range(w.Hkv):
            Kf = synth.to_f64(K[b, h], w.dtype)
            for j in range(w.G):
                ref = O.exact_log_mass(Qf[b, h * w.G + j], Kf, w.block)
                # float32 logits (|s| < 40) and exp / log: a few float32 ulps of the logits
                assert np.abs(got[b, h * w.G + j] - ref).max() <= 1e-4 + 4e-6 * np.abs(ref).max()
