"""GPU parity of the decode step entry points against the oracle and against the separate calls
they replace: cobs_decode_step (summary update, selection, then the attention as a programmatic
dependent of the selection) and cobs_decode_step_fused (selection and attention in one persistent
kernel).

Bars: selected indices bit-exact (the oracle's float32 canonical selection, and the separate
cobs_select); outputs within 2e-2 (bf16) of the oracle and of the separate calls. The fused
kernel's cross-CTA state (epoch, barrier counter, tagged segment lists) lives in the workspace,
so each entry point is also run several times in a row on one workspace, and replayed from a
CUDA graph.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import cobs_oracle as O
from gpu_common import TOL, cobs, dev, f64, inputs_decode, params_of, summaries_blocks

pytestmark = pytest.mark.gpu


class Problem:
    def __init__(self, w, variance="channel", seed=None):
        if seed is not None:
            w = w.replace(seed=seed)
        self.w = w
        C = cobs()
        self.K, self.V, self.Q, self.g, self.Pk, self.Pv = inputs_decode(w)
        self.p = params_of(w, variance)
        self.t = dict(K=dev(self.K, w.dtype), V=dev(self.V, w.dtype), Q=dev(self.Q, w.dtype),
                      Pk=dev(self.Pk, "f32"), Pv=dev(self.Pv, "f32"), g=torch.from_numpy(self.g).cuda())
        self.buf = C.alloc(self.p, prefill=False)

    def step(self, path="step", t_begin=0, buf=None):
        C = cobs()
        t = self.t
        C.decode_step(self.p, t["Q"], t["K"], t["V"], t["Pk"], t["Pv"], t["g"], buf or self.buf, t_begin=t_begin,
                      path=path)


def _oracle_check(pr, units, check_out=True, variance="channel"):
    w = pr.w
    G = w.G
    idx_g = pr.buf.idx.cpu().numpy()
    O_g = f64(pr.buf.O)
    Qf = synth.to_f64(pr.Q, w.dtype)
    for (b, h) in units:
        Kf, Vf, summ, Kc, Vc = O.unit_cache(w, pr.K[b, h], pr.V[b, h], pr.Pk, pr.Pv)
        if variance == "isotropic":
            summ = O.canonical_summaries_iso(Kf.astype(np.float32), w.block)
        qs = Qf[b, h * G:(h + 1) * G]
        sel, _ = O.select_decode(w, qs.astype(np.float32), summ)
        assert np.array_equal(idx_g[b, h], sel), f"idx unit {(b, h)}: {idx_g[b, h]} vs {sel}"
        if check_out:
            ref = O.position_output(qs, pr.g[b, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, sel, w.T - 1, w.block, w.window,
                                    w.cmp_block, w.cmp_stride)
            err = np.abs(O_g[b, h * G:(h + 1) * G] - ref).max()
            assert err <= TOL[w.dtype], f"unit {(b, h)} max-abs {err}"


def _against_calls(pr):
    """The separate calls on a second set of buffers: same idx, outputs within the bf16 tolerance."""
    C = cobs()
    ref = C.alloc(pr.p, prefill=False)
    pr.step(path="calls", buf=ref)
    torch.cuda.synchronize()
    assert torch.equal(pr.buf.idx, ref.idx)
    err = (pr.buf.O.float() - ref.O.float()).abs().max().item()
    assert err <= TOL[pr.w.dtype], err
    return err


SHAPES = [
    dict(B=2, Hkv=2, Hq=8),                        # the 32k decode workload, 4 units
    dict(B=1, Hkv=1, Hq=16, T=4096 + 37),          # ragged tail, G = 16
    dict(B=1, Hkv=2, Hq=2, T=2000, topk=32),       # G = 1, k > nB
    dict(B=1, Hkv=1, Hq=4, T=700, window=1024),    # W > T
    dict(B=1, Hkv=1, Hq=4, T=40, topk=4, window=64),   # no complete block
    dict(B=1, Hkv=1, Hq=4, T=20, topk=4, window=64),   # no compressed token either
    dict(B=2, Hkv=1, Hq=8, d=64, T=3000),          # d = 64
    dict(B=4, Hkv=4, Hq=16, T=32768),              # 16 units: phases with fewer elements than warps
    dict(B=64, Hkv=8, Hq=32, T=2048, topk=8),      # 512 units of one summary group each
]


PATHS = ["step", "fused"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("over", SHAPES)
def test_step_matches_oracle_and_calls(over, path):
    pr = Problem(synth.WORKLOADS["decode32k"].replace(**over))
    cobs().device_error(reset=True)
    pr.step(path)
    torch.cuda.synchronize()
    assert cobs().device_error() == 0
    w = pr.w
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    if len(units) > 16:
        _oracle_check(pr, units[:: max(1, len(units) // 16)])
    else:
        _oracle_check(pr, units)
    _against_calls(pr)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("over", [dict(B=2, Hkv=2, Hq=8, T=8192 + 64), dict(B=1, Hkv=2, Hq=4, d=64, T=3000, topk=32)])
def test_step_isotropic(over, path):
    pr = Problem(synth.WORKLOADS["decode32k"].replace(**over), variance="isotropic")
    cobs().device_error(reset=True)
    pr.step(path)
    torch.cuda.synchronize()
    assert cobs().device_error() == 0
    _oracle_check(pr, [(b, h) for b in range(pr.w.B) for h in range(pr.w.Hkv)], variance="isotropic")
    _against_calls(pr)


@pytest.mark.parametrize("path", PATHS)
def test_step_decode32k_full_size(path):
    pr = Problem(synth.WORKLOADS["decode32k"])
    cobs().device_error(reset=True)
    pr.step(path)
    torch.cuda.synchronize()
    assert cobs().device_error() == 0
    w = pr.w
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    sampled = [(0, 0), (3, 5), (7, 7), (5, 2)]
    _oracle_check(pr, [u for u in units if u not in sampled], check_out=False)
    _oracle_check(pr, sampled)
    _against_calls(pr)


@pytest.mark.parametrize("path", PATHS)
def test_step_decode128k_full_size(path):
    pr = Problem(synth.WORKLOADS["decode128k"])
    cobs().device_error(reset=True)
    pr.step(path)
    torch.cuda.synchronize()
    assert cobs().device_error() == 0
    _oracle_check(pr, [(0, h) for h in range(pr.w.Hkv)])
    _against_calls(pr)


@pytest.mark.parametrize("path", PATHS)
def test_step_repeated_on_one_workspace_and_in_a_graph(path):
    """Consecutive steps on one workspace (different queries each time), then the same step captured
    in a CUDA graph and replayed: each result equals the separate calls on the same inputs."""
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=2, Hkv=4, Hq=16, T=16384 + 64)
    pr = Problem(w)
    C.device_error(reset=True)
    for seed in (7, 8, 9):
        pr.t["Q"] = dev(synth.queries_decode(w.replace(seed=seed)), w.dtype)
        pr.step(path)
        torch.cuda.synchronize()
        assert C.device_error() == 0
        _against_calls(pr)
    # the update path (t_begin = T - 1) as a decoding loop issues it, captured once and replayed
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pr.step(path, t_begin=w.T - 1)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager_idx, eager_O = pr.buf.idx.clone(), pr.buf.O.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pr.step(path, t_begin=w.T - 1)
    for _ in range(3):
        pr.buf.O.zero_()
        pr.buf.idx.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        assert C.device_error() == 0
        assert torch.equal(pr.buf.idx, eager_idx)
        assert torch.equal(pr.buf.O, eager_O)
    del g


@pytest.mark.parametrize("path", PATHS)
def test_step_incremental_update_matches_full_build(path):
    """cobs_decode_step with t_begin = T - 1 on a cache built without the last row's block and token
    rewrites them exactly as the full build does."""
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=8192)
    pr = Problem(w)
    pr.step(path, t_begin=0)
    torch.cuda.synchronize()
    full_s, full_idx, full_O = pr.buf.summaries.clone(), pr.buf.idx.clone(), pr.buf.O.clone()
    nb = w.T // 64
    view = pr.buf.summaries.view(pr.p.B, pr.p.Hkv, -1, 2, pr.p.d // 4, 32, 4)
    view[:, :, (nb - 1) // 32, :, :, (nb - 1) % 32, :] = float("nan")
    pr.step(path, t_begin=w.T - 1)
    torch.cuda.synchronize()
    assert C.device_error() == 0
    assert np.array_equal(summaries_blocks(pr.buf.summaries, pr.p), summaries_blocks(full_s, pr.p))
    assert torch.equal(pr.buf.idx, full_idx)
    assert (pr.buf.O.float() - full_O.float()).abs().max().item() <= TOL["bf16"]


def test_fused_step_refuses_shapes_it_does_not_take():
    """float32 and the low-rank summaries: COBS_ERR_UNSUPPORTED on the host, no workspace size."""
    C = cobs()
    for name, variance in (("tiny", "channel"), ("decode32k", "lowrank")):
        w = synth.WORKLOADS[name].replace(B=1, Hkv=1, Hq=4, T=2048)
        p = params_of(w, variance)
        assert C.workspace_bytes(p, C.COBS_WS_STEP_FUSED) == 0
        buf = C.alloc(p, prefill=False)
        assert buf.ws_step_fused is None
        t = {k: torch.zeros(1, device="cuda") for k in ("Q", "K", "V", "Pk", "Pv", "g")}
        ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
        with pytest.raises(C.CobsError) as ei:
            C.cobs_decode_step_fused(p, t["Q"], t["K"], t["V"], t["Pk"], t["Pv"], p.T, buf.summaries, buf.Kc, buf.Vc,
                                     buf.idx, t["g"], buf.O, ws)
        assert ei.value.status == -2
