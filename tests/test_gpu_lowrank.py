"""GPU parity of the low-rank covariance selector (the leading eigenpairs of each block's key
covariance) against the oracle: means, eigenvectors, eigenvalues and selected blocks bit for bit
(both sides run the same fixed float32 subspace iteration), outputs within tolerance."""
import numpy as np
import pytest
import torch

import synth
from oracle import cobs_oracle as O
from gpu_common import TOL, cobs, dev, f64, inputs_decode, params_of, run_decode, summaries_blocks

pytestmark = pytest.mark.gpu


def _unit_ref(w, Kst, R):
    return O.canonical_summaries_lowrank(synth.to_f64(Kst, w.dtype).astype(np.float32), w.block, R)


@pytest.mark.parametrize("name,over,R", [
    ("tiny", dict(), 4),                                              # float32, d = 64
    ("decode32k", dict(B=2, Hkv=2, Hq=8, T=4096), 4),                  # bf16, d = 128, G = 4
    ("decode32k", dict(B=1, Hkv=1, Hq=16, T=2048 + 37), 2),            # G = 16, ragged tail
    ("decode32k", dict(B=1, Hkv=2, Hq=2, d=64, T=3000, topk=32), 8),  # d = 64, G = 1, rank 8, k > candidates
])
def test_lowrank_decode_matches_oracle(name, over, R):
    w = synth.WORKLOADS[name].replace(**over)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv, variance="lowrank", rank=R)
    assert cobs().device_error() == 0
    mu_g, u_g, lam_g = summaries_blocks(buf.summaries, p)
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    Qf = synth.to_f64(Q, w.dtype)
    G = w.G
    for b in range(w.B):
        for h in range(w.Hkv):
            ref = _unit_ref(w, K[b, h], R)
            assert np.array_equal(mu_g[b, h], ref[0]), f"means differ at {(b, h)}"
            assert np.array_equal(u_g[b, h], ref[1]), f"eigenvectors differ at {(b, h)}"
            assert np.array_equal(lam_g[b, h], ref[2]), f"eigenvalues differ at {(b, h)}"
            qs = Qf[b, h * G:(h + 1) * G]
            sel, _ = O.select_decode(w, qs.astype(np.float32), ref)
            assert np.array_equal(idx_g[b, h], sel), f"idx {(b, h)}: {idx_g[b, h]} vs {sel}"
            Kf, Vf, _, Kc, Vc = O.unit_cache(w, K[b, h], V[b, h], Pk, Pv)
            out = O.position_output(qs, g[b, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, sel, w.T - 1, w.block, w.window,
                                    w.cmp_block, w.cmp_stride)
            assert np.abs(O_g[b, h * G:(h + 1) * G] - out).max() <= TOL[w.dtype]


@pytest.mark.parametrize("back", [1, 64])   # t_begin = T - 1 (the decode-step path) and T - 64
def test_lowrank_incremental_update_matches_full_build(back):
    C = cobs()
    w = synth.WORKLOADS["decode32k"].replace(B=1, Hkv=2, Hq=8, T=4096)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p = params_of(w, "lowrank", 4)
    tK, tV, tPk, tPv = dev(K, w.dtype), dev(V, w.dtype), dev(Pk, "f32"), dev(Pv, "f32")
    full = C.alloc(p, prefill=False)
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, 0, full.summaries, full.Kc, full.Vc)
    inc = C.alloc(p, prefill=False)
    inc.summaries.copy_(full.summaries)
    inc.Kc.copy_(full.Kc)
    inc.Vc.copy_(full.Vc)
    nb = w.T // 64
    gf = 32 * (p.d + 4 * p.d + 4)
    view = inc.summaries.view(p.B, p.Hkv, -1, gf)
    grp = (nb - 1) // 32
    view[:, :, grp] = float("nan")  # the whole group of the last block
    C.cobs_build_summaries(p, tK, tV, tPk, tPv, w.T - back, inc.summaries, inc.Kc, inc.Vc)
    torch.cuda.synchronize()
    # the update rewrites exactly the last block; the poisoned lanes of earlier blocks in the
    # group stay poisoned, so compare the last block only, bit for bit (and the compressed
    # tokens the update rewrote within one bf16 ulp of the full build)
    mu_f, u_f, lam_f = summaries_blocks(full.summaries, p)
    mu_i, u_i, lam_i = summaries_blocks(inc.summaries, p)
    assert np.array_equal(mu_i[:, :, nb - 1], mu_f[:, :, nb - 1])
    assert np.array_equal(u_i[:, :, nb - 1], u_f[:, :, nb - 1])
    assert np.array_equal(lam_i[:, :, nb - 1], lam_f[:, :, nb - 1])
    from gpu_common import kc_close
    assert kc_close(f64(inc.Kc[:, :, -1]), f64(full.Kc[:, :, -1]), "bf16").all()


@pytest.mark.parametrize("name,over,R", [
    ("tiny", dict(), 4),                                              # float32, d = 64
    ("decode32k", dict(B=2, Hkv=2, Hq=8, T=4096), 4),                  # bf16, d = 128, G = 4
    ("decode32k", dict(B=1, Hkv=1, Hq=16, T=2048 + 37), 3),            # G = 16, odd rank, ragged tail
    ("decode32k", dict(B=1, Hkv=2, Hq=2, d=64, T=3000, topk=32), 8),  # d = 64, G = 1, rank 8
])
def test_lowrank_fp4_decode_matches_oracle(name, over, R):
    """FP4 eigenvectors and bf16 means: codes, scales, eigenvalues, means and selected blocks bit
    for bit against the oracle's quantisation of its canonical eigenpairs."""
    w = synth.WORKLOADS[name].replace(**over)
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv, variance="lowrank_fp4", rank=R)
    assert cobs().device_error() == 0
    mu_g, codes_g, sc_g, lam_g = summaries_blocks(buf.summaries, p)
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    Qf = synth.to_f64(Q, w.dtype)
    G = w.G
    for b in range(w.B):
        for h in range(w.Hkv):
            ref = O.canonical_summaries_lowrank_fp4(synth.to_f64(K[b, h], w.dtype).astype(np.float32), w.block, R)
            mu_q, codes, scales, lam, _ = ref
            assert np.array_equal(mu_g[b, h], mu_q), f"bf16 means differ at {(b, h)}"
            assert np.array_equal(codes_g[b, h], codes), f"E2M1 codes differ at {(b, h)}"
            assert np.array_equal(sc_g[b, h], scales), f"scales differ at {(b, h)}"
            assert np.array_equal(lam_g[b, h], lam), f"eigenvalues differ at {(b, h)}"
            qs = Qf[b, h * G:(h + 1) * G]
            sel, _ = O.select_decode(w, qs.astype(np.float32), ref)
            assert np.array_equal(idx_g[b, h], sel), f"idx {(b, h)}: {idx_g[b, h]} vs {sel}"
            Kf, Vf, _, Kc, Vc = O.unit_cache(w, K[b, h], V[b, h], Pk, Pv)
            out = O.position_output(qs, g[b, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, sel, w.T - 1, w.block, w.window,
                                    w.cmp_block, w.cmp_stride)
            assert np.abs(O_g[b, h * G:(h + 1) * G] - out).max() <= TOL[w.dtype]


def test_lowrank_prefill_selection_is_rejected():
    C = cobs()
    w = synth.WORKLOADS["prefill32k"].replace(B=1, Hq=16, Hkv=1, T=512)
    p = params_of(w, "lowrank", 4)
    buf = C.alloc(p, prefill=True)
    Q = torch.zeros((w.B, w.T, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(C.CobsError) as ei:
        C.cobs_select(p, Q, buf.summaries, 1, buf.idx, buf.ws_select)
    assert ei.value.status == -2
