"""The compressed covariance forms at the full decode workloads (32k: 64 units of 512 blocks; 128k:
8 units of 2048 blocks): low-rank eigenpairs, FP4 eigenvectors with bf16 means, query-subspace
coordinates, and query-subspace coordinates in FP4 with bf16 means. For every unit the stored summaries and the selected blocks equal the oracle's bit for
bit (both sides run the same fixed float32 solver and canonical sums); the outputs of two units per
workload are within the bf16 bar of the oracle's float64 attention."""
import numpy as np
import pytest

import synth
from oracle import cobs_oracle as O
from gpu_common import TOL, cobs, f64, inputs_decode, run_decode, summaries_blocks

pytestmark = pytest.mark.gpu


def _reference(variance, K32, L, R, P):
    if variance == "lowrank":
        return O.canonical_summaries_lowrank(K32, L, R)
    if variance == "lowrank_fp4":
        return O.canonical_summaries_lowrank_fp4(K32, L, R)
    if variance == "subspace_fp4":
        return O.canonical_summaries_subspace_fp4(K32, L, R, P)
    return O.canonical_summaries_subspace(K32, L, R, P)


def _stored(variance, ref):
    """The oracle fields the device layout stores, in summaries_blocks order."""
    if variance in ("lowrank_fp4", "subspace_fp4"):
        return tuple(ref[:4])   # bf16 means, codes, scales, eigenvalues
    return tuple(ref[:3])


@pytest.mark.parametrize("variance", ["lowrank", "lowrank_fp4", "subspace", "subspace_fp4"])
@pytest.mark.parametrize("name", ["decode32k", "decode128k"])
def test_compressed_forms_full_size(name, variance):
    w = synth.WORKLOADS[name]
    R, s = 4, 84
    K, V, Q, g, Pk, Pv = inputs_decode(w)
    P = synth.subspace_basis(w, s) if variance.startswith("subspace") else None
    if P is not None:
        Q = synth.queries_decode_subspace(w, P)
    p, buf = run_decode(w, K, V, Q, g, Pk, Pv, variance=variance, rank=R, basis=P)
    assert cobs().device_error() == 0
    got = summaries_blocks(buf.summaries, p)
    idx_g = buf.idx.cpu().numpy()
    O_g = f64(buf.O)
    Qf = synth.to_f64(Q, w.dtype)
    G = w.G
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    for (b, h) in units:
        ref = _reference(variance, synth.to_f64(K[b, h], w.dtype).astype(np.float32), w.block, R, P)
        for i, (x, y) in enumerate(zip((a[b, h] for a in got), _stored(variance, ref))):
            assert np.array_equal(x, y), f"summary field {i} differs at unit {(b, h)}"
        qs = Qf[b, h * G:(h + 1) * G]
        sel, _ = O.select_decode(w, qs.astype(np.float32), ref)
        assert np.array_equal(idx_g[b, h], sel), f"idx {(b, h)}: {idx_g[b, h]} vs {sel}"
        if (b, h) in (units[0], units[-1]):
            Kf, Vf, _, Kc, Vc = O.unit_cache(w, K[b, h], V[b, h], Pk, Pv)
            out = O.position_output(qs, g[b, h * G:(h + 1) * G], Kf, Vf, Kc, Vc, sel, w.T - 1, w.block, w.window,
                                    w.cmp_block, w.cmp_stride)
            assert np.abs(O_g[b, h * G:(h + 1) * G] - out).max() <= TOL[w.dtype]
