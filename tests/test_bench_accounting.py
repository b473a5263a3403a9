"""The benchmark's algorithmic byte and FLOP counts (the numerators of its roofline figures),
checked on CPU against brute-force counts and against the library's own summary sizes."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _rand_idx(rng, shape, nB, k):
    idx = np.full(shape + (k,), -1, np.int32)
    for pos in np.ndindex(*shape):
        n = rng.integers(0, min(k, nB) + 1)
        idx[pos][:n] = np.sort(rng.choice(nB, size=n, replace=False))
    return idx


def test_decode_bytes_counts_the_token_union_once():
    rng = np.random.default_rng(7)
    w = synth.WORKLOADS["decode32k"].replace(B=2, Hkv=2, Hq=8, T=3000, window=512)
    idx = _rand_idx(rng, (w.B, w.Hkv), w.nB, w.topk)
    by = bench.decode_bytes(w, idx)
    t = w.T - 1
    esz, d = 2, w.d
    kv = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            toks = set(range(max(0, t - w.window + 1), t + 1))
            for blk in idx[b, h]:
                if blk >= 0:
                    toks |= set(range(blk * w.block, blk * w.block + w.block))
            kv += len(toks)
    ncv = (t - w.cmp_block + 1) // w.cmp_stride + 1
    units = w.B * w.Hkv
    attn = kv * 2 * d * esz + units * ncv * 2 * d * esz + w.B * w.Hq * d * esz * 2 + w.B * w.Hq * 3 * 4 \
        + units * w.topk * 4
    assert by["attn"] == attn
    assert by["select"] == units * w.nB * 2 * d * 4 + w.B * w.Hq * d * esz + units * w.topk * 4


def test_prefill_flops_match_a_per_position_count():
    rng = np.random.default_rng(8)
    w = synth.WORKLOADS["prefill32k"].replace(B=1, Hq=8, Hkv=2, T=700, window=128)
    idx = np.full((w.B, w.T, w.Hkv, w.topk), -1, np.int32)
    for t in range(w.T):
        ncand = (t + 1) // w.block
        for g in range(w.Hkv):
            n = min(w.topk, ncand)
            if n:
                idx[0, t, g, :n] = np.sort(rng.choice(ncand, size=n, replace=False))
    total = 0
    for t in range(w.T):
        win = min(w.window, t + 1)
        vis = sum(1 for i in range(w.nC) if w.cmp_stride * i + w.cmp_block - 1 <= t)
        for g in range(w.Hkv):
            slc = int((idx[0, t, g] >= 0).sum()) * w.block
            total += 4 * w.d * w.G * (slc + win + vis)
    assert bench.prefill_flops(w, idx) == float(total)


@pytest.mark.parametrize("variance,rank,sub", [("channel", 0, 0), ("isotropic", 0, 0), ("lowrank", 4, 0),
                                               ("lowrank_fp4", 3, 0), ("subspace", 4, 84),
                                               ("subspace_fp4", 4, 84), ("subspace_fp4", 2, 64)])
def test_summary_bytes_per_block_match_the_library_layout(variance, rank, sub):
    from block_sparse_long_summary_b200 import build as B
    B.build()
    from block_sparse_long_summary_b200.cobs import Params, summaries_elems
    T = 64 * 32 * 3      # three full groups of 32 blocks
    p = Params(B=1, Hq=4, Hkv=1, d=128, T=T, topk=16, window=512, variance=variance, rank=max(rank, 1),
               sub=sub or 84)
    per_block_lib = summaries_elems(p) * 4 / (T // 64)
    assert bench.summary_block_bytes(128, variance, rank, sub) == per_block_lib
