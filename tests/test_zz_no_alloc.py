"""The allocation-free decode call (cobs_sparse_attn_decode_noalloc).

Some callers cannot give the library device memory of their own (their allocations all go
through a pool they have already divided up, or their host forbids device allocations once
running); this call keeps its scratch in a fixed array inside the library instead. Its
output must match the ordinary workspace-taking call on the same inputs, on consecutive
calls (the array keeps the previous call's contents, which must not leak into the next),
and problems too large for the array must be refused before anything is launched.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from gpu_common import TOL, cobs, dev, params_of

pytestmark = pytest.mark.gpu


# the bf16 stream kernel at d = 128 and d = 64, and the float32 chunk kernel (a different record
# layout in the scratch array)
CASES = [("decode32k", dict(B=2, Hkv=2, Hq=8, T=8192 + 64)),
         ("decode32k", dict(B=2, Hkv=1, Hq=8, d=64, T=3000)),
         ("tiny", dict(T=2048 + 17, Hq=4, Hkv=2))]


def _problem(name, over, seed):
    w = synth.WORKLOADS[name].replace(seed=seed, **over)
    K, V = synth.kv_cache(w)
    Q, g = synth.queries_decode(w), synth.gates_decode(w)
    Pk, Pv = synth.projections(w)
    C = cobs()
    p = params_of(w)
    buf = C.alloc(p, prefill=False)
    t = dict(K=dev(K, w.dtype), V=dev(V, w.dtype), Q=dev(Q, w.dtype), g=torch.from_numpy(g).cuda())
    C.cobs_build_summaries(p, t["K"], t["V"], dev(Pk, "f32"), dev(Pv, "f32"), 0, buf.summaries, buf.Kc, buf.Vc)
    C.cobs_select(p, t["Q"], buf.summaries, 0, buf.idx, buf.ws_select)
    return p, buf, t


@pytest.mark.parametrize("name,over", CASES)
def test_noalloc_decode_matches_workspace_call_on_consecutive_calls(name, over):
    C = cobs()
    lib = C._lib
    for seed in (4242, 4343):   # two calls in a row, on different inputs
        p, buf, t = _problem(name, over, seed)
        ref = torch.empty_like(buf.O)
        C.cobs_sparse_attn_decode(p, t["Q"], t["K"], t["V"], buf.Kc, buf.Vc, buf.idx, t["g"], ref, buf.ws_attn)
        out = torch.full_like(buf.O, float("nan"))
        cp = p.c()
        st = lib.cobs_sparse_attn_decode_noalloc(
            ctypes.byref(cp), t["Q"].data_ptr(), t["K"].data_ptr(), t["V"].data_ptr(), buf.Kc.data_ptr(),
            buf.Vc.data_ptr(), buf.idx.data_ptr(), t["g"].data_ptr(), out.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert st == 0, lib.cobs_last_error()
        torch.cuda.synchronize()
        assert C.device_error() == 0
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= TOL[p.dtype], err
        # the same kernels on the same inputs: the results agree bit for bit
        assert torch.equal(out, ref)


def test_noalloc_refuses_problems_beyond_its_scratch():
    C = cobs()
    lib = C._lib
    big = C.Params(B=64, Hq=256, Hkv=16, d=128, T=131072, topk=32, window=1024)
    assert C.workspace_bytes(big, C.COBS_WS_DECODE) > (8 << 20)
    cp = big.c()
    fake = ctypes.c_void_p(256)   # refused on the host before any pointer is used
    st = lib.cobs_sparse_attn_decode_noalloc(ctypes.byref(cp), fake, fake, fake, fake, fake, fake, fake, fake, None)
    assert st == C.COBS_ERR_WORKSPACE
    assert b"scratch" in lib.cobs_last_error()
