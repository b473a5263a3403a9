"""Helpers shared by the GPU parity tests: moving seeded inputs to the device, running the
library through its C ABI, and reshaping its outputs for comparison with the oracle."""
import numpy as np
import torch

import synth

TOL = {"bf16": 2e-2, "f32": 1e-4}


def cobs():
    from block_sparse_long_summary_b200 import build as B
    B.build()
    from block_sparse_long_summary_b200 import cobs as C
    return C


def dev(arr, dtype):
    """Storage-form numpy array (uint16 bf16 bits or float32) -> CUDA tensor."""
    if arr is None:
        return None
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def params_of(w, variance="channel", rank=4, basis=None):
    """basis: the query-subspace basis [d, s] (numpy float32) for variance "subspace(_fp4)"."""
    C = cobs()
    extra = {}
    if basis is not None:
        extra = dict(sub=basis.shape[1], basis=torch.from_numpy(np.ascontiguousarray(basis)).cuda())
    return C.Params(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T=w.T, topk=w.topk, window=w.window, block=w.block,
                    cmp_block=w.cmp_block, cmp_stride=w.cmp_stride, alpha=w.alpha, dtype=w.dtype, variance=variance,
                    rank=rank, **extra)


def summaries_blocks(flat, p, check_padding=True):
    """Device summaries (channel-interleaved groups of 32 blocks) -> [B, Hkv, nB, 2, d] float32
    (per-channel variance) or [B, Hkv, nB, d + 1] (isotropic: means, then the block's scalar)."""
    nB = p.T // p.block
    nG = max(1, -(-nB // 32))
    if p.variance in ("lowrank_fp4", "subspace_fp4"):
        # codes of cw entries per vector: the d channels, or the sub coordinates padded to 32
        R, d = p.rank, p.d
        n = p.sub if p.variance == "subspace_fp4" else d
        cw = -(-n // 32) * 32
        gb = 32 * (2 * d + R * cw // 2 + 8 * R)
        raw = flat[: p.B * p.Hkv * nG * gb // 4].cpu().numpy().view(np.uint8).reshape(p.B, p.Hkv, nG, gb)
        mub = raw[..., :64 * d].copy().view(np.uint16).reshape(p.B, p.Hkv, nG, d // 8, 32, 8)
        mu = (mub.astype(np.uint32) << 16).view(np.float32).transpose(0, 1, 2, 4, 3, 5).reshape(p.B, p.Hkv, nG * 32, d)
        cb = raw[..., 64 * d:64 * d + R * 16 * cw].reshape(p.B, p.Hkv, nG, R, cw // 32, 32, 16)
        codes = np.stack([cb & 15, cb >> 4], axis=-1).reshape(p.B, p.Hkv, nG, R, cw // 32, 32, 32)
        codes = codes.transpose(0, 1, 2, 5, 3, 4, 6).reshape(p.B, p.Hkv, nG * 32, R, cw)
        if check_padding:
            assert not codes[:, :, :nB, :, n:].any(), "codes past the stored entries must be zero"
        tail = raw[..., 64 * d + R * 16 * cw:].copy().view(np.float32).reshape(p.B, p.Hkv, nG, 2, R, 32)
        scales = tail[..., 0, :, :].transpose(0, 1, 2, 4, 3).reshape(p.B, p.Hkv, nG * 32, R)
        lam = tail[..., 1, :, :].transpose(0, 1, 2, 4, 3).reshape(p.B, p.Hkv, nG * 32, R)
        return mu[:, :, :nB], codes[:, :, :nB, :, :n].astype(np.uint8), scales[:, :, :nB], lam[:, :, :nB]
    if p.variance == "subspace":
        R, d, S = p.rank, p.d, p.sub
        gf = 32 * (d + R * S + R)
        a = flat[: p.B * p.Hkv * nG * gf].cpu().numpy().reshape(p.B, p.Hkv, nG, gf)
        mu = a[..., :d * 32].reshape(p.B, p.Hkv, nG, d // 4, 32, 4).transpose(0, 1, 2, 4, 3, 5)
        mu = mu.reshape(p.B, p.Hkv, nG * 32, d)[:, :, :nB]
        ut = a[..., d * 32:(d + R * S) * 32].reshape(p.B, p.Hkv, nG, R, S // 4, 32, 4).transpose(0, 1, 2, 5, 3, 4, 6)
        ut = ut.reshape(p.B, p.Hkv, nG * 32, R, S)[:, :, :nB]
        lam = a[..., (d + R * S) * 32:].reshape(p.B, p.Hkv, nG, R, 32).transpose(0, 1, 2, 4, 3)
        lam = lam.reshape(p.B, p.Hkv, nG * 32, R)[:, :, :nB]
        return mu, ut, lam
    if p.variance == "lowrank":
        R, d = p.rank, p.d
        gf = 32 * (d + R * d + R)
        a = flat[: p.B * p.Hkv * nG * gf].cpu().numpy().reshape(p.B, p.Hkv, nG, gf)

        def planes(x, n):   # [B, Hkv, nG, n, d/4, 32, 4] -> [B, Hkv, nG*32, n, d]
            x = x.reshape(p.B, p.Hkv, nG, n, d // 4, 32, 4).transpose(0, 1, 2, 5, 3, 4, 6)
            return x.reshape(p.B, p.Hkv, nG * 32, n, d)
        mu = planes(a[..., :d * 32], 1)[:, :, :nB, 0]
        u = planes(a[..., d * 32:(1 + R) * d * 32], R)[:, :, :nB]
        lam = a[..., (1 + R) * d * 32:].reshape(p.B, p.Hkv, nG, R, 32).transpose(0, 1, 2, 4, 3)
        lam = lam.reshape(p.B, p.Hkv, nG * 32, R)[:, :, :nB]
        return mu, u, lam
    if p.variance == "isotropic":
        gf = (p.d + 1) * 32
        a = flat[: p.B * p.Hkv * nG * gf].cpu().numpy().reshape(p.B, p.Hkv, nG, gf)
        mu = a[..., :p.d * 32].reshape(p.B, p.Hkv, nG, p.d // 4, 32, 4).transpose(0, 1, 2, 4, 3, 5)
        mu = mu.reshape(p.B, p.Hkv, nG * 32, p.d)
        sig = a[..., p.d * 32:].reshape(p.B, p.Hkv, nG * 32, 1)
        return np.concatenate([mu, sig], axis=-1)[:, :, :nB]
    a = flat[: p.B * p.Hkv * nG * 2 * p.d * 32].cpu().numpy()
    a = a.reshape(p.B, p.Hkv, nG, 2, p.d // 4, 32, 4).transpose(0, 1, 2, 5, 3, 4, 6)
    return a.reshape(p.B, p.Hkv, nG * 32, 2, p.d)[:, :, :nB]


def run_decode(w, K, V, Q, gates, Pk, Pv, variance="channel", rank=4, basis=None, path="step"):
    """The decode step through cobs_decode_step (path "step"), cobs_decode_step_fused ("fused") or
    the three separate calls ("calls")."""
    C = cobs()
    p = params_of(w, variance, rank, basis)
    buf = C.alloc(p, prefill=False)
    C.device_error(reset=True)
    C.decode_step(p, dev(Q, w.dtype), dev(K, w.dtype), dev(V, w.dtype), dev(Pk, "f32"), dev(Pv, "f32"),
                  torch.from_numpy(gates).cuda(), buf, t_begin=0, path=path)
    torch.cuda.synchronize()
    return p, buf


def run_prefill(w, K, V, Q, gates, Pk, Pv, variance="channel"):
    C = cobs()
    p = params_of(w, variance)
    buf = C.alloc(p, prefill=True)
    C.device_error(reset=True)
    C.prefill(p, dev(Q, w.dtype), dev(K, w.dtype), dev(V, w.dtype), dev(Pk, "f32"), dev(Pv, "f32"),
              torch.from_numpy(gates).cuda(), buf)
    torch.cuda.synchronize()
    return p, buf


def inputs_decode(w):
    K, V = synth.kv_cache(w)
    return K, V, synth.queries_decode(w), synth.gates_decode(w), *synth.projections(w)


def kc_close(gpu, ref, dtype):
    """Compressed tokens: the GPU rounds its float32 result once to the storage type; the oracle
    rounds the exact value. They differ by at most one unit in the last place of the storage type."""
    if dtype == "bf16":
        # one bf16 ulp is at most 2^-7 of the value; 1e-5 covers the float32 sum near zero
        tol = np.abs(ref) * 2.0 ** -7 + 1e-5
    else:
        tol = np.abs(ref) * 1e-5 + 1e-6
    return np.abs(gpu - ref) <= tol
