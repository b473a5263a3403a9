"""Seeded synthetic workloads for block-sparse attention with cumulant-order block selection.

This module draws inputs only: it holds none of the method's arithmetic (no
summaries, scores, selection or attention). Tests, the benchmark and the oracle's
callers all take their inputs from here, so the CUDA path and the oracle see the
same bytes.

Workloads (the five configurations the build is measured on):

* ``tiny``     fp32, B=1, Hq=Hkv=1, d=64, T=1024, top-4, window 128, mean-pool compression.
* ``decode32k`` bf16, B=8, 32 query heads over 8 KV heads, d=128, T=32768, top-16,
  window 512, seeded random projection of the pooled K/V, 8 needle blocks.
* ``decode128k`` bf16, B=1, 64 query heads over 8 KV heads, T=131072, top-32,
  window 1024, 16 needle blocks.
* ``prefill32k`` bf16 causal prefill, B=1, 64 query heads over 4 KV heads, T=32768,
  top-16 per position, window 512.
* ``sweep``    selector-only, B=64, 8 KV heads (32 query heads), contexts 8192..1048576.

Distribution (per (batch, KV head) unit): key rows of block j are
N(mu_j, sigma_j^2 I) with mu_j ~ N(0, 0.5^2 I) and sigma_j = 0.25 * 8^u,
u ~ U[0, 1) (log-uniform in [0.25, 2]). Needle blocks, placed at distinct seeded
blocks that end before the final window, have mu_j ~ N(0, 0.1^2 I) and
sigma_j = 3. V, Q ~ N(0, 1). Gates are sigmoid(N(0, 1)) (1/3 each for ``tiny``).
Projections P_k, P_v have iid N(0, 1/d) entries. Values are formed in double,
rounded to float32 and, for bf16 workloads, to bfloat16 (round to nearest even).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

# stream tags
TAG_KMU, TAG_KSIG, TAG_KZ, TAG_V, TAG_Q, TAG_GATE, TAG_PK, TAG_PV, TAG_NEEDLE, TAG_NMU = range(1, 11)
TAG_KU = 11  # per-block direction bases of the anisotropic key model
TAG_QB, TAG_QZ = 12, 13  # query-subspace basis and the queries drawn in it


def build(force: bool = False) -> str:
    """Compile the generator library in place (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64 = ctypes.c_uint64, ctypes.c_int64
        vp = ctypes.c_void_p
        lib.synth_mix64.restype = u64
        lib.synth_mix64.argtypes = [u64]
        lib.synth_key.restype = u64
        lib.synth_key.argtypes = [u64, u64, u64, u64]
        for name in ("synth_normals_f32", "synth_normals_f64", "synth_uniforms_f64", "synth_words"):
            getattr(lib, name).restype = None
            getattr(lib, name).argtypes = [u64, u64, i64, vp]
        lib.synth_block_rows_f32.restype = None
        lib.synth_block_rows_f32.argtypes = [u64, vp, vp, i64, i64, i64, i64, vp]
        lib.synth_f32_to_bf16.restype = None
        lib.synth_f32_to_bf16.argtypes = [vp, i64, vp]
        lib.synth_bf16_to_f32.restype = None
        lib.synth_bf16_to_f32.argtypes = [vp, i64, vp]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def key(seed: int, a: int, b: int = 0, c: int = 0) -> int:
    return int(_load().synth_key(seed, a, b, c))


def normals_f32(k: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, np.float32)
    _load().synth_normals_f32(k, offset, n, _ptr(out))
    return out


def normals_f64(k: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, np.float64)
    _load().synth_normals_f64(k, offset, n, _ptr(out))
    return out


def uniforms_f64(k: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, np.float64)
    _load().synth_uniforms_f64(k, offset, n, _ptr(out))
    return out


def words(k: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, np.uint64)
    _load().synth_words(k, offset, n, _ptr(out))
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 values, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().synth_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    out = np.empty(x.shape, np.float32)
    _load().synth_bf16_to_f32(_ptr(x), x.size, _ptr(out))
    return out


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of a stored tensor (uint16 bf16 bits or float32)."""
    if dtype == "bf16":
        return bf16_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def to_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_to_f32(x)
    return np.ascontiguousarray(x, dtype=np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    topk: int
    window: int
    block: int = 64
    cmp_block: int = 32
    cmp_stride: int = 16
    alpha: float = 1.0
    dtype: str = "bf16"          # storage type of Q/K/V/Kc/Vc/O
    gates: str = "sigmoid"       # "sigmoid" or "third"
    proj: bool = True            # seeded random projection of pooled K/V (else identity)
    n_needles: int = 0
    seed: int = 0
    mode: str = "decode"         # "decode" or "prefill"

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nB(self) -> int:
        return self.T // self.block

    @property
    def nC(self) -> int:
        if self.T < self.cmp_block:
            return 0
        return (self.T - self.cmp_block) // self.cmp_stride + 1

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=1, Hkv=1, d=64, T=1024, topk=4, window=128, dtype="f32",
                     gates="third", proj=False, n_needles=0, seed=1001),
    "decode32k": Workload("decode32k", B=8, Hq=32, Hkv=8, d=128, T=32768, topk=16, window=512,
                          n_needles=8, seed=1002),
    "decode128k": Workload("decode128k", B=1, Hq=64, Hkv=8, d=128, T=131072, topk=32, window=1024,
                           n_needles=16, seed=1003),
    "prefill32k": Workload("prefill32k", B=1, Hq=64, Hkv=4, d=128, T=32768, topk=16, window=512,
                           n_needles=8, seed=1004, mode="prefill"),
    "sweep": Workload("sweep", B=64, Hq=32, Hkv=8, d=128, T=8192, topk=16, window=512,
                      n_needles=8, seed=1005),
}
SWEEP_CONTEXTS = [8192 << i for i in range(8)]  # 8192 .. 1048576


def needle_blocks(w: Workload, b: int, h: int) -> np.ndarray:
    """Distinct seeded needle blocks that end before the final window (partial Fisher-Yates)."""
    n_elig = max(0, (w.T - w.window) // w.block)
    n = min(w.n_needles, n_elig)
    if n == 0:
        return np.zeros(0, np.int64)
    perm = np.arange(n_elig, dtype=np.int64)
    wd = words(key(w.seed, TAG_NEEDLE, b, h), n)
    for i in range(n):
        j = i + int(wd[i] % np.uint64(n_elig - i))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:n])


def block_params(w: Workload, b: int, h: int):
    """Per-block mean (nb, d) and spread (nb,) of unit (b, h) as float32; needles applied."""
    nb = max(1, -(-w.T // w.block))
    mu = (0.5 * normals_f64(key(w.seed, TAG_KMU, b, h), nb * w.d)).astype(np.float32).reshape(nb, w.d)
    u = uniforms_f64(key(w.seed, TAG_KSIG, b, h), nb)
    sigma = (0.25 * np.power(8.0, u)).astype(np.float32)
    for j in needle_blocks(w, b, h):
        mu[j] = (0.1 * normals_f64(key(w.seed, TAG_NMU, b, h), w.d, offset=int(j) * w.d)).astype(np.float32)
        sigma[j] = np.float32(3.0)
    return np.ascontiguousarray(mu), np.ascontiguousarray(sigma)


def _store(x32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16(x32) if dtype == "bf16" else np.ascontiguousarray(x32, np.float32)


def keys_unit(w: Workload, b: int, h: int, T: Optional[int] = None) -> np.ndarray:
    """K rows [T, d] of unit (b, h) in storage form."""
    T = w.T if T is None else T
    mu, sigma = block_params(w, b, h)
    out = np.empty((T, w.d), np.float32)
    _load().synth_block_rows_f32(key(w.seed, TAG_KZ, b, h), _ptr(mu), _ptr(sigma), mu.shape[0],
                                 T, w.d, w.block, _ptr(out))
    return _store(out, w.dtype)


def values_unit(w: Workload, b: int, h: int, T: Optional[int] = None) -> np.ndarray:
    T = w.T if T is None else T
    return _store(normals_f32(key(w.seed, TAG_V, b, h), T * w.d).reshape(T, w.d), w.dtype)


def kv_cache(w: Workload):
    """K, V [B, Hkv, T, d] in storage form."""
    sdt = np.uint16 if w.dtype == "bf16" else np.float32
    K = np.empty((w.B, w.Hkv, w.T, w.d), sdt)
    V = np.empty((w.B, w.Hkv, w.T, w.d), sdt)
    for b in range(w.B):
        for h in range(w.Hkv):
            K[b, h] = keys_unit(w, b, h)
            V[b, h] = values_unit(w, b, h)
    return K, V


def queries_decode(w: Workload) -> np.ndarray:
    """Q [B, Hq, d]: the query at position T-1 (the same draws as prefill row T-1)."""
    q = np.empty((w.B, w.Hq, w.d), np.float32)
    for b in range(w.B):
        for hq in range(w.Hq):
            q[b, hq] = normals_f32(key(w.seed, TAG_Q, b, hq), w.d, offset=(w.T - 1) * w.d)
    return _store(q, w.dtype)


def queries_prefill(w: Workload, positions: Optional[np.ndarray] = None) -> np.ndarray:
    """Q [B, T, Hq, d] (or [B, len(positions), Hq, d] for a subset of positions)."""
    if positions is None:
        q = np.empty((w.B, w.Hq, w.T, w.d), np.float32)
        for b in range(w.B):
            for hq in range(w.Hq):
                q[b, hq] = normals_f32(key(w.seed, TAG_Q, b, hq), w.T * w.d).reshape(w.T, w.d)
        q = np.ascontiguousarray(q.transpose(0, 2, 1, 3))
    else:
        positions = np.asarray(positions, np.int64)
        q = np.empty((w.B, len(positions), w.Hq, w.d), np.float32)
        for b in range(w.B):
            for hq in range(w.Hq):
                k = key(w.seed, TAG_Q, b, hq)
                for i, t in enumerate(positions):
                    q[b, i, hq] = normals_f32(k, w.d, offset=int(t) * w.d)
    return _store(q, w.dtype)


def subspace_basis(w: Workload, s: int) -> np.ndarray:
    """P [d, s] float32 with orthonormal columns: the QR factor of a seeded Gaussian d x s matrix
    (column signs fixed by a positive diagonal of R). It stands for the leading eigenvectors of the
    queries' second moment, the subspace the query-subspace summaries are kept in."""
    a = normals_f64(key(w.seed, TAG_QB), w.d * s).reshape(w.d, s)
    q, r = np.linalg.qr(a)
    q = q * np.where(np.diag(r) < 0, -1.0, 1.0)
    return np.ascontiguousarray(q.astype(np.float32))


def queries_decode_subspace(w: Workload, P: np.ndarray, leak: float = 0.1) -> np.ndarray:
    """Q [B, Hq, d] concentrated in span(P): q = sqrt(1 - leak^2) sqrt(d/s) P z + leak n with
    z ~ N(0, I_s) and n ~ N(0, I_d), so E|q|^2 = d as for the plain N(0, I) queries and a share
    leak^2 of it lies (mostly) outside the subspace."""
    d, s = P.shape
    q = np.empty((w.B, w.Hq, d), np.float32)
    a = np.sqrt(1.0 - leak * leak) * np.sqrt(d / s)
    for b in range(w.B):
        for hq in range(w.Hq):
            z = normals_f64(key(w.seed, TAG_QZ, b, hq), s + d)
            q[b, hq] = (a * (P.astype(np.float64) @ z[:s]) + leak * z[s:]).astype(np.float32)
    return _store(q, w.dtype)


def _sigmoid32(z: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-z))).astype(np.float32)


def gates_decode(w: Workload) -> np.ndarray:
    """Gates [B, Hq, 3] in order (compressed, selected, window), post-sigmoid, float32."""
    if w.gates == "third":
        return np.full((w.B, w.Hq, 3), np.float32(1.0 / 3.0), np.float32)
    g = np.empty((w.B, w.Hq, 3), np.float32)
    for b in range(w.B):
        for hq in range(w.Hq):
            g[b, hq] = _sigmoid32(normals_f64(key(w.seed, TAG_GATE, b, hq), 3, offset=(w.T - 1) * 3))
    return g


def gates_prefill(w: Workload, positions: Optional[np.ndarray] = None) -> np.ndarray:
    """Gates [B, T, Hq, 3] (or for a subset of positions)."""
    pos = np.arange(w.T) if positions is None else np.asarray(positions, np.int64)
    if w.gates == "third":
        return np.full((w.B, len(pos), w.Hq, 3), np.float32(1.0 / 3.0), np.float32)
    g = np.empty((w.B, len(pos), w.Hq, 3), np.float32)
    for b in range(w.B):
        for hq in range(w.Hq):
            k = key(w.seed, TAG_GATE, b, hq)
            if positions is None:
                g[b, :, hq] = _sigmoid32(normals_f64(k, 3 * w.T).reshape(w.T, 3))
            else:
                for i, t in enumerate(pos):
                    g[b, i, hq] = _sigmoid32(normals_f64(k, 3, offset=int(t) * 3))
    return g


def projections(w: Workload):
    """P_k, P_v [d, d] float32 with N(0, 1/d) entries, or (None, None) for plain mean-pooling."""
    if not w.proj:
        return None, None
    s = 1.0 / np.sqrt(w.d)
    pk = (s * normals_f64(key(w.seed, TAG_PK), w.d * w.d)).astype(np.float32).reshape(w.d, w.d)
    pv = (s * normals_f64(key(w.seed, TAG_PV), w.d * w.d)).astype(np.float32).reshape(w.d, w.d)
    return pk, pv


# ------------------------------------------------------------------ device-side generation (large workloads)

_CU_SRC = os.path.join(_HERE, "synth_cuda.cu")
_CU_LIB_PATH = os.path.join(_HERE, "libsynth_cuda.so")
_cu_lib = None


def build_cuda(force: bool = False) -> str:
    """Compile the device-side generator (nvcc, sm_100a) in place."""
    if force or not os.path.exists(_CU_LIB_PATH) or os.path.getmtime(_CU_LIB_PATH) < os.path.getmtime(_CU_SRC):
        tmp = _CU_LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
                               "-shared", "-cudart", "static", "-o", tmp, _CU_SRC])
        os.replace(tmp, _CU_LIB_PATH)
    return _CU_LIB_PATH


def _cu():
    global _cu_lib
    if _cu_lib is None:
        build_cuda()
        lib = ctypes.CDLL(_CU_LIB_PATH)
        vp, u64, i64 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64
        lib.synth_gpu_block_rows_bf16.argtypes = [u64, vp, vp, i64, i64, i64, i64, vp, vp]
        lib.synth_gpu_block_rows_bf16.restype = ctypes.c_int
        lib.synth_gpu_aniso_rows_bf16.argtypes = [u64, u64, vp, vp, i64, i64, i64, i64, ctypes.c_int, vp, vp]
        lib.synth_gpu_aniso_rows_bf16.restype = ctypes.c_int
        _cu_lib = lib
    return _cu_lib


def keys_unit_on_device(w: Workload, b: int, h: int, out, T: Optional[int] = None, stream=None,
                        aniso_rank: int = 0) -> None:
    """Fill a CUDA bf16 tensor out [T, d] with the keys of unit (b, h), drawn on the device.

    Same streams and distribution as keys_unit; the device's double-precision log/cos may put a
    value on a neighbouring bf16. Use keys_unit where both sides must see identical bytes.
    aniso_rank > 0 draws the anisotropic model instead: each block's spread sigma_j concentrated
    on aniso_rank seeded directions with variances decaying by halves, plus 10% isotropic noise
    (device only; for measurements that compare selectors, not for bit-exact parity).
    """
    import torch
    T = w.T if T is None else T
    assert w.dtype == "bf16" and out.dtype == torch.bfloat16 and out.is_contiguous() and out.numel() == T * w.d
    mu, sigma = block_params(w, b, h)
    dmu = torch.from_numpy(mu).to(out.device)
    dsig = torch.from_numpy(sigma).to(out.device)
    s = torch.cuda.current_stream(out.device) if stream is None else stream
    if aniso_rank > 0:
        rc = _cu().synth_gpu_aniso_rows_bf16(key(w.seed, TAG_KZ, b, h), key(w.seed, TAG_KU, b, h), dmu.data_ptr(),
                                             dsig.data_ptr(), mu.shape[0], T, w.d, w.block, int(aniso_rank),
                                             out.data_ptr(), s.cuda_stream)
    else:
        rc = _cu().synth_gpu_block_rows_bf16(key(w.seed, TAG_KZ, b, h), dmu.data_ptr(), dsig.data_ptr(),
                                             mu.shape[0], T, w.d, w.block, out.data_ptr(), s.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"device generator launch failed ({rc})")
    s.synchronize()  # dmu / dsig go out of scope
