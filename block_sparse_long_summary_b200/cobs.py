"""Thin Python binding of the COBS C ABI (``include/cobs.h``).

Argument marshalling only: tensors are passed as device pointers and every step runs in
the CUDA library. PyTorch provides device memory and the current stream. The library
must be built (``python -m block_sparse_long_summary_b200.build``); importing this module
without it raises an error: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libcobs.so")

COBS_OK = 0
COBS_ERR_INVALID_ARG = -1
COBS_ERR_UNSUPPORTED = -2
COBS_ERR_CUDA = -3
COBS_ERR_WORKSPACE = -4
COBS_F32 = 0
COBS_BF16 = 1
COBS_VAR_CHANNEL, COBS_VAR_ISOTROPIC, COBS_VAR_LOWRANK, COBS_VAR_LOWRANK_FP4, COBS_VAR_SUBSPACE = 0, 1, 2, 3, 4
COBS_VAR_SUBSPACE_FP4 = 5
COBS_WS_SELECT = 0
COBS_WS_DECODE = 1
COBS_WS_PREFILL = 2
COBS_WS_STEP = 3
COBS_WS_STEP_FUSED = 4
COBS_WS_BASIS = 5

EXPORTED = [
    "cobs_build_summaries", "cobs_select", "cobs_sparse_attn_decode", "cobs_sparse_attn_prefill",
    "cobs_sparse_attn_decode_noalloc", "cobs_workspace_bytes", "cobs_summaries_elems", "cobs_status_string", "cobs_last_error",
    "cobs_device_error", "cobs_launch_count", "cobs_version", "cobs_block_log_mass", "cobs_decode_step",
    "cobs_decode_step_fused", "cobs_query_basis",
]


class cobs_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("T", ctypes.c_int32), ("block", ctypes.c_int32), ("cmp_block", ctypes.c_int32),
                ("cmp_stride", ctypes.c_int32), ("topk", ctypes.c_int32), ("window", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("dtype", ctypes.c_int32), ("variance", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("sub", ctypes.c_int32), ("basis", ctypes.c_void_p)]


class CobsError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"COBS CUDA library not built: {path} is missing "
                          "(run python -m block_sparse_long_summary_b200.build)")
    lib = ctypes.CDLL(path)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    P = ctypes.POINTER(cobs_params)
    lib.cobs_build_summaries.argtypes = [P, vp, vp, vp, vp, i32, vp, vp, vp, vp]
    lib.cobs_select.argtypes = [P, vp, vp, i32, vp, vp, sz, vp]
    lib.cobs_sparse_attn_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cobs_sparse_attn_prefill.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cobs_sparse_attn_decode_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.cobs_block_log_mass.argtypes = [P, vp, vp, vp, vp]
    lib.cobs_decode_step.argtypes = [P, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cobs_decode_step_fused.argtypes = [P, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.cobs_query_basis.argtypes = [P, vp, ctypes.c_int64, vp, vp, vp, sz, vp]
    lib.cobs_query_basis.restype = ctypes.c_int
    for f in ("cobs_build_summaries", "cobs_select", "cobs_sparse_attn_decode", "cobs_sparse_attn_prefill",
              "cobs_sparse_attn_decode_noalloc", "cobs_block_log_mass", "cobs_decode_step", "cobs_decode_step_fused"):
        getattr(lib, f).restype = ctypes.c_int
    lib.cobs_workspace_bytes.argtypes = [P, i32]
    lib.cobs_workspace_bytes.restype = sz
    lib.cobs_summaries_elems.argtypes = [P]
    lib.cobs_summaries_elems.restype = sz
    lib.cobs_status_string.argtypes = [ctypes.c_int]
    lib.cobs_status_string.restype = ctypes.c_char_p
    lib.cobs_last_error.argtypes = []
    lib.cobs_last_error.restype = ctypes.c_char_p
    lib.cobs_device_error.argtypes = [i32]
    lib.cobs_device_error.restype = i32
    lib.cobs_version.argtypes = []
    lib.cobs_version.restype = i32
    lib.cobs_launch_count.argtypes = [i32]
    lib.cobs_launch_count.restype = ctypes.c_int64
    return lib


_lib = load_library()


@dataclasses.dataclass
class Params:
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
    dtype: str = "bf16"
    variance: str = "channel"   # "channel", "isotropic", "lowrank", "lowrank_fp4", "subspace", "subspace_fp4"
    rank: int = 4               # eigenpairs per block for the low-rank forms
    sub: int = 84               # "subspace(_fp4)": coordinates kept per eigenvector
    basis: object = dataclasses.field(default=None, compare=False, repr=False)  # "subspace(_fp4)": [d, sub] f32

    def c(self) -> cobs_params:
        var = {"channel": COBS_VAR_CHANNEL, "isotropic": COBS_VAR_ISOTROPIC, "lowrank": COBS_VAR_LOWRANK,
               "lowrank_fp4": COBS_VAR_LOWRANK_FP4, "subspace": COBS_VAR_SUBSPACE,
               "subspace_fp4": COBS_VAR_SUBSPACE_FP4}[self.variance]
        sub = var in (COBS_VAR_SUBSPACE, COBS_VAR_SUBSPACE_FP4)
        if sub and self.basis is not None and (self.basis.dtype != torch.float32 or
                                                tuple(self.basis.shape) != (self.d, self.sub)):
            raise ValueError("basis must be a float32 [d, sub] tensor")
        return cobs_params(self.B, self.Hq, self.Hkv, self.d, self.T, self.block, self.cmp_block, self.cmp_stride,
                           self.topk, self.window, float(self.alpha), COBS_BF16 if self.dtype == "bf16" else COBS_F32,
                           var, int(self.rank), int(self.sub) if sub else 0,
                           _ptr(self.basis) if sub and self.basis is not None else None)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def nC(self) -> int:
        return (self.T - self.cmp_block) // self.cmp_stride + 1 if self.T >= self.cmp_block else 0

    @property
    def nB(self) -> int:
        return self.T // self.block


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status: int):
    if status != COBS_OK:
        raise CobsError(status, _lib.cobs_last_error().decode() or _lib.cobs_status_string(status).decode())


def workspace_bytes(p: Params, which: int) -> int:
    return int(_lib.cobs_workspace_bytes(ctypes.byref(p.c()), which))


def summaries_elems(p: Params) -> int:
    return int(_lib.cobs_summaries_elems(ctypes.byref(p.c())))


def device_error(reset: bool = False) -> int:
    return int(_lib.cobs_device_error(1 if reset else 0))


def version() -> int:
    return int(_lib.cobs_version())


def launch_count(reset: bool = False) -> int:
    """Kernel launches issued by the library in this process."""
    return int(_lib.cobs_launch_count(1 if reset else 0))


# -------------------------------------------------------------- the four calls (same names as the C ABI)

def cobs_build_summaries(p: Params, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, stream=None):
    cp = p.c()
    _check(_lib.cobs_build_summaries(ctypes.byref(cp), _ptr(K), _ptr(V), _ptr(Pk), _ptr(Pv), int(t_begin),
                                     _ptr(summaries), _ptr(Kc), _ptr(Vc), _stream(stream)))


def cobs_select(p: Params, Q, summaries, prefill, idx, workspace, stream=None):
    cp = p.c()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.cobs_select(ctypes.byref(cp), _ptr(Q), _ptr(summaries), int(prefill), _ptr(idx), _ptr(workspace),
                            nbytes, _stream(stream)))


def cobs_sparse_attn_decode(p: Params, Q, K, V, Kc, Vc, idx, gates, O, workspace, stream=None):
    cp = p.c()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.cobs_sparse_attn_decode(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(Vc), _ptr(idx),
                                        _ptr(gates), _ptr(O), _ptr(workspace), nbytes, _stream(stream)))


def cobs_decode_step(p: Params, Q, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, idx, gates, O, workspace,
                     stream=None):
    """Summary update from t_begin, selection and decode attention enqueued as one step."""
    cp = p.c()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.cobs_decode_step(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(Pk), _ptr(Pv), int(t_begin),
                                 _ptr(summaries), _ptr(Kc), _ptr(Vc), _ptr(idx), _ptr(gates), _ptr(O),
                                 _ptr(workspace), nbytes, _stream(stream)))


def cobs_decode_step_fused(p: Params, Q, K, V, Pk, Pv, t_begin, summaries, Kc, Vc, idx, gates, O, workspace,
                           stream=None):
    """The same step with the selection and the attention in one persistent kernel."""
    cp = p.c()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.cobs_decode_step_fused(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(Pk), _ptr(Pv),
                                       int(t_begin), _ptr(summaries), _ptr(Kc), _ptr(Vc), _ptr(idx), _ptr(gates),
                                       _ptr(O), _ptr(workspace), nbytes, _stream(stream)))


def cobs_query_basis(p: Params, Q, n, basis, eigenvalues, workspace, stream=None):
    """Query-subspace basis [d, p.sub] (and eigenvalues, or None) from n query rows of Q."""
    cp = p.c()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.cobs_query_basis(ctypes.byref(cp), _ptr(Q), int(n), _ptr(basis), _ptr(eigenvalues), _ptr(workspace),
                                 nbytes, _stream(stream)))


def query_basis(p: Params, Q, stream=None):
    """Allocate and compute the basis [d, p.sub] float32 and eigenvalues [p.sub] from the rows of Q
    (any shape [..., d] in p's storage type)."""
    rows = Q.reshape(-1, p.d)
    basis = torch.empty((p.d, p.sub), dtype=torch.float32, device=Q.device)
    evals = torch.empty(p.sub, dtype=torch.float32, device=Q.device)
    ws = torch.empty(max(16, workspace_bytes(p, COBS_WS_BASIS)), dtype=torch.uint8, device=Q.device)
    cobs_query_basis(p, rows, rows.shape[0], basis, evals, ws, stream)
    return basis, evals


def cobs_sparse_attn_decode_noalloc(p: Params, Q, K, V, Kc, Vc, idx, gates, O, stream=None):
    """Decode attention using the library's built-in device scratch instead of a workspace,
    for callers that cannot provide device memory of their own (see include/cobs.h)."""
    cp = p.c()
    _check(_lib.cobs_sparse_attn_decode_noalloc(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(Vc),
                                                _ptr(idx), _ptr(gates), _ptr(O), _stream(stream)))


def cobs_sparse_attn_prefill(p: Params, Q, K, V, Kc, Vc, idx, gates, O, workspace, stream=None):
    cp = p.c()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.cobs_sparse_attn_prefill(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(Vc),
                                         _ptr(idx), _ptr(gates), _ptr(O), _ptr(workspace), nbytes, _stream(stream)))


def cobs_block_log_mass(p: Params, Q, K, out, stream=None):
    """Evaluation only: ln of the exact attention mass of every complete block, out [B, Hq, T // 64]."""
    cp = p.c()
    _check(_lib.cobs_block_log_mass(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(out), _stream(stream)))


# -------------------------------------------------------------- buffers (allocated by torch, not the library)

@dataclasses.dataclass
class Buffers:
    summaries: torch.Tensor
    Kc: torch.Tensor
    Vc: torch.Tensor
    idx: torch.Tensor
    O: torch.Tensor
    ws_select: torch.Tensor
    ws_attn: torch.Tensor
    ws_step: torch.Tensor | None = None
    ws_step_fused: torch.Tensor | None = None  # None: a shape cobs_decode_step_fused does not take


def alloc(p: Params, prefill: bool, device="cuda") -> Buffers:
    """Output and workspace tensors for one problem (workspaces zero-filled)."""
    dt = p.torch_dtype
    nq = p.T if prefill else 1
    summ = torch.empty(max(1, summaries_elems(p)), dtype=torch.float32, device=device)
    Kc = torch.empty((p.B, p.Hkv, max(1, p.nC), p.d), dtype=dt, device=device)
    Vc = torch.empty_like(Kc)
    idx = torch.empty((p.B, nq, p.Hkv, p.topk) if prefill else (p.B, p.Hkv, p.topk), dtype=torch.int32,
                      device=device)
    O = torch.empty((p.B, nq, p.Hq, p.d) if prefill else (p.B, p.Hq, p.d), dtype=dt, device=device)
    ws_sel = torch.zeros(max(16, workspace_bytes(p, COBS_WS_SELECT)), dtype=torch.uint8, device=device)
    ws_attn = torch.zeros(max(16, workspace_bytes(p, COBS_WS_PREFILL if prefill else COBS_WS_DECODE)),
                          dtype=torch.uint8, device=device)
    ws_step = None if prefill else torch.zeros(max(16, workspace_bytes(p, COBS_WS_STEP)), dtype=torch.uint8,
                                               device=device)
    nf = 0 if prefill else workspace_bytes(p, COBS_WS_STEP_FUSED)
    ws_fused = torch.zeros(nf, dtype=torch.uint8, device=device) if nf else None
    return Buffers(summ, Kc, Vc, idx, O, ws_sel, ws_attn, ws_step, ws_fused)


def decode_step(p: Params, Q, K, V, Pk, Pv, gates, buf: Buffers, t_begin: int, stream=None, path: str = "step"):
    """Summaries update from t_begin, selection and attention for the query at T - 1: one
    cobs_decode_step call (path "step"), one cobs_decode_step_fused call ("fused"), or the three
    separate calls ("calls")."""
    if path == "step":
        cobs_decode_step(p, Q, K, V, Pk, Pv, t_begin, buf.summaries, buf.Kc, buf.Vc, buf.idx, gates, buf.O,
                         buf.ws_step, stream)
        return
    if path == "fused":
        cobs_decode_step_fused(p, Q, K, V, Pk, Pv, t_begin, buf.summaries, buf.Kc, buf.Vc, buf.idx, gates, buf.O,
                               buf.ws_step_fused, stream)
        return
    if path != "calls":
        raise ValueError(f"unknown decode step path {path!r}")
    cobs_build_summaries(p, K, V, Pk, Pv, t_begin, buf.summaries, buf.Kc, buf.Vc, stream)
    cobs_select(p, Q, buf.summaries, 0, buf.idx, buf.ws_select, stream)
    cobs_sparse_attn_decode(p, Q, K, V, buf.Kc, buf.Vc, buf.idx, gates, buf.O, buf.ws_attn, stream)


def prefill(p: Params, Q, K, V, Pk, Pv, gates, buf: Buffers, stream=None):
    """Summaries of the whole context, per-position selection and causal attention."""
    cobs_build_summaries(p, K, V, Pk, Pv, 0, buf.summaries, buf.Kc, buf.Vc, stream)
    cobs_select(p, Q, buf.summaries, 1, buf.idx, buf.ws_select, stream)
    cobs_sparse_attn_prefill(p, Q, K, V, buf.Kc, buf.Vc, buf.idx, gates, buf.O, buf.ws_attn, stream)
