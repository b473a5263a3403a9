"""The C ABI library builds, loads, exports every declared entry point and validates
arguments on the host (no GPU needed: invalid arguments are rejected before any launch)."""
import ctypes
import os
import re

import pytest

from block_sparse_long_summary_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    path = B.build()
    from block_sparse_long_summary_b200 import cobs
    return cobs


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(cobs_[a-z0-9_]+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert {"cobs_build_summaries", "cobs_select", "cobs_sparse_attn_decode", "cobs_sparse_attn_prefill"} <= syms
    so = ctypes.CDLL(B.LIB)
    for name in sorted(syms):
        assert hasattr(so, name), name
    assert set(lib.EXPORTED) <= syms


def test_version_and_status_strings(lib):
    assert lib.version() == 102
    assert lib._lib.cobs_status_string(0) == b"ok"
    assert lib._lib.cobs_status_string(-1) == b"invalid argument"


def _p(**kw):
    from block_sparse_long_summary_b200.cobs import Params
    base = dict(B=1, Hq=4, Hkv=1, d=128, T=4096, topk=16, window=512)
    base.update(kw)
    return Params(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), -2),
    (dict(block=32), -2),
    (dict(topk=0), -1),
    (dict(topk=33), -2),
    (dict(window=32), -1),
    (dict(Hq=6, Hkv=4), -1),
    (dict(Hq=64, Hkv=2), -2),
    (dict(T=0), -1),
    (dict(cmp_stride=0), -1),
    (dict(alpha=float("nan")), -1),
    (dict(B=65535, Hkv=1, Hq=1, T=65536), -2),          # B * Hkv * T rows beyond int32 coordinates
])
def test_host_validation_rejects_before_launch(lib, kw, status):
    p = _p(**kw)
    cp = p.c()
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    r = lib._lib.cobs_build_summaries(ctypes.byref(cp), fake, fake, None, None, 0, fake, fake, fake, None)
    assert r == status, lib._lib.cobs_last_error()
    assert lib._lib.cobs_last_error() != b""
    assert lib.workspace_bytes(p, lib.COBS_WS_DECODE) == 0


def test_prefill_query_rows_bounded_by_int32(lib):
    """B * Hq * T query rows beyond int32 coordinates: prefill calls refuse on the host; the decode
    selection of the same shape (queries [B, Hq, d] only) is accepted by validation."""
    p = _p(B=1024, Hkv=1, Hq=16, T=1 << 18)
    cp = p.c()
    fake = ctypes.c_void_p(256)
    assert lib._lib.cobs_select(ctypes.byref(cp), fake, fake, 1, fake, fake, 1 << 40, None) == -2
    assert b"query rows" in lib._lib.cobs_last_error()
    assert lib._lib.cobs_sparse_attn_prefill(ctypes.byref(cp), fake, fake, fake, fake, fake, fake, fake, fake,
                                             fake, 1 << 40, None) == -2
    assert lib.summaries_elems(p) > 0


def test_null_and_misaligned_pointers_rejected(lib):
    p = _p()
    cp = p.c()
    fake = ctypes.c_void_p(256)
    assert lib._lib.cobs_select(ctypes.byref(cp), None, fake, 0, fake, fake, 1 << 20, None) == -1
    assert b"Q is NULL" in lib._lib.cobs_last_error()
    bad = ctypes.c_void_p(258)
    assert lib._lib.cobs_select(ctypes.byref(cp), bad, fake, 0, fake, fake, 1 << 20, None) == -1
    assert b"aligned" in lib._lib.cobs_last_error()
    assert lib._lib.cobs_select(ctypes.byref(cp), fake, fake, 2, fake, fake, 1 << 20, None) == -1


def test_workspace_sizes(lib):
    p = _p(B=8, Hq=32, Hkv=8, T=32768)
    n_units = 8 * 8
    # bf16 decode partials: units x 3 branches x record slots x G x (d + 4) floats
    ws = lib.workspace_bytes(p, lib.COBS_WS_DECODE)
    assert ws > 0 and ws % (n_units * 3 * 4 * 132 * 4) == 0
    assert ws <= (8 << 20)
    assert lib.summaries_elems(p) == n_units * 16 * 2 * 128 * 32
    assert lib.workspace_bytes(p, lib.COBS_WS_SELECT) > 0


@pytest.mark.parametrize("kw,status", [
    (dict(variance="lowrank", rank=0), -2),
    (dict(variance="lowrank", rank=9), -2),
    (dict(variance="lowrank_fp4", rank=9), -2),
    (dict(variance="subspace", rank=4, sub=82), -2),   # not a multiple of 4
    (dict(variance="subspace", rank=4, sub=0), -2),
    (dict(variance="subspace", rank=4, sub=132), -2),  # more than d
    (dict(variance="subspace_fp4", rank=4, sub=82), -2),
    (dict(variance="subspace_fp4", rank=9, sub=84), -2),
])
def test_summary_form_validation(lib, kw, status):
    p = _p(**kw)
    cp = p.c()
    fake = ctypes.c_void_p(256)
    r = lib._lib.cobs_build_summaries(ctypes.byref(cp), fake, fake, None, None, 0, fake, fake, fake, None)
    assert r == status, lib._lib.cobs_last_error()
    assert lib.summaries_elems(p) == 0


def test_unknown_variance_rejected(lib):
    cp = _p().c()
    cp.variance = 6   # one past COBS_VAR_SUBSPACE_FP4
    fake = ctypes.c_void_p(256)
    assert lib._lib.cobs_build_summaries(ctypes.byref(cp), fake, fake, None, None, 0, fake, fake, fake, None) == -1
    assert b"variance" in lib._lib.cobs_last_error()


@pytest.mark.parametrize("variance", ["subspace", "subspace_fp4"])
def test_subspace_needs_a_basis(lib, variance):
    p = _p(variance=variance, rank=4, sub=84)   # no basis: sizing works, compute calls refuse
    assert lib.summaries_elems(p) > 0
    cp = p.c()
    fake = ctypes.c_void_p(256)
    assert lib._lib.cobs_select(ctypes.byref(cp), fake, fake, 0, fake, fake, 1 << 30, None) == -1
    assert b"basis is NULL" in lib._lib.cobs_last_error()
    assert lib._lib.cobs_build_summaries(ctypes.byref(cp), fake, fake, None, None, 0, fake, fake, fake, None) == -1
    assert b"basis is NULL" in lib._lib.cobs_last_error()
    cp.basis = ctypes.c_void_p(264)   # misaligned
    assert lib._lib.cobs_select(ctypes.byref(cp), fake, fake, 0, fake, fake, 1 << 30, None) == -1
    assert b"aligned" in lib._lib.cobs_last_error()


def test_summary_sizes_of_every_form(lib):
    """Floats per unit: nG groups of 32 blocks, each group in the layout of its form."""
    B_, Hkv, d, T = 2, 8, 128, 32768 + 64 * 5      # nB = 517 -> nG = 17
    units, nG = B_ * Hkv, 17
    kw = dict(B=B_, Hq=32, Hkv=Hkv, d=d, T=T)
    assert lib.summaries_elems(_p(**kw)) == units * nG * 2 * d * 32
    assert lib.summaries_elems(_p(variance="isotropic", **kw)) == units * nG * (d + 1) * 32
    assert lib.summaries_elems(_p(variance="lowrank", rank=4, **kw)) == units * nG * 32 * (d + 4 * d + 4)
    assert lib.summaries_elems(_p(variance="lowrank_fp4", rank=3, **kw)) == units * nG * 8 * (2 * d + 3 * d // 2 + 24)
    assert lib.summaries_elems(_p(variance="subspace", rank=4, sub=84, **kw)) == units * nG * 32 * (d + 4 * 84 + 4)
    # FP4 coordinates: 84 codes padded to 96 per vector
    assert lib.summaries_elems(_p(variance="subspace_fp4", rank=4, sub=84, **kw)) == units * nG * 8 * (2 * d + 4 * 96 // 2
                                                                                                        + 32)
    # the query-subspace form's selection workspace adds the projected heads [units, G, s] float32
    ws_lr = lib.workspace_bytes(_p(variance="lowrank", rank=4, **kw), lib.COBS_WS_SELECT)
    ws_sub = lib.workspace_bytes(_p(variance="subspace", rank=4, sub=84, **kw), lib.COBS_WS_SELECT)
    assert ws_sub >= ws_lr + units * 4 * 84 * 4


def test_header_compiles_as_c99_and_links_from_c(lib, tmp_path):
    """The public header is plain C: a C99 program includes it with all warnings as errors,
    links against the library and runs the host-side part of the ABI."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "abi_from_c")
    lib_dir = os.path.dirname(B.LIB)
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_from_c.c"),
                           "-L", lib_dir, "-lcobs", f"-Wl,-rpath,{lib_dir}", "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
