#!/usr/bin/env python3
"""Benchmark of the COBS decode hot path on B200.

One step = one decode step of the 32k decode workload (B=8, 32 query heads over 8 KV
heads, d=128, T=32768, top-16, window 512): the summary update for the token appended at
T-1 (cobs_build_summaries from T-1), the block selection (cobs_select) and the three-branch
attention (cobs_sparse_attn_decode). Inputs are seeded synthetic tensors resident in HBM
when the timed region starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs the whole workload on its own GPU (independent decode
batches, no collective on the data path: weak scaling); the step time is the max over ranks.
`--impl reference` times the CPU oracle (the reference arm) on host cores instead.
"""
from __future__ import annotations

import argparse
import contextlib
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode query-heads/s + achieved HBM GB/s at 32k ctx; prefill TFLOP/s"
CSRC = os.path.join(ROOT, "block_sparse_long_summary_b200", "csrc")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode32k", choices=["decode32k", "decode128k", "prefill32k", "sweep"])
    ap.add_argument("--contexts", default=None, help="sweep: comma-separated context lengths (default 8k .. 1M)")
    ap.add_argument("--variance", choices=["channel", "isotropic", "lowrank", "lowrank_fp4", "subspace",
                                           "subspace_fp4"],
                    default="channel",
                    help="second-order statistic of the summaries (per-channel variance, one scalar per block, "
                         "or the leading eigenpairs of each block's covariance)")
    ap.add_argument("--rank", type=int, default=4, help="eigenpairs per block with the low-rank variances")
    ap.add_argument("--sub", type=int, default=84,
                    help="query-subspace dimension with --variance subspace (seeded orthonormal basis; the "
                         "queries are drawn concentrated in its span)")
    ap.add_argument("--subspace-queries", action="store_true",
                    help="draw the queries concentrated in the seeded --sub basis with any --variance (to "
                         "compare the summary forms on the queries the query-subspace form is built for)")
    ap.add_argument("--aniso", type=int, default=0,
                    help="sweep: draw anisotropic key blocks (spread on this many directions) instead of isotropic")
    ap.add_argument("--prefill-steps", type=int, default=5, help="timed prefill steps in the default run")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill sub-measurement")
    ap.add_argument("--no-subrecords", action="store_true",
                    help="skip the decode128k and selector-sweep sub-measurements of the default run")
    ap.add_argument("--T", type=int, default=None, help="override the context length (small profiling cases)")
    ap.add_argument("--copies", type=int, default=6, help="KV-cache copies rotated between steps (L2 defeat)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override the batch size (small profiling cases)")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank time over all ranks (identity without a process group). Every rank
    must call it at the same point; works with nccl (device tensor) and gloo (host tensor)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# the sources a kernel's DRAM traffic depends on (its own file and the headers it includes)
KERNEL_SOURCES = {
    "decode_step": ["decode_step.cu", "select_core.cuh", "stream_tile.cuh", "common.cuh", "dims.h", "tma.cu",
                    "tma.h"],
    "decode_attention": ["decode_stream.cu", "stream_tile.cuh", "common.cuh", "dims.h", "tma.cu", "tma.h"],
    "select_decode": ["select.cu", "select_core.cuh", "common.cuh", "dims.h"],
    "prefill_tc": ["prefill.cu", "tc.cuh", "common.cuh", "dims.h", "tma.cu", "tma.h"],
}


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for fn in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(CSRC, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken on the
    current sources and on `workload` (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(kernel)
    if not ent or ent.get("source_hash") != source_hash(kernel) or ent.get("workload") != workload:
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        self.out.seek(0)
        rows = [ln.strip().split(", ") for ln in self.out.read().splitlines() if ln.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ algorithmic bytes

def summary_block_bytes(d, variance, rank, sub):
    """Summary bytes per selection block for each second-order form."""
    return {"isotropic": (d + 1) * 4, "lowrank": (d + rank * d + rank) * 4,
            "lowrank_fp4": 2 * d + rank * d // 2 + 8 * rank,
            "subspace": (d + rank * sub + rank) * 4,
            "subspace_fp4": 2 * d + rank * (-(-sub // 32) * 32) // 2 + 8 * rank}.get(variance, 2 * d * 4)


def decode_bytes(w, idx, variance="channel", rank=4, sub=84):
    """Algorithmic HBM bytes of one decode step, from the selected blocks (idx [B, Hkv, k])."""
    import numpy as np
    d, esz = w.d, 2 if w.dtype == "bf16" else 4
    t = w.T - 1
    w0 = max(0, t - w.window + 1)
    win = set(range(w0, t + 1))
    ncv = min(w.nC, (t - w.cmp_block + 1) // w.cmp_stride + 1) if t >= w.cmp_block - 1 else 0
    kv_tokens = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            toks = set(win)
            for blk in idx[b, h]:
                if blk >= 0:
                    toks.update(range(blk * w.block, (blk + 1) * w.block))
            kv_tokens += len(toks)
    units = w.B * w.Hkv
    attn = kv_tokens * 2 * d * esz + units * ncv * 2 * d * esz          # K/V union + compressed K/V
    attn += w.B * w.Hq * d * esz * 2 + w.B * w.Hq * 3 * 4 + units * w.topk * 4   # Q, O, gates, idx
    per_block = summary_block_bytes(d, variance, rank, sub)
    select = units * w.nB * per_block + w.B * w.Hq * d * esz + units * w.topk * 4
    if variance in ("subspace", "subspace_fp4"):
        select += d * sub * 4   # the basis
    # summary update for the appended token: the completed block (64 K rows) and the last
    # compressed token (cmp_block K and V rows), plus their outputs
    update = units * (w.block * d * esz + per_block + 2 * w.cmp_block * d * esz + 2 * d * esz)
    return {"attn": attn, "select": select, "update": update, "total": attn + select + update,
            "kv_tokens_per_unit": kv_tokens / units}


# ------------------------------------------------------------------ CPU oracle

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


_ORACLE_STATE = {}


def _oracle_worker_init(w, shm_names, shapes, dtypes, Q, g, Pk, Pv, variance, rank, basis):
    """Pool worker: attach the shared K / V cache (no copy) and keep the small inputs."""
    import numpy as np
    from multiprocessing import shared_memory
    os.environ["OMP_NUM_THREADS"] = "1"
    shms = [shared_memory.SharedMemory(name=n) for n in shm_names]
    arrs = [np.ndarray(sh, dtype=dt, buffer=m.buf) for m, sh, dt in zip(shms, shapes, dtypes)]
    _ORACLE_STATE.update(w=w, shms=shms, K=arrs[0], V=arrs[1], Q=Q, g=g, Pk=Pk, Pv=Pv, variance=variance,
                         rank=rank, basis=basis)


def _oracle_worker_unit(unit):
    """The oracle (as it stands, float64) on one (batch, KV-head) unit: its idx row, its output
    rows and its near-tie report."""
    from oracle import cobs_oracle as O
    st = _ORACLE_STATE
    w = st["w"]
    b, h = unit
    res = O.decode(w, st["K"], st["V"], st["Q"], st["g"], st["Pk"], st["Pv"], units=[unit],
                   variance=st["variance"], rank=st["rank"], basis=st["basis"])
    return unit, res["idx"][b, h], res["O"][b, h * w.G:(h + 1) * w.G], res["near_ties"]


class OraclePool:
    """The oracle on all host cores: one process per core (spawned, so safe after CUDA is up),
    each taking whole (batch, KV-head) units; K and V are shared, not copied."""

    def __init__(self, w, K, V, Q, g, Pk, Pv, variance="channel", rank=4, basis=None, procs=None):
        import numpy as np
        from multiprocessing import get_context, shared_memory
        self.procs = procs or host_cores()
        self.shms = []
        names, shapes, dtypes = [], [], []
        for a in (K, V):
            a = np.ascontiguousarray(a)
            m = shared_memory.SharedMemory(create=True, size=max(1, a.nbytes))
            np.ndarray(a.shape, dtype=a.dtype, buffer=m.buf)[...] = a
            self.shms.append(m)
            names.append(m.name)
            shapes.append(a.shape)
            dtypes.append(a.dtype)
        os.environ.setdefault("OMP_NUM_THREADS", "1")
        self.pool = get_context("spawn").Pool(self.procs, initializer=_oracle_worker_init,
                                              initargs=(w, names, shapes, dtypes, Q, g, Pk, Pv, variance, rank,
                                                        basis))
        # every worker started before any timing (bounded: a worker that cannot start fails the run)
        self.pool.map_async(int, range(self.procs)).get(timeout=300)

    def run(self, units):
        """(seconds of wall time, results per unit)."""
        t0 = time.perf_counter()
        out = self.pool.map_async(_oracle_worker_unit, units, chunksize=1).get(timeout=3600)
        return time.perf_counter() - t0, out

    def close(self):
        self.pool.close()
        self.pool.join()
        for m in self.shms:
            m.close()
            m.unlink()


def decode_config(w, args, R=None, world=1):
    """The `config` object of a decode line (identical for both arms)."""
    cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T, "topk": w.topk,
           "window": w.window, "cmp_block": w.cmp_block, "cmp_stride": w.cmp_stride, "alpha": w.alpha,
           "variance": args.variance}
    if args.variance in ("lowrank", "lowrank_fp4", "subspace", "subspace_fp4"):
        cfg["rank"] = args.rank
    if args.variance in ("subspace", "subspace_fp4"):
        cfg.update(sub=args.sub, queries="concentrated in the subspace (leak 0.1)")
    cfg["step"] = ("cobs_decode_step: summary update at T-1, selection, then the decode attention as a "
                   "programmatic dependent of the selection; one CUDA graph")
    cfg["l2"] = f"{R or max(1, args.copies)} KV-cache copies rotated between steps (working set > L2)"
    cfg["parallelism"] = f"dp{world} (independent decode batches per GPU)"
    return cfg


def run_reference(args):
    """Reference arm: the CPU oracle on the host cores, every step all units of the workload
    spread over one process per core (rank 0 only)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import synth
    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.replace(B=args.batch)
    units_all = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    K, V = synth.kv_cache(w)
    Q, g = synth.queries_decode(w), synth.gates_decode(w)
    Pk, Pv = synth.projections(w)
    pool = OraclePool(w, K, V, Q, g, Pk, Pv)
    # a bounded sample per step: as many units as there are worker processes
    per_step = min(len(units_all), pool.procs)
    try:
        for i in range(args.warmup):
            pool.run([units_all[(i * per_step + j) % len(units_all)] for j in range(per_step)])
        secs, heads = 0.0, 0
        for i in range(args.steps):
            sec, _ = pool.run([units_all[(i * per_step + j) % len(units_all)] for j in range(per_step)])
            secs += sec
            heads += per_step * w.G
    finally:
        pool.close()
    value = heads / secs
    sample = (f"{per_step} (batch, KV-head) units of {w.name} per step ({per_step * w.G} query heads, "
              f"one process per unit), full oracle decode incl. summaries")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "query-heads/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(w, args, world=world),
        "cpu_baseline": {"value": value, "unit": "query-heads/s", "cores": pool.procs, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "query-heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def to_dev(a, dtype, dev):
    import numpy as np
    import torch
    if a is None:
        return None
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def read_tflops():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), "measured"
    return 1590.0, 1400.0, "fallback"


def prefill_flops(w, idx):
    """Algorithmic attention FLOPs of a causal prefill: 4 d per (position, head, attended key),
    from the selected blocks idx [B, T, Hkv, k] and the window / compressed-token visibility."""
    import numpy as np
    t = np.arange(w.T)
    win = np.minimum(w.window, t + 1).astype(np.int64)
    vis = np.where(t >= w.cmp_block - 1, np.minimum(w.nC, (t - w.cmp_block + 1) // w.cmp_stride + 1), 0)
    slc = (idx >= 0).sum(axis=-1).astype(np.int64) * w.block          # [B, T, Hkv]
    keys_per_group = slc + win[None, :, None] + vis[None, :, None]
    return float(4 * w.d * w.G * keys_per_group.sum())


def bench_prefill(w, steps, warmup, dev, cobs):
    """One step = full summary build + per-position selection + prefill attention."""
    import numpy as np
    import torch
    import synth
    p = cobs.Params(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T=w.T, topk=w.topk, window=w.window, block=w.block,
                    cmp_block=w.cmp_block, cmp_stride=w.cmp_stride, alpha=w.alpha, dtype=w.dtype)
    K, V = synth.kv_cache(w)
    Q, g = synth.queries_prefill(w), synth.gates_prefill(w)
    Pk, Pv = synth.projections(w)
    tQ, tK, tV = to_dev(Q, w.dtype, dev), to_dev(K, w.dtype, dev), to_dev(V, w.dtype, dev)
    tPk, tPv, tg = to_dev(Pk, "f32", dev), to_dev(Pv, "f32", dev), torch.from_numpy(g).to(dev)
    buf = cobs.alloc(p, prefill=True, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            cobs.prefill(p, tQ, tK, tV, tPk, tPv, tg, buf)
    stream.synchronize()
    n0 = cobs.launch_count()
    times = []
    with torch.cuda.stream(stream):
        for _ in range(steps):
            e = [ev() for _ in range(4)]
            e[0].record(stream)
            cobs.cobs_build_summaries(p, tK, tV, tPk, tPv, 0, buf.summaries, buf.Kc, buf.Vc)
            e[1].record(stream)
            cobs.cobs_select(p, tQ, buf.summaries, 1, buf.idx, buf.ws_select)
            e[2].record(stream)
            cobs.cobs_sparse_attn_prefill(p, tQ, tK, tV, buf.Kc, buf.Vc, buf.idx, tg, buf.O, buf.ws_attn)
            e[3].record(stream)
            times.append(e)
    torch.cuda.synchronize()
    launches = cobs.launch_count() - n0
    t_sum = sum(e[0].elapsed_time(e[1]) for e in times) / steps
    t_sel = sum(e[1].elapsed_time(e[2]) for e in times) / steps
    t_att = sum(e[2].elapsed_time(e[3]) for e in times) / steps
    flops = prefill_flops(w, buf.idx.cpu().numpy())
    burst, sustained, kind = read_tflops()
    att_tf = flops / (t_att * 1e-3) / 1e12
    kv_bytes = 2 * w.B * w.Hkv * w.T * w.d * 2
    return {
        "value": flops / ((t_sum + t_sel + t_att) * 1e-3) / 1e12, "unit": "TFLOP/s",
        "definition": "algorithmic attention FLOPs (4 d per position, head and attended key) / "
                      "(summary build + selection + attention)",
        "tflops_select_attn": flops / ((t_sel + t_att) * 1e-3) / 1e12,
        "ms": {"build_summaries": t_sum, "select": t_sel, "sparse_attn_prefill": t_att},
        "flops_per_step": flops,
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T, "topk": w.topk,
                   "window": w.window, "l2": "inputs larger than L2 (Q 0.5 GB)"},
        # the attention kernel is timed on its own (events on either side of its one launch):
        # the burst peak; the sustained one beside it
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel", "achieved": att_tf, "peak": burst,
                     "unit": "TFLOP/s", "frac": att_tf / burst, "peak_kind": f"{kind} burst bf16",
                     "frac_of_sustained": att_tf / sustained, "traffic": recorded_traffic("prefill_tc", traffic_key(w))},
        "summary_build_gbs": (kv_bytes + buf.summaries.numel() * 4 + 2 * buf.Kc.numel() * 2) / (t_sum * 1e-3) / 1e9,
        "gpu_launches": launches,
        "steps": steps,
        "device_error": cobs.device_error(),
    }


def traffic_ratios(w, idx, idx_a0, variance="channel", rank=4, sub=84):
    """KV-cache read traffic of one decode step ([COBS] §4.1 "Verkehrseffizienz"): dense attention
    (every K and V row of the context), COBS (its summaries, the compressed K/V and the K/V of the
    selected blocks and the window, from idx) and first-order mean-pool selection (alpha = 0: the
    means alone, the compressed K/V and the K/V of its own selected blocks and the window)."""
    d, esz = w.d, 2 if w.dtype == "bf16" else 4
    units = w.B * w.Hkv
    dense = units * w.T * 2 * d * esz
    cobs_b = decode_bytes(w, idx, variance, rank, sub)
    first = decode_bytes(w, idx_a0, "isotropic")
    # first order keeps only the block means: drop the isotropic scalar from the summary bytes
    first_sel = first["select"] - units * w.nB * 4
    cobs_read = cobs_b["select"] + cobs_b["attn"]
    first_read = first_sel + first["attn"]
    return {"dense_bytes": dense, "cobs_bytes": cobs_read, "first_order_bytes": first_read,
            "dense_over_cobs": dense / cobs_read, "cobs_over_first_order": cobs_read / first_read,
            "definition": "bytes read per decode step from idx: dense = all K/V rows; COBS = summaries + "
                          "compressed K/V + K/V of (selected blocks U window) + Q, gates, O; first order = "
                          "block means + the same with its own alpha = 0 selection"}


def measure_decode(w, args, dev, cobs, world, R, steps, warmup, with_e2e=True, clocks=True):
    """Time the decode step of workload w on this GPU (see the module docstring); returns the
    measurements, the selected blocks and outputs of copy 0, and the host inputs."""
    import numpy as np
    import torch
    import torch.distributed as dist
    import synth
    basis = synth.subspace_basis(w, args.sub) if args.variance in ("subspace", "subspace_fp4") else None
    p = cobs.Params(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T=w.T, topk=w.topk, window=w.window, block=w.block,
                    cmp_block=w.cmp_block, cmp_stride=w.cmp_stride, alpha=w.alpha, dtype=w.dtype,
                    variance=args.variance, rank=args.rank,
                    **(dict(sub=args.sub, basis=torch.from_numpy(basis).to(dev)) if basis is not None else {}))
    K, V = synth.kv_cache(w)
    Q = synth.queries_decode(w) if basis is None else synth.queries_decode_subspace(w, basis)
    g = synth.gates_decode(w)
    Pk, Pv = synth.projections(w)

    tQ, tg = to_dev(Q, w.dtype, dev), torch.from_numpy(g).to(dev)
    tPk, tPv = to_dev(Pk, "f32", dev), to_dev(Pv, "f32", dev)
    Ks = [to_dev(K, w.dtype, dev) for _ in range(R)]
    Vs = [to_dev(V, w.dtype, dev) for _ in range(R)]
    bufs = [cobs.alloc(p, prefill=False, device=dev) for _ in range(R)]
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for r in range(R):   # cache state: full summaries of every copy
            cobs.cobs_build_summaries(p, Ks[r], Vs[r], tPk, tPv, 0, bufs[r].summaries, bufs[r].Kc, bufs[r].Vc)
    stream.synchronize()
    cobs.device_error(reset=True)

    def step(r):
        cobs.decode_step(p, tQ, Ks[r], Vs[r], tPk, tPv, tg, bufs[r], t_begin=w.T - 1)

    # warm-up, then one CUDA graph per cache copy
    with torch.cuda.stream(stream):
        for i in range(max(3, warmup)):
            step(i % R)
    stream.synchronize()
    launches0 = cobs.launch_count()
    graphs = []
    for r in range(R):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            step(r)
        graphs.append(gr)
    launches_per_step = (cobs.launch_count() - launches0) // R
    for r in range(R):
        graphs[r].replay()
    stream.synchronize()
    idx0 = bufs[0].idx.cpu().numpy()
    O0 = bufs[0].O.float().cpu().numpy()
    # first-order (alpha = 0) selection on the same summaries, for the traffic comparison
    p0 = dataclasses.replace(p, alpha=0.0)
    idx_a0_t = torch.empty_like(bufs[0].idx)
    with torch.cuda.stream(stream):
        cobs.cobs_select(p0, tQ, bufs[0].summaries, 0, idx_a0_t, bufs[0].ws_select)
    stream.synchronize()
    idx_a0 = idx_a0_t.cpu().numpy()

    # ---- timed region: K graph replays, cache copies rotated (L2 defeat) ----
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    gpu = dev.index if dev.index is not None else 0
    with (ClockSampler(gpu) if clocks else contextlib.nullcontext()) as clk, torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(steps):
            graphs[i % R].replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
    if world > 1:
        dist.barrier()
    clk_summary = clk.summary() if clocks else None

    # ---- per-call durations: graphs of one part of the step each, replayed one at a time on the
    # launching stream with the same copy rotation (cold, isolated figures: no overlap with the
    # neighbouring kernels, so they add up to more than the step, whose attention grid overlaps the
    # selection as its programmatic dependent): the three separate calls; and the one-kernel
    # alternative (cobs_decode_step_fused with nothing to update) ----
    def timed_parts(build_parts, nparts):
        graphs_, evs_ = [], []
        for r in range(R):
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nparts + 1)]
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                evs[0].record(stream)
                for j, part in enumerate(build_parts(r)):
                    part()
                    evs[j + 1].record(stream)
            graphs_.append(gr)
            evs_.append(evs)
        out = []
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for i in range(steps + R):
                r = i % R
                graphs_[r].replay()
                stream.synchronize()
                if i >= R:   # the first pass over the copies is a warm-up
                    e = evs_[r]
                    out.append([e[j].elapsed_time(e[j + 1]) for j in range(nparts)])
        del graphs_
        # the mean, not the median: event pairs recorded inside a graph resolve about 2 us, so
        # single samples fall on that grid and only their mean resolves the launch's duration
        return [statistics.fmean(x[j] for x in out) for j in range(nparts)]

    def upd(r):
        return lambda: cobs.cobs_build_summaries(p, Ks[r], Vs[r], tPk, tPv, w.T - 1, bufs[r].summaries, bufs[r].Kc,
                                                 bufs[r].Vc)

    def fused_only(r):
        return lambda: cobs.cobs_decode_step_fused(p, tQ, Ks[r], Vs[r], tPk, tPv, w.T, bufs[r].summaries,
                                                   bufs[r].Kc, bufs[r].Vc, bufs[r].idx, tg, bufs[r].O,
                                                   bufs[r].ws_step_fused)

    has_fused = bufs[0].ws_step_fused is not None
    t_fused = timed_parts(lambda r: [fused_only(r)], 1)[0] if has_fused else None
    t_upd, t_sel, t_att = timed_parts(lambda r: [
        upd(r),
        lambda: cobs.cobs_select(p, tQ, bufs[r].summaries, 0, bufs[r].idx, bufs[r].ws_select),
        lambda: cobs.cobs_sparse_attn_decode(p, tQ, Ks[r], Vs[r], bufs[r].Kc, bufs[r].Vc, bufs[r].idx, tg,
                                             bufs[r].O, bufs[r].ws_attn)], 3)

    # the roofline kernel alone: one graph per copy holding only the attention call, each replay
    # timed by events on the launching stream outside the graph (no event nodes inside it)
    def time_alone(call):
        graphs_ = []
        for r in range(R):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                call(r)
            graphs_.append(gr)
        torch.cuda.synchronize()
        out = []
        with torch.cuda.stream(stream):
            for i in range(steps + R):
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                graphs_[i % R].replay()
                a1.record(stream)
                stream.synchronize()
                if i >= R:   # the first pass over the copies is a warm-up
                    out.append(a0.elapsed_time(a1))
        del graphs_
        return statistics.fmean(out)

    t_att = time_alone(lambda r: cobs.cobs_sparse_attn_decode(p, tQ, Ks[r], Vs[r], bufs[r].Kc, bufs[r].Vc,
                                                              bufs[r].idx, tg, bufs[r].O, bufs[r].ws_attn))
    # the same step through the three separate calls, and through the one-kernel alternative, each
    # as one graph per copy, for comparison with the headline
    def step_graph_ms(path):
        ugraphs = []
        for r in range(R):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                cobs.decode_step(p, tQ, Ks[r], Vs[r], tPk, tPv, tg, bufs[r], t_begin=w.T - 1, path=path)
            ugraphs.append(gr)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for i in range(R):
                ugraphs[i].replay()
            e0.record(stream)
            for i in range(steps):
                ugraphs[i % R].replay()
            e1.record(stream)
        torch.cuda.synchronize()
        del ugraphs
        return e0.elapsed_time(e1) / steps

    ms_calls = step_graph_ms("calls")
    ms_fused = step_graph_ms("fused") if has_fused else None

    e2e = None
    if with_e2e:
        e2e = measure_e2e(w, p, Q, g, Ks, Vs, bufs, tPk, tPv, tQ, tg, stream, dev, cobs, R, steps)
    out = {"ms": ms, "clocks": clk_summary, "t_upd": t_upd, "t_fused": t_fused, "t_sel": t_sel,
           "t_att": t_att, "ms_calls": ms_calls, "ms_fused": ms_fused, "e2e": e2e,
           "launches_per_step": launches_per_step,
           "device_error": cobs.device_error(), "idx0": idx0, "O0": O0, "idx_a0": idx_a0,
           "host": (K, V, Q, g, Pk, Pv, basis)}
    del graphs[:], Ks, Vs, bufs
    torch.cuda.empty_cache()
    return out


def measure_e2e(w, p, Q, g, Ks, Vs, bufs, tPk, tPv, tQ, tg, stream, dev, cobs, R, steps):
    """The step end to end through the public API: the step's inputs in one pinned host buffer
    (Q | gates | the appended token's K rows | its V rows, byte offsets 16-aligned), copied to the
    device with one host-to-device copy (Q and gates used in place, the K / V rows scattered into
    the cache at T-1), cobs_decode_step, and O back with one device-to-host copy."""
    import numpy as np
    import torch
    esz = 2 if w.dtype == "bf16" else 4
    nq, ng, nkv = Q.size * esz, g.size * 4, w.B * w.Hkv * w.d * esz
    offs = [0, nq, nq + ng, nq + ng + nkv]
    assert all(o % 16 == 0 for o in offs)
    h_in = torch.empty(offs[3] + nkv, dtype=torch.uint8).pin_memory()
    h_in[offs[0]:offs[1]].copy_(torch.from_numpy(np.ascontiguousarray(Q).view(np.uint8).reshape(-1)))
    h_in[offs[1]:offs[2]].copy_(torch.from_numpy(np.ascontiguousarray(g).view(np.uint8).reshape(-1)))
    h_in[offs[2]:offs[3]].copy_(Ks[0][:, :, w.T - 1].contiguous().view(torch.uint8).reshape(-1).cpu())
    h_in[offs[3]:].copy_(Vs[0][:, :, w.T - 1].contiguous().view(torch.uint8).reshape(-1).cpu())
    d_in = torch.empty_like(h_in, device=dev)
    dQ = d_in[offs[0]:offs[1]].view(tQ.dtype).view(tQ.shape)
    dg = d_in[offs[1]:offs[2]].view(torch.float32).view(tg.shape)
    dk = d_in[offs[2]:offs[3]].view(Ks[0].dtype).view(w.B, w.Hkv, w.d)
    dv = d_in[offs[3]:].view(Vs[0].dtype).view(w.B, w.Hkv, w.d)
    hO = torch.empty(bufs[0].O.shape, dtype=bufs[0].O.dtype).pin_memory()
    h2d = h_in.numel()
    d2h = hO.numel() * hO.element_size()

    def e2e_step(r):
        d_in.copy_(h_in, non_blocking=True)
        Ks[r][:, :, w.T - 1].copy_(dk)
        Vs[r][:, :, w.T - 1].copy_(dv)
        cobs.decode_step(p, dQ, Ks[r], Vs[r], tPk, tPv, dg, bufs[r], t_begin=w.T - 1)
        hO.copy_(bufs[r].O, non_blocking=True)

    # eager: every call issued from Python each step (host launch overhead included)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a0.record(stream)
        for i in range(steps):
            e2e_step(i % R)
        a1.record(stream)
    torch.cuda.synchronize()
    ms_eager = max_over_ranks(a0.elapsed_time(a1) / steps, dev)
    # the same step (copies in from pinned memory, the call, the copy out) captured once in a CUDA
    # graph per cache copy and replayed: how a serving loop would issue it
    e2e_graphs = []
    for r in range(R):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            e2e_step(r)
        e2e_graphs.append(gr)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(R):
            e2e_graphs[i].replay()
        a0.record(stream)
        for i in range(steps):
            e2e_graphs[i % R].replay()
        a1.record(stream)
    torch.cuda.synchronize()
    e2e_graphs.clear()
    ms_graph = max_over_ranks(a0.elapsed_time(a1) / steps, dev)
    return {"ms": ms_graph, "ms_eager": ms_eager, "h2d": h2d, "d2h": d2h}


def oracle_parity(w, idx_g, O_g, res_units, tol):
    """Compare the GPU's idx and outputs of copy 0 with the oracle results of the listed units."""
    import numpy as np
    same_idx, err, gaps = True, 0.0, []
    for (unit, idx_u, O_u, near) in res_units:
        b, h = unit
        same_idx &= bool(np.array_equal(idx_u, idx_g[b, h]))
        err = max(err, float(np.abs(O_u - O_g[b, h * w.G:(h + 1) * w.G]).max()))
        gaps += [gp for (_, _, gp) in near]
    return {"units": len(res_units), "idx_bit_exact": same_idx, "out_max_abs_err": err, "out_tol": tol,
            "fp64_near_ties": len(gaps), "fp64_near_tie_max_rel_gap": max(gaps) if gaps else None}


def traffic_key(w) -> str:
    """The workload a recorded ncu capture must have been taken on to stand for this run."""
    return f"{w.name} B={w.B} T={w.T}"


def decode_roofline(by, m, peak, peak_kind, workload):
    """Roofline of the step's dominant kernel, the three-branch decode attention (the largest share
    of the step's bytes), timed alone."""
    att_gbs = by["attn"] / (m["t_att"] * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "decode_stream_kernel (three-branch decode attention)",
            "achieved": att_gbs, "peak": peak, "unit": "GB/s", "frac": att_gbs / peak,
            "peak_kind": f"{peak_kind} (copy, read + write)", "algorithmic_bytes_per_launch": by["attn"],
            "timing": "CUDA events on the launching stream around each replay of a graph holding only "
                      "cobs_sparse_attn_decode (one graph per cache copy), mean over the timed replays",
            "traffic": recorded_traffic("decode_attention", workload)}


def decode_calls(by, m, peak):
    """Per-call durations and the alternative schedules of the same step."""
    out = {"build_summaries_update": m["t_upd"], "select": m["t_sel"], "sparse_attn_decode": m["t_att"],
           "select_gbs": by["select"] / (m["t_sel"] * 1e-3) / 1e9,
           "attn_gbs": by["attn"] / (m["t_att"] * 1e-3) / 1e9,
           "separate_calls_ms_per_step": m["ms_calls"]}
    if m["t_fused"] is not None:
        gbs = (by["select"] + by["attn"]) / (m["t_fused"] * 1e-3) / 1e9
        out["fused"] = {"ms_per_step": m["ms_fused"], "decode_step_kernel": m["t_fused"], "kernel_gbs": gbs,
                        "kernel_frac": gbs / peak,
                        "definition": "cobs_decode_step_fused: selection and attention in one persistent kernel"}
    return out


def decode_subrecord(name, args, dev, cobs, world, steps=50, warmup=5, R=4):
    """A decode workload other than the headline one, measured the same way (no end-to-end
    pass): step time, the attention kernel's roofline, traffic ratios, oracle parity on two units."""
    import synth
    w = synth.WORKLOADS[name]
    m = measure_decode(w, args, dev, cobs, world, R, steps, warmup, with_e2e=False, clocks=False)
    by = decode_bytes(w, m["idx0"], args.variance, args.rank, args.sub)
    peak, peak_kind = read_peaks()
    hbm = by["total"] / (m["ms"] * 1e-3) / 1e9
    rec = {"workload": name, "config": decode_config(w, args, R, world), "ms_per_step": m["ms"],
           "value": w.B * w.Hq * world / (m["ms"] * 1e-3), "unit": "query-heads/s",
           "hbm_gbs": hbm, "hbm_bytes_per_step": by["total"], "step_frac": hbm / peak,
           "roofline": decode_roofline(by, m, peak, peak_kind, traffic_key(w)),
           "calls_ms": decode_calls(by, m, peak),
           "traffic": traffic_ratios(w, m["idx0"], m["idx_a0"], args.variance, args.rank, args.sub),
           "gpu_launches": m["launches_per_step"] * steps, "steps": steps, "device_error": m["device_error"]}
    if not args.no_cpu_baseline:
        K, V, Q, g, Pk, Pv, basis = m["host"]
        pool = OraclePool(w, K, V, Q, g, Pk, Pv, args.variance, args.rank, basis, procs=min(2, host_cores()))
        try:
            _, res = pool.run([(0, 0), (w.B - 1, w.Hkv - 1)])
        finally:
            pool.close()
        rec["parity"] = oracle_parity(w, m["idx0"], m["O0"], res, 2e-2)
    return rec


def sweep_subrecord(args, dev, cobs, contexts):
    """The selector sweep at a few context lengths (GB/s and recall), as run_sweep measures it."""
    rows = sweep_rows(args, dev, cobs, contexts)
    return {"workload": "sweep", "contexts": contexts, "rows": rows,
            "definition": "cobs_select on 64 sequences x 8 KV heads (32 query heads, top-16); GB/s of the "
                          "summaries read; recall@16 of alpha = 1 and alpha = 0 against the exact-mass top-16 "
                          "on the first 8 sequences"}


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from block_sparse_long_summary_b200 import build as B
    if rank == 0:
        B.build()
    if world > 1:
        dist.barrier()
    from block_sparse_long_summary_b200 import cobs
    import synth

    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.replace(B=args.batch)
    if args.T:
        w = w.replace(T=args.T)
    if w.mode == "prefill":
        return run_prefill_line(args, w, dev, cobs, rank, world)
    R = max(1, args.copies)
    m = measure_decode(w, args, dev, cobs, world, R, args.steps, args.warmup)
    ms, e2e = m["ms"], m["e2e"]
    idx0, O0 = m["idx0"], m["O0"]
    qheads = w.B * w.Hq * world
    by = decode_bytes(w, idx0, args.variance, args.rank, args.sub)
    peak, peak_kind = read_peaks()
    result = {
        "metric": METRIC, "value": qheads / (ms * 1e-3), "unit": "query-heads/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": decode_config(w, args, R, world),
        "hbm_gbs": by["total"] / (ms * 1e-3) / 1e9,
        "hbm_bytes_per_step": by["total"],
        "step_frac": by["total"] / (ms * 1e-3) / 1e9 / peak,
        "roofline": decode_roofline(by, m, peak, peak_kind, traffic_key(w)),
        "calls_ms": decode_calls(by, m, peak),
        "traffic": traffic_ratios(w, idx0, m["idx_a0"], args.variance, args.rank, args.sub),
        "e2e": {"value": qheads / (e2e["ms"] * 1e-3), "unit": "query-heads/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e["ms"],
                "issue": "one CUDA graph per step: one H2D copy of Q, gates and the appended K/V rows "
                         "from pinned memory, the rows scattered into the cache, cobs_decode_step, one D2H "
                         "copy of O",
                "eager_value": qheads / (e2e["ms_eager"] * 1e-3), "eager_ms_per_step": e2e["ms_eager"]},
        "gpu_launches": m["launches_per_step"] * args.steps,
        "clocks": m["clocks"],
        "device_error": m["device_error"],
        "kv_tokens_per_unit": by["kv_tokens_per_unit"],
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle as it stands on every host core: all units of the workload, one process per core
        K, V, Q, g, Pk, Pv, basis = m["host"]
        units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
        pool = OraclePool(w, K, V, Q, g, Pk, Pv, args.variance, args.rank, basis)
        try:
            secs, res = pool.run(units)
        finally:
            pool.close()
        result["cpu_baseline"] = {"value": len(units) * w.G / secs, "unit": "query-heads/s", "cores": pool.procs,
                                  "kind": "oracle",
                                  "sample": f"all {len(units)} (batch, KV-head) units of {w.name} over "
                                            f"{pool.procs} processes, full oracle decode incl. summaries "
                                            f"({secs:.1f} s)"}
        # the same oracle run checks what the bench ran: indices bit for bit, outputs within 2e-2
        result["parity"] = oracle_parity(w, idx0, O0, res, 2e-2)
    if world == 1 and args.workload == "decode32k" and not args.no_subrecords:
        result["decode128k"] = decode_subrecord("decode128k", args, dev, cobs, world)
        result["sweep"] = sweep_subrecord(args, dev, cobs, [8192, 131072, 1048576])
    if not args.no_prefill and world == 1:
        wp = synth.WORKLOADS["prefill32k"]
        torch.cuda.empty_cache()
        result["prefill"] = bench_prefill(wp, args.prefill_steps, 2, dev, cobs)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_prefill_line(args, w, dev, cobs, rank, world):
    import torch.distributed as dist
    res = bench_prefill(w, args.steps, max(3, args.warmup), dev, cobs)
    ms = max_over_ranks(sum(res["ms"].values()), dev)
    line = {"metric": METRIC, "value": res["flops_per_step"] * world / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": res["config"], "roofline": res["roofline"], "calls_ms": res["ms"],
            "tflops_select_attn": res["tflops_select_attn"], "gpu_launches": res["gpu_launches"],
            "device_error": res["device_error"], "summary_build_gbs": res["summary_build_gbs"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ selector sweep over context length

def osa_top_k(E, k):
    """Indices of the k largest entries of E (ties to the lower index), ascending."""
    import numpy as np
    order = np.lexsort((np.arange(E.shape[0]), -E))
    return np.sort(order[:k])


def sweep_rows(args, dev, cobs, contexts):
    """Decode selection (cobs_select) on 64 sequences x 8 KV heads (32 query heads, top-16) at
    each context length: GB/s of the selector, and recall@16 of alpha = 1 and alpha = 0 against
    the oracle sparse attention (top-16 blocks by exact attention mass, from cobs_block_log_mass)
    on the first 8 sequences. Keys are drawn on the device; only summaries stay resident."""
    import numpy as np
    import torch
    import synth
    base = synth.WORKLOADS["sweep"]
    if args.batch:
        base = base.replace(B=args.batch)
    peak, peak_kind = read_peaks()
    n_rec = min(8, base.B)
    l2_bytes = 126e6
    rows = []
    stream = torch.cuda.Stream(device=dev)

    basis = synth.subspace_basis(base, args.sub) if args.variance in ("subspace", "subspace_fp4") else None
    tbasis = torch.from_numpy(basis).to(dev) if basis is not None else None
    qbasis = synth.subspace_basis(base, args.sub) if (basis is not None or args.subspace_queries) else None

    def params(w, **over):
        kw = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T=w.T, topk=w.topk, window=w.window, block=w.block,
                  cmp_block=w.cmp_block, cmp_stride=w.cmp_stride, alpha=w.alpha, dtype=w.dtype,
                  variance=args.variance, rank=args.rank)
        if basis is not None:
            kw.update(sub=args.sub, basis=tbasis)
        kw.update(over)
        return cobs.Params(**kw)

    for T in contexts:
        w = base.replace(T=T)
        p, p0, p1 = params(w), params(w, alpha=0.0), params(w, B=1)
        nB = T // w.block
        per_b = cobs.summaries_elems(p1)
        summ = torch.empty(w.B * per_b, dtype=torch.float32, device=dev)
        Kb = torch.empty((w.Hkv, T, w.d), dtype=torch.bfloat16, device=dev)
        nC = max(1, (T - w.cmp_block) // w.cmp_stride + 1)
        Kc = torch.empty((1, w.Hkv, nC, w.d), dtype=torch.bfloat16, device=dev)
        Vc = torch.empty_like(Kc)
        Pk, Pv = synth.projections(w)
        tPk, tPv = to_dev(Pk, "f32", dev), to_dev(Pv, "f32", dev)
        tQ = to_dev(synth.queries_decode(w) if qbasis is None else synth.queries_decode_subspace(w, qbasis), "bf16",
                    dev)
        mass = torch.empty((n_rec, w.Hq, nB), dtype=torch.float32, device=dev)
        n0 = cobs.launch_count()
        with torch.cuda.stream(stream):
            for b in range(w.B):
                for h in range(w.Hkv):
                    synth.keys_unit_on_device(w, b, h, Kb[h], stream=stream, aniso_rank=args.aniso)
                cobs.cobs_build_summaries(p1, Kb, Kb, tPk, tPv, 0, summ[b * per_b:(b + 1) * per_b], Kc, Vc)
                if b < n_rec:
                    cobs.cobs_block_log_mass(p1, tQ[b:b + 1], Kb, mass[b:b + 1])
        stream.synchronize()
        del Kb, Kc, Vc
        # L2 defeat: enough summary copies that the rotated working set exceeds 4 x L2
        sbytes = summ.numel() * 4
        R = max(1, min(16, int(np.ceil(4 * l2_bytes / sbytes))))
        copies = [summ] + [summ.clone() for _ in range(R - 1)]
        idx = torch.empty((w.B, w.Hkv, w.topk), dtype=torch.int32, device=dev)
        ws = torch.zeros(max(16, cobs.workspace_bytes(p, cobs.COBS_WS_SELECT)), dtype=torch.uint8, device=dev)
        with torch.cuda.stream(stream):
            cobs.cobs_select(p0, tQ, summ, 0, idx, ws)
        stream.synchronize()
        idx_a0 = idx.cpu().numpy()
        graphs = []
        for r in range(R):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                cobs.cobs_select(p, tQ, copies[r], 0, idx, ws)
            graphs.append(gr)
        n_rep = max(20, 3 * R)
        with torch.cuda.stream(stream):
            for i in range(max(3, args.warmup) * R):
                graphs[i % R].replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(n_rep):
                graphs[i % R].replay()
            e1.record(stream)
        stream.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / n_rep
        idx_a1 = idx.cpu().numpy()
        launches = cobs.launch_count() - n0
        m = mass.cpu().numpy().astype(np.float64)
        rec1, rec0 = [], []
        for b in range(n_rec):
            for g in range(w.Hkv):
                osa = osa_top_k(m[b, g * w.G:(g + 1) * w.G].sum(axis=0), w.topk)
                ref = set(osa.tolist())
                rec1.append(len(ref & set(int(x) for x in idx_a1[b, g] if x >= 0)) / w.topk)
                rec0.append(len(ref & set(int(x) for x in idx_a0[b, g] if x >= 0)) / w.topk)
        per_block = summary_block_bytes(w.d, args.variance, args.rank, args.sub)
        by = w.B * w.Hkv * nB * per_block + w.B * w.Hq * w.d * 2 + w.B * w.Hkv * w.topk * 4
        gbs = by / (us * 1e-6) / 1e9
        rows.append({"T": T, "nB": nB, "bytes": by, "us": us, "gbs": gbs, "frac": gbs / peak,
                     "recall_alpha1": float(np.mean(rec1)), "recall_alpha0": float(np.mean(rec0)),
                     "l2": f"{R} summary copies rotated" if R > 1 else "summaries larger than L2",
                     "gpu_launches": launches, "steps": n_rep})
        del graphs, copies, summ, mass
        torch.cuda.empty_cache()
    return rows


def run_sweep(args):
    """The selector sweep as its own line (sweep_rows over the listed or all context lengths)."""
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from block_sparse_long_summary_b200 import build as B
    B.build()
    from block_sparse_long_summary_b200 import cobs
    import synth
    base = synth.WORKLOADS["sweep"]
    if args.batch:
        base = base.replace(B=args.batch)
    contexts = [int(x) for x in args.contexts.split(",")] if args.contexts else list(synth.SWEEP_CONTEXTS)
    peak, peak_kind = read_peaks()
    n_rec = min(8, base.B)
    rows = sweep_rows(args, dev, cobs, contexts)
    basis_used = args.variance in ("subspace", "subspace_fp4") or args.subspace_queries
    top = rows[-1]
    line = {"metric": "selector GB/s over context length (decode selection, 64 x 8 units, top-16)",
            "value": top["gbs"], "unit": "GB/s", "n_gpus": 1, "steps": top["steps"], "warmup": max(3, args.warmup),
            "ms_per_step": top["us"] * 1e-3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (keys drawn on the device" +
                                    (f", anisotropic blocks of rank {args.aniso})" if args.aniso else ")"),
            "config": {"workload": "sweep", "B": base.B, "Hq": base.Hq, "Hkv": base.Hkv, "d": base.d,
                       "topk": base.topk, "contexts": contexts, "variance": args.variance,
                       **({"sub": args.sub, "queries": "concentrated in the subspace (leak 0.1)"}
                          if basis_used else {}),
                       "recall_on": f"first {n_rec} sequences x {base.Hkv} KV heads"},
            "roofline": {"bound": "hbm", "kernel": "select_decode_kernel", "achieved": top["gbs"], "peak": peak,
                         "unit": "GB/s", "frac": top["frac"], "peak_kind": peak_kind,
                         "traffic": recorded_traffic("select_decode", "sweep")},
            "sweep": rows, "gpu_launches": sum(r["gpu_launches"] for r in rows), "device_error": cobs.device_error()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "sweep":
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
