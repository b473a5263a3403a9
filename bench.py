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
    ap.add_argument("--variance", choices=["channel", "isotropic", "lowrank", "lowrank_fp4", "subspace"],
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
    "decode_attention": ["decode_stream.cu", "common.cuh", "dims.h", "tma.cu", "tma.h"],
    "select_decode": ["select.cu", "common.cuh", "dims.h"],
    "prefill_tc": ["prefill.cu", "tc.cuh", "common.cuh", "dims.h", "tma.cu", "tma.h"],
}


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for fn in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(CSRC, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken on the
    current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(kernel)
    if not ent or ent.get("source_hash") != source_hash(kernel):
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
            "subspace": (d + rank * sub + rank) * 4}.get(variance, 2 * d * 4)


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
    if variance == "subspace":
        select += d * sub * 4   # the basis
    # summary update for the appended token: the completed block (64 K rows) and the last
    # compressed token (cmp_block K and V rows), plus their outputs
    update = units * (w.block * d * esz + per_block + 2 * w.cmp_block * d * esz + 2 * d * esz)
    return {"attn": attn, "select": select, "update": update, "total": attn + select + update,
            "kv_tokens_per_unit": kv_tokens / units}


# ------------------------------------------------------------------ CPU oracle

def oracle_decode_sample(w, K, V, Q, g, Pk, Pv, units, with_result=False, variance="channel", rank=4,
                         basis=None):
    """Time the oracle (as it stands) on the listed units; returns (seconds, query heads[, result])."""
    from oracle import cobs_oracle as O
    t0 = time.perf_counter()
    res = O.decode(w, K, V, Q, g, Pk, Pv, units=units, variance=variance, rank=rank, basis=basis)
    secs = time.perf_counter() - t0
    return (secs, len(units) * w.G, res) if with_result else (secs, len(units) * w.G)


def limit_threads():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        return None


def run_reference(args):
    """Reference arm: the CPU oracle on host cores, bounded sample per step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import synth
    w = synth.WORKLOADS[args.workload]
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    lim = limit_threads()
    units_all = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    K, V = synth.kv_cache(w)
    Q, g = synth.queries_decode(w), synth.gates_decode(w)
    Pk, Pv = synth.projections(w)
    per_step = 1
    for i in range(args.warmup):
        oracle_decode_sample(w, K, V, Q, g, Pk, Pv, [units_all[i % len(units_all)]])
    secs, heads = 0.0, 0
    for i in range(args.steps):
        s, hh = oracle_decode_sample(w, K, V, Q, g, Pk, Pv, [units_all[i % len(units_all)]])
        secs += s
        heads += hh
    value = heads / secs
    sample = f"{per_step} (batch, KV-head) unit of {w.name} per step ({w.G} query heads), full oracle decode"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "query-heads/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T, "topk": w.topk,
                   "window": w.window},
        "cpu_baseline": {"value": value, "unit": "query-heads/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "query-heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    del lim
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
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel", "achieved": att_tf, "peak": sustained,
                     "unit": "TFLOP/s", "frac": att_tf / sustained, "peak_kind": f"{kind} sustained bf16",
                     "traffic": recorded_traffic("prefill_tc")},
        "summary_build_gbs": (kv_bytes + buf.summaries.numel() * 4 + 2 * buf.Kc.numel() * 2) / (t_sum * 1e-3) / 1e9,
        "gpu_launches": launches,
        "steps": steps,
        "device_error": cobs.device_error(),
    }


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
    basis = synth.subspace_basis(w, args.sub) if args.variance == "subspace" else None
    p = cobs.Params(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T=w.T, topk=w.topk, window=w.window, block=w.block,
                    cmp_block=w.cmp_block, cmp_stride=w.cmp_stride, alpha=w.alpha, dtype=w.dtype,
                    variance=args.variance, rank=args.rank,
                    **(dict(sub=args.sub, basis=torch.from_numpy(basis).to(dev)) if basis is not None else {}))
    K, V = synth.kv_cache(w)
    Q = synth.queries_decode(w) if basis is None else synth.queries_decode_subspace(w, basis)
    g = synth.gates_decode(w)
    Pk, Pv = synth.projections(w)

    R = max(1, args.copies)
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
        for i in range(max(3, args.warmup)):
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

    # ---- timed region: K graph replays, cache copies rotated (L2 defeat) ----
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk, torch.cuda.stream(stream):   # replay() launches on the current stream
        e0.record(stream)
        for i in range(args.steps):
            graphs[i % R].replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    if world > 1:
        dist.barrier()
    clocks = clk.summary()

    # ---- per-call durations inside the step: a second set of step graphs with timing events
    # captured between the calls (event-record nodes), replayed one at a time on the launching
    # stream with the same copy rotation; the headline graphs above carry no events ----
    tgraphs, tevs = [], []
    for r in range(R):
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            evs[0].record(stream)
            cobs.cobs_build_summaries(p, Ks[r], Vs[r], tPk, tPv, w.T - 1, bufs[r].summaries, bufs[r].Kc, bufs[r].Vc)
            evs[1].record(stream)
            cobs.cobs_select(p, tQ, bufs[r].summaries, 0, bufs[r].idx, bufs[r].ws_select)
            evs[2].record(stream)
            cobs.cobs_sparse_attn_decode(p, tQ, Ks[r], Vs[r], bufs[r].Kc, bufs[r].Vc, bufs[r].idx, tg, bufs[r].O,
                                         bufs[r].ws_attn)
            evs[3].record(stream)
        tgraphs.append(gr)
        tevs.append(evs)
    t_parts = []
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.steps + R):
            r = i % R
            tgraphs[r].replay()
            stream.synchronize()
            if i >= R:   # the first pass over the copies is a warm-up
                e = tevs[r]
                t_parts.append((e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])))
    t_upd = statistics.median(x[0] for x in t_parts)
    t_sel = statistics.median(x[1] for x in t_parts)
    t_att = statistics.median(x[2] for x in t_parts)
    del tgraphs

    # ---- end to end through the public API: pinned host inputs in, output back, every step ----
    # The step's inputs travel in one pinned host buffer: Q | gates | the appended token's K rows
    # | its V rows (byte offsets 16-aligned), copied to a device staging buffer with one
    # host-to-device copy; Q and gates are used in place, the K / V rows are scattered into
    # the cache at T-1. O comes back with one device-to-host copy.
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
        for i in range(args.steps):
            e2e_step(i % R)
        a1.record(stream)
    torch.cuda.synchronize()
    ms_e2e_eager = max_over_ranks(a0.elapsed_time(a1) / args.steps, dev)
    # the same step (copies in from pinned memory, the three calls, the copy out) captured once
    # in a CUDA graph per cache copy and replayed: how a serving loop would issue it
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
        for i in range(args.steps):
            e2e_graphs[i % R].replay()
        a1.record(stream)
    torch.cuda.synchronize()
    e2e_graphs.clear()
    ms_e2e = max_over_ranks(a0.elapsed_time(a1) / args.steps, dev)
    dev_err = cobs.device_error()

    qheads = w.B * w.Hq * world
    by = decode_bytes(w, idx0, args.variance, args.rank, args.sub)
    peak, peak_kind = read_peaks()
    att_gbs = by["attn"] / (t_att * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": qheads / (ms * 1e-3), "unit": "query-heads/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T, "topk": w.topk,
                   "window": w.window, "cmp_block": w.cmp_block, "cmp_stride": w.cmp_stride, "alpha": w.alpha,
                   "variance": args.variance,
                   **({"rank": args.rank} if args.variance in ("lowrank", "lowrank_fp4", "subspace") else {}),
                   **({"sub": args.sub, "queries": "concentrated in the subspace (leak 0.1)"}
                      if args.variance == "subspace" else {}),
                   "step": "summary update at T-1 + select + decode attention, one CUDA graph",
                   "l2": f"{R} KV-cache copies rotated between steps (working set {R} x step bytes > L2)",
                   "parallelism": f"dp{world} (independent decode batches per GPU)"},
        "hbm_gbs": by["total"] / (ms * 1e-3) / 1e9,
        "hbm_bytes_per_step": by["total"],
        "roofline": {"bound": "hbm", "kernel": "cobs_sparse_attn_decode (decode_stream_kernel + decode_stream_merge)",
                     "achieved": att_gbs, "peak": peak, "unit": "GB/s", "frac": att_gbs / peak,
                     "peak_kind": peak_kind, "algorithmic_bytes_per_launch": by["attn"],
                     "traffic": recorded_traffic("decode_attention")},
        "calls_ms": {"build_summaries_update": t_upd, "select": t_sel, "sparse_attn_decode": t_att,
                     "select_gbs": by["select"] / (t_sel * 1e-3) / 1e9},
        "e2e": {"value": qheads / (ms_e2e * 1e-3), "unit": "query-heads/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                "issue": "one CUDA graph per step: one H2D copy of Q, gates and the appended K/V rows "
                         "from pinned memory, the rows scattered into the cache, cobs_build_summaries + "
                         "cobs_select + cobs_sparse_attn_decode, one D2H copy of O",
                "eager_value": qheads / (ms_e2e_eager * 1e-3), "eager_ms_per_step": ms_e2e_eager},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "device_error": dev_err,
        "kv_tokens_per_unit": by["kv_tokens_per_unit"],
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        os.environ.setdefault("OMP_NUM_THREADS", "1")
        lim = limit_threads()
        units = [(b, h) for b in range(w.B) for h in range(w.Hkv)][:24]
        secs, heads, ref = oracle_decode_sample(w, K, V, Q, g, Pk, Pv, units, with_result=True,
                                                variance=args.variance, rank=args.rank, basis=basis)
        result["cpu_baseline"] = {"value": heads / secs, "unit": "query-heads/s", "cores": 1, "kind": "oracle",
                                  "sample": f"{len(units)} of {w.B * w.Hkv} (batch, KV-head) units of {w.name}, "
                                            f"full oracle decode incl. summaries ({secs:.1f} s)"}
        # the same oracle run checks what the bench ran: indices bit for bit, outputs within 2e-2
        same_idx = all(np.array_equal(ref["idx"][b, h], idx0[b, h]) for (b, h) in units)
        err = max(float(np.abs(ref["O"][b, h * w.G:(h + 1) * w.G] - O0[b, h * w.G:(h + 1) * w.G]).max())
                  for (b, h) in units)
        gaps = [gp for (_, _, gp) in ref["near_ties"]]
        result["parity"] = {"units": len(units), "idx_bit_exact": same_idx, "out_max_abs_err": err,
                            "out_tol": 2e-2,
                            "fp64_near_ties": len(gaps), "fp64_near_tie_max_rel_gap": max(gaps) if gaps else None}
        del lim
    if not args.no_prefill and world == 1:
        wp = synth.WORKLOADS["prefill32k"]
        del Ks, Vs, bufs, graphs[:]
        torch.cuda.empty_cache()
        result["prefill"] = bench_prefill(wp, args.prefill_steps, 2, dev, cobs)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        graphs.clear()
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


def run_sweep(args):
    """Decode selection (cobs_select) on 64 sequences x 8 KV heads (32 query heads, top-16) at
    each context length: GB/s of the selector, and recall@16 of alpha = 1 and alpha = 0 against
    the oracle sparse attention (top-16 blocks by exact attention mass, from cobs_block_log_mass)
    on the first 8 sequences. Keys are drawn on the device; only summaries stay resident."""
    import numpy as np
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
    l2_bytes = 126e6
    rows, launches = [], 0
    stream = torch.cuda.Stream(device=dev)

    basis = synth.subspace_basis(base, args.sub) if args.variance == "subspace" else None
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
        launches += cobs.launch_count() - n0
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
                     "l2": f"{R} summary copies rotated" if R > 1 else "summaries larger than L2"})
        del graphs, copies, summ, mass
        torch.cuda.empty_cache()
    top = rows[-1]
    line = {"metric": "selector GB/s over context length (decode selection, 64 x 8 units, top-16)",
            "value": top["gbs"], "unit": "GB/s", "n_gpus": 1, "steps": n_rep, "warmup": max(3, args.warmup),
            "ms_per_step": top["us"] * 1e-3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (keys drawn on the device" +
                                    (f", anisotropic blocks of rank {args.aniso})" if args.aniso else ")"),
            "config": {"workload": "sweep", "B": base.B, "Hq": base.Hq, "Hkv": base.Hkv, "d": base.d,
                       "topk": base.topk, "contexts": contexts, "variance": args.variance,
                       **({"sub": args.sub, "queries": "concentrated in the subspace (leak 0.1)"}
                          if qbasis is not None else {}),
                       "recall_on": f"first {n_rec} sequences x {base.Hkv} KV heads"},
            "roofline": {"bound": "hbm", "kernel": "select_decode_kernel", "achieved": top["gbs"], "peak": peak,
                         "unit": "GB/s", "frac": top["frac"], "peak_kind": peak_kind,
                         "traffic": recorded_traffic("select_decode")},
            "sweep": rows, "gpu_launches": launches, "device_error": cobs.device_error()}
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
