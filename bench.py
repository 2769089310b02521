#!/usr/bin/env python
"""Decode-step throughput of the BasisKV hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one decode step of one attention layer for every sequence of the
batch: append (latent + residual + page summary), route (page scores + top-k),
decode_attn (exact attention on the routed pages), out_proj (fused factor).
The metric is decode tokens/s per layer (batch / step time).  The whole step
(append on a forked stream concurrently with route, then decode_attn and
out_proj) is captured once into a CUDA graph; a timed step is one replay
bracketed by CUDA events on the launching stream.  A second pass replays one
graph per phase, with events between them, for the per-kernel breakdown and
the roofline of the attention kernel.  L2 is flushed before every step by
reading a 256 MiB buffer (outside the events).

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica on its own sequences (weak scaling; the path has no exchange step);
``--tp`` instead shards the heads of one workload over the ranks and adds one
NCCL all-reduce of the layer output per step (strong scaling).
``--routing group_sum|group_max`` routes once per KV group instead of once per
query head.  After the decode measurements the line also reports the prefill
append of the whole context (tensor-core path and fp64 path; ``prefill``).
``--impl reference`` times the fp64 CPU oracle on the same workload instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402

METRIC = "decode tokens/s per layer on 1 B200; route+attn HBM GB/s vs ~8 TB/s roofline"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
# kernels one decode step launches: append_decode, route_score, route_select,
# the sparse attention kernel (union slice, attention and split merge in one
# launch) and the out-projection kernel
KERNELS_PER_STEP = 5


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="llama3_8b_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--context", type=int, default=None,
                    help="tokens per sequence instead of the workload's (a smaller case of the same "
                         "kernels, for profiling; a ragged workload becomes uniform)")
    ap.add_argument("--routing", default="head", choices=["head", "group_sum", "group_max"],
                    help="one page selection per query head (the method as stated), or per KV group")
    ap.add_argument("--oracle-repeats", type=int, default=200,
                    help="decode steps per host process in the CPU baseline, at most")
    ap.add_argument("--oracle-budget", type=float, default=3.0,
                    help="seconds each host process spends on decode steps in the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill-append measurement")
    ap.add_argument("--tp", action="store_true",
                    help="shard the heads of one workload over the N ranks (one NCCL all-reduce of y per "
                         "step) instead of running N independent replicas")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world > 1:
        import datetime
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def chosen_workload(args):
    """The named workload, or a shorter-context case of it (--context)."""
    wl = WORKLOADS[args.workload]
    if args.context is not None:
        wl = dataclasses.replace(shrink(wl, context=args.context, name=f"{wl.name}@{args.context}"), ragged=None)
    return wl


def replica_workload(wl, rank: int, world: int):
    """Weak scaling: every rank decodes its own sequences (a different seed per rank)."""
    if world > 1:
        return dataclasses.replace(wl, seed=wl.seed + 1000 * rank)
    return wl


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled from a thread)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int, period_s: float = 0.001):
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # noqa: BLE001
            self.err = repr(exc)
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                try:
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append(mhz)
                self.reasons |= int(rs)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        names = [k for k, v in self.REASONS.items() if self.reasons & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "window": "warm-up, timed steps, per-phase pass and end-to-end pass"}


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must move)
# ---------------------------------------------------------------------------
def algorithmic_bytes(eng):
    case, cfg = eng.case, eng.cfg
    wl = case.wl
    es = 2 if wl.dtype == "bf16" else 4
    B, Hq, Hkv, d, r, s, P, k = (wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.rank_v,
                                 wl.rank_k, wl.page_size, wl.top_k)
    G = Hq // Hkv
    pages = [-(-L // P) for L in case.lengths]
    sel = eng.sel.cpu().numpy()
    cnt = eng.sel_cnt.cpu().numpy()
    score_rows = Hq if eng.routing == "head" else Hkv
    union = 0
    for b in range(B):
        for g in range(Hkv):
            u = set()
            for h in range(g * G, (g + 1) * G):
                u.update(sel[b, h, :cnt[b, h]].tolist())
            union += len(u)
    q_bytes = B * Hq * d * es
    sel_bytes = B * Hq * (k + 2) * 4
    route = sum(pages) * Hkv * d * 4 + 2 * sum(pages) * score_rows * 4 + q_bytes + sel_bytes
    decode = union * P * (d + r) * es + q_bytes + sel_bytes + B * Hq * r * 4
    out = Hq * r * wl.hidden * es + B * Hq * r * 4 + B * wl.hidden * 4
    append = B * Hkv * ((2 * d * r + d * s) * es + 2 * d * es + P * (r + s) * es + d * 4)
    return {"append": append, "route": route, "decode_attn": decode, "out_proj": out,
            "union_pages": union}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(kernel_file: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "long_context_decode_basiskv_b200", "csrc", kernel_file)
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if rec.get("source_sha256") != sha:
            return None
        return rec
    except Exception:  # noqa: BLE001
        return None


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample, on every host core
# ---------------------------------------------------------------------------
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - not Linux
        return os.cpu_count() or 1


def _oracle_worker(conn, path: str, b: int, wl_fields: dict, routing: str):
    """One host process: load sequence b of the dumped case, build its oracle
    cache (untimed), then on each request run `repeats` decode steps of that
    sequence and send back (start, end, per-step seconds)."""
    from threadpoolctl import threadpool_limits

    from oracle import basiskv_oracle as O

    with threadpool_limits(1):
        storage = wl_fields["storage"]
        fac = np.load(os.path.join(path, "factors.npz"))
        A, P, E = (fac[k].astype(np.float64) for k in ("A", "P", "E"))
        G = O.fuse_out_factor(fac["Bf"].astype(np.float64), fac["W_O"].astype(np.float64),
                              wl_fields["num_q_heads"], storage)
        seq = np.load(os.path.join(path, f"seq{b}.npz"))
        K, V, q = (seq[k].astype(np.float64) for k in ("K", "V", "q"))
        L = K.shape[0]
        cache = O.prefill(K[:-1], V[:-1], A, P, E, wl_fields["page_size"], storage, capacity=L)
        conn.send("ready")
        while True:
            req = conn.recv()
            if req is None:
                break
            repeats, budget = req
            times = []
            t_start = time.perf_counter()
            while len(times) < repeats and (budget is None or time.perf_counter() - t_start < budget):
                cache.length = L - 1
                t0 = time.perf_counter()
                O.decode_step(cache, K[-1], V[-1], q, A, P, E, G, wl_fields["top_k"], routing=routing)
                times.append(time.perf_counter() - t0)
            conn.send((t_start, time.perf_counter(), times))
    conn.close()


class OracleHost:
    """The fp64 oracle on the host cores: one spawned process per core, each
    decoding one sequence of the case (sequence i mod B on process i), with
    one BLAS thread each.  The case's tensors travel through files in a
    temporary directory (storage values, converted exactly to fp64 by the
    workers).  Processes are capped by free host memory."""

    def __init__(self, case, routing: str = "head", workers: int | None = None):
        import multiprocessing as mp
        import tempfile

        wl = case.wl
        self.wl, self.routing = wl, routing
        cores = host_cores()
        L_max = max(case.lengths)
        per_worker = (L_max * wl.num_kv_heads * 8 * (3 * wl.head_dim + wl.rank_v + wl.rank_k)
                      + wl.num_q_heads * wl.rank_v * wl.hidden * 8 * 2 + (256 << 20))
        try:
            import psutil
            mem_cap = max(1, int(psutil.virtual_memory().available * 0.5 // per_worker))
        except Exception:  # noqa: BLE001
            mem_cap = cores
        self.workers = max(1, min(workers or cores, cores, mem_cap))
        self.dir = tempfile.mkdtemp(prefix="bkv_oracle_", dir="/dev/shm" if os.path.isdir("/dev/shm") else None)

        def f32(t):
            return t.detach().to("cpu", torch.float32).numpy()

        np.savez(os.path.join(self.dir, "factors.npz"), A=f32(case.A), P=f32(case.P), E=f32(case.E),
                 Bf=f32(case.Bf), W_O=f32(case.W_O))
        seqs = sorted({i % wl.batch for i in range(self.workers)})
        for b in seqs:
            np.savez(os.path.join(self.dir, f"seq{b}.npz"), K=f32(case.keys[b]), V=f32(case.values[b]),
                     q=f32(case.q[b]))
        fields = {"storage": "f32" if wl.dtype == "f32" else "bf16", "num_q_heads": wl.num_q_heads,
                  "page_size": wl.page_size, "top_k": wl.top_k}
        ctx = mp.get_context("spawn")
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        self.procs, self.conns = [], []
        try:
            for i in range(self.workers):
                parent, child = ctx.Pipe()
                p = ctx.Process(target=_oracle_worker, args=(child, self.dir, i % wl.batch, fields, routing),
                                daemon=True)
                p.start()
                self.procs.append(p)
                self.conns.append(parent)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        for c in self.conns:
            if c.recv() != "ready":
                raise RuntimeError("oracle worker failed to start")

    def run(self, repeats: int, workers: int | None = None, budget: float | None = None):
        """Up to `repeats` decode steps (stopping after `budget` seconds, if given) on
        each of the first `workers` processes at once.  Returns (steps, wall seconds
        from the first start to the last end, all step times)."""
        use = self.conns[:workers or self.workers]
        for c in use:
            c.send((repeats, budget))
        res = [c.recv() for c in use]
        wall = max(r[1] for r in res) - min(r[0] for r in res)
        times = [t for r in res for t in r[2]]
        return len(times), wall, times

    def close(self):
        import shutil

        for c in self.conns:
            try:
                c.send(None)
            except Exception:  # noqa: BLE001
                pass
        for p in self.procs:
            p.join(timeout=30)
            if p.is_alive():
                p.terminate()
        shutil.rmtree(self.dir, ignore_errors=True)

    def describe(self, what: str) -> str:
        wl = self.wl
        return (f"fp64 numpy oracle on {self.workers} host processes (1 BLAS thread each; "
                f"{host_cores()} cores available): process i decodes sequence i mod {wl.batch} of the "
                f"workload, {what} (decode step = append, summary, {self.routing} route, attention, "
                f"out-projection), prefill untimed; value = decode steps / wall time")


def cpu_baseline(case, routing: str, repeats: int, budget: float):
    """The oracle on all host cores (throughput of independent decode steps), plus
    the same decode step on one core alone.  Each process runs up to `repeats`
    steps and stops after `budget` seconds."""
    host = OracleHost(case, routing)
    try:
        n1, w1, _ = host.run(repeats, workers=1, budget=budget)
        steps, wall, _ = host.run(repeats, budget=budget)
    finally:
        host.close()
    return {"value": round(steps / wall, 3), "unit": UNIT, "cores": host.workers, "kind": "oracle",
            "sample": host.describe(f"{steps // host.workers} decode steps per process"),
            "seconds": round(wall, 3), "cpu_seconds": round(wall * host.workers, 1),
            "single_thread": {"value": round(n1 / w1, 3), "unit": UNIT, "cores": 1,
                              "sample": f"one process alone: {n1} decode steps of sequence 0"}}


# ---------------------------------------------------------------------------
# prefill append: the whole context of every sequence in one call
# ---------------------------------------------------------------------------
def measure_prefill(eng, stream, reps: int = 3):
    """Time basiskv_prefill (tensor cores) and basiskv_append (fp64) rebuilding the
    cache of all but the last token of every sequence (equal lengths only: one
    call for the batch).  Runs after the decode measurements; it rewrites the
    cache with the tensor-core values.  Returns a dict, or None for ragged batches."""
    from long_context_decode_basiskv_b200 import binding as bk

    case, cfg = eng.case, eng.cfg
    lengths = set(case.lengths)
    if len(lengths) != 1 or cfg.dtype != torch.bfloat16:
        return None
    L = lengths.pop()
    B = case.wl.batch
    k = torch.stack([x[:-1] for x in case.keys]).contiguous()
    v = torch.stack([x[:-1] for x in case.values]).contiguous()
    sub = bk.PagedCache.__new__(bk.PagedCache)
    sub.__dict__.update(eng.cache.__dict__)
    sub.seq_len = torch.full((B,), L - 1, dtype=torch.int32, device=k.device)
    res = {"tokens": B * (L - 1)}
    with torch.cuda.stream(stream):
        for name, fn in [("tensor_core", bk.prefill), ("fp64_append", bk.append)]:
            fn(cfg, sub, eng.factors, k, v, eng.err)  # warm-up
            evs = []
            for _ in range(reps):
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn(cfg, sub, eng.factors, k, v, eng.err)
                b_.record(stream)
                evs.append((a, b_))
            torch.cuda.synchronize()
            us = sum(a.elapsed_time(b_) for a, b_ in evs) / reps * 1e3
            res[name] = {"us": round(us, 1), "tokens_per_s": round(B * (L - 1) / (us * 1e-6), 1)}
    # bytes the tensor-core path must move: k, v in; raw k, C, R out; C, R re-read for the
    # summaries; one fp32 summary row per page and head
    d, r, s_, P = cfg.head_dim, cfg.rank_v, cfg.rank_k, cfg.page_size
    tok_heads = B * (L - 1) * cfg.num_kv_heads
    nbytes = tok_heads * (3 * d * 2 + 2 * (r + s_) * 2) + B * (-(-(L - 1) // P)) * cfg.num_kv_heads * d * 4
    peak, kind = measured_peak()
    gbs = nbytes / (res["tensor_core"]["us"] * 1e-6) / 1e9
    res["roofline"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                       "frac": round(gbs / peak, 4), "algorithmic_bytes": nbytes,
                       "peak_source": f"{kind} copy bandwidth"}
    res["err"] = int(eng.err.item())
    return res


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    from long_context_decode_basiskv_b200.engine import DecodeEngine

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    if args.tp:
        from long_context_decode_basiskv_b200.tensor_parallel import reduce_y, shard_case

        full_wl = chosen_workload(args)
        case = shard_case(make_case(full_wl, dev), rank, world)   # every rank builds the same case
        wl = case.wl
        tokens_per_step = full_wl.batch                           # the ranks share one batch
    else:
        full_wl = wl = replica_workload(chosen_workload(args), rank, world)
        case = make_case(wl, dev)
        tokens_per_step = world * wl.batch                        # independent replicas

    def exchange():
        if args.tp:
            reduce_y(eng.y, world)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        eng = DecodeEngine(case, device=dev, routing=args.routing)
        eng.step()
    torch.cuda.synchronize()
    if int(eng.err.item()) != 0:
        raise RuntimeError(f"device error flag {int(eng.err.item())}")
    nbytes = algorithmic_bytes(eng)

    # the whole step as one CUDA graph, and one graph per phase for the breakdown
    graphs = {}
    for name, fn in [("step", eng.step), ("append_route", eng.append_route), ("decode_attn", eng.decode_attn),
                     ("out_proj", eng.out_proj)]:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        graphs[name] = g
    torch.cuda.synchronize()
    order = ["append_route", "decode_attn", "out_proj"]
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB > L2
    sink = torch.zeros((), dtype=torch.float32, device=dev)

    def run_steps(n, record, phases):
        evs = []
        with torch.cuda.stream(stream):
            for _ in range(n):
                torch.sum(flush, dim=0, out=sink)
                e = [torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)] if record else None
                if record:
                    e[0].record(stream)
                for i, name in enumerate(phases):
                    graphs[name].replay()
                    if name == "step":
                        exchange()
                    if record:
                        e[i + 1].record(stream)
                if record:
                    evs.append(e)
        return evs

    # clocks are sampled over the whole measurement (warm-up, timed steps, per-phase
    # pass, end-to-end pass): the timed region alone is too short for NVML's rate
    clk = ClockSampler(local, period_s=0.0005)
    with clk:
        run_steps(args.warmup, False, ["step"])
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        evs = run_steps(args.steps, True, ["step"])
        torch.cuda.synchronize()
        barrier(world)
        step_ms = [ev[0].elapsed_time(ev[1]) for ev in evs]
        total_ms = max_over_ranks(sum(step_ms), world, dev)
        # per-phase breakdown (separate pass; not part of the headline number)
        run_steps(max(3, args.warmup), False, order)
        evs = run_steps(min(args.steps, 100), True, order)
        torch.cuda.synchronize()
        per = {name: [ev[i].elapsed_time(ev[i + 1]) for ev in evs] for i, name in enumerate(order)}
        ms_per_step = total_ms / args.steps
        value = tokens_per_step * args.steps / (total_ms / 1e3)

        mean = {k: sum(v) / len(v) for k, v in per.items()}
        peak, peak_kind = measured_peak()
        attn_gbs = nbytes["decode_attn"] / (mean["decode_attn"] * 1e-3) / 1e9
        ra_gbs = (nbytes["route"] + nbytes["decode_attn"]) / ((mean["append_route"] + mean["decode_attn"]) * 1e-3) / 1e9
        # the committed counters are for per-head routing (other routings read other pages)
        traffic_rec = profiled_traffic("decode_attn.cu") if args.routing == "head" else None
        if traffic_rec and (traffic_rec.get("workload") != full_wl.name or args.context):
            traffic_rec = None  # the counters were taken on another workload
        roofline = {
            "kernel": "basiskv_decode_attn (one launch: union slice, attention, split merge)",
            "bound": "hbm", "achieved": round(attn_gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(attn_gbs / peak, 4), "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
            "algorithmic_bytes": nbytes["decode_attn"],
            "traffic": traffic_rec["dram_bytes_per_launch"] if traffic_rec else None,
        }

        # end to end through the public API: pinned host inputs -> step -> host output
        e2e = None
        if not args.no_e2e:
            hin = eng.input_buffer().cpu().pin_memory()   # q, k_new, v_new of the step, packed
            hy = torch.empty(eng.y.shape, dtype=eng.y.dtype).pin_memory()
            bi = hin.numel() * hin.element_size()
            bo = hy.numel() * hy.element_size()

            def e2e_steps(n, record):
                out = []
                with torch.cuda.stream(stream):
                    for _ in range(n):
                        torch.sum(flush, dim=0, out=sink)
                        if record:
                            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                            a.record(stream)
                        if args.tp:
                            eng.input_buffer().copy_(hin, non_blocking=True)
                            eng.graph_step()
                            exchange()
                            hy.copy_(eng.y, non_blocking=True)
                        else:
                            eng.graph_step_host(hin, hy)   # inputs in by a copy kernel, step, y stored on the host: one graph
                        if record:
                            b_.record(stream)
                            out.append((a, b_))
                return out

            e2e_steps(max(3, args.warmup), False)
            torch.cuda.synchronize()
            barrier(world)
            pairs = e2e_steps(args.steps, True)
            torch.cuda.synchronize()
            barrier(world)
            e2e_ms = max_over_ranks(sum(a.elapsed_time(b_) for a, b_ in pairs), world, dev)
            e2e = {"value": round(tokens_per_step * args.steps / (e2e_ms / 1e3), 1), "unit": UNIT,
                   "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                   "path": "copy-engine copies of pinned tensors" if args.tp else "basiskv_copy kernel in, out_proj stores y on the host",
                   "ms_per_step": round(e2e_ms / args.steps, 4)}

    prefill = None
    if not args.no_prefill:
        prefill = measure_prefill(eng, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, args.routing, args.oracle_repeats, args.oracle_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "strong" if args.tp else "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic (seeded generator)",
            "config": {"workload": full_wl.name, "batch": full_wl.batch,
                       "context": full_wl.context if not full_wl.ragged else list(full_wl.ragged),
                       "q_heads": full_wl.num_q_heads, "kv_heads": full_wl.num_kv_heads, "head_dim": wl.head_dim,
                       "page_size": wl.page_size, "rank_v": wl.rank_v, "rank_k": wl.rank_k,
                       "top_k": wl.top_k, "hidden": wl.hidden, "routing": args.routing,
                       "parallelism": (f"tp{world}: KV heads sharded, NCCL all-reduce of y per step"
                                       if args.tp else f"replicas x{world}"),
                       "l2": "flushed between steps (read of a 256 MiB buffer)",
                       "timing": "one CUDA graph per step (append || route on forked streams, decode_attn, out_proj), CUDA events around each replay; kernels_us from per-phase graphs in a separate pass; route+attn GB/s counts the append || route phase time"},
            "kernels_us": {k: round(v * 1e3, 2) for k, v in mean.items()},
            "algorithmic_bytes": nbytes,
            "route_attn_gbs": round(ra_gbs, 1),
            "route_attn_frac_of_8tbs": round(ra_gbs / 8000.0, 4),
            "route_attn_frac_of_measured": round(ra_gbs / peak, 4),
            "roofline": roofline,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clk.summary(),
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "prefill": prefill,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, world, rank):
    """The fp64 oracle on the host cores (rank 0 only).  One step = one decode step
    on every host process at once (process i decodes sequence i mod B)."""
    if rank != 0:
        return
    wl = chosen_workload(args)
    case = make_case(wl, "cpu")
    host = OracleHost(case, args.routing)
    try:
        host.run(args.warmup)
        steps, wall, times = host.run(args.steps)
    finally:
        host.close()
    value = steps / wall
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * wall / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded generator)", "impl": "reference",
        "config": {"workload": wl.name, "batch": wl.batch, "routing": args.routing,
                   "sample": f"one step = one decode step on each of {host.workers} host processes"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": host.workers, "kind": "oracle",
                         "sample": host.describe(f"{args.warmup} untimed + {args.steps} timed decode steps "
                                                 f"per process")},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
