"""Benchmark of TwoTower block attention on B200 through the C ABI.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ID] [--only] [--impl native|reference]

One step = one call of the whole hot path (Q pack, context KV stream, QK^T,
online softmax, PV, block-KV fold-in, ragged mask, epilogue, split combine)
over one batch of the named workload.  The headline is the long-context
decode (B=4, Hq=32, Hkv=2, D=128, S=16, L=131072), the largest decode that
fits one GPU; the line also carries one record per other workload (the
L=4096 peaky decode, the ragged B=64 decode and the block-causal N=8192
training form), each timed the same way, unless --only is given.  Inputs are
resident in HBM before timing; each timed step reads a different copy of the
inputs and the copies together exceed twice the L2 size, so no step is
served from L2.  Timing: CUDA events on the launching stream around K
graph-launched steps, max over ranks.

Prints one JSON line (rank 0).  Multi-GPU runs are replicas: every rank runs
the same per-GPU batch on its own GPU (weak scaling, no data-path
collective); the process group only carries the barrier and the max of the
timings.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-attn KV GB/s & TFLOP/s on 1 B200, % of roofline; oracle CPU time"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--only", action="store_true", help="time the named workload alone (no per-workload records)")
    ap.add_argument("--no-backward", action="store_true", help="skip the block-causal backward measurement")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (same per-sequence recipe): small cases for profiler captures")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "tcgen05", "mma_sync"])
    ap.add_argument("--no-graph", action="store_true", help="launch steps directly instead of via CUDA graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-paged", action="store_true", help="skip the paged-cache decode measurement")
    ap.add_argument("--page-size", type=int, default=64, help="rows per page of the paged-cache measurement")
    ap.add_argument("--num-ctas", type=int, default=0, help="work ranges (0: the plan's choice)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(kind: str) -> str:
    files = {"tcgen05": ["attn_tcgen05.cu", "tc_common.cuh"], "tcgen05_pt": ["attn_tcgen05_pt.cu", "tc_common.cuh"],
             "bwd_tc": ["attn_bwd_tc.cu", "attn_bwd.h"], "unmask": ["unmask.cu"],
             "tcgen05_2sm": ["attn_tcgen05_2sm.cu", "tc_common.cuh"], "mma_sync": ["attn_mma_sync.cu"]}[kind]
    h = hashlib.sha256()
    for f in files + ["ptx.cuh", "walker.cuh", "problem.h", "sched.cuh"]:
        h.update(open(os.path.join(ROOT, "two_tower_block_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kind: str, workload: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    want = kernel_source_hash(kind)
    for line in open(p):
        line = line.split("#", 1)[0].split()
        if len(line) == 4 and line[0] == kind and line[1] == want and int(line[2]) == workload:
            return float(line[3])
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:7]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        sm = [r[0] for r in rows]
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if args.impl == "native" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(pg, value, device=None):
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def replica_rate(world, units_per_replica, ms_max):
    """Whole-job rate of `world` replicas that each process `units_per_replica` in a step whose
    slowest rank took `ms_max` milliseconds: units per second summed over all ranks."""
    return world * units_per_replica / (ms_max * 1e-3)


def workload_cost(wid, inp):
    from two_tower_block_b200.workloads import WORKLOADS, causal_cost, decode_cost
    w = WORKLOADS[wid]
    B = int(inp.q.shape[0])   # the inputs' batch (a --batch override changes it)
    if w.kind == "decode":
        return decode_cost(B, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim, inp.ctx_lens)
    return causal_cost(B, w.seq_len, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim)


# --------------------------------------------------------------- oracle arm --
def oracle_sample(wid, inp, seconds):
    """Time the float64 oracle, as it stands, on a bounded sample of the workload.
    Returns (GB/s of algorithmic bytes, description, threads)."""
    from oracle import block_attn, block_causal
    from two_tower_block_b200.workloads import WORKLOADS, bf16_to_f64, causal_cost, decode_cost
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    w = WORKLOADS[wid]
    done_bytes = 0
    units = 0
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < seconds:
        if w.kind == "decode":
            b = n % w.batch
            sl = slice(b, b + 1)
            block_attn(bf16_to_f64(inp.q[sl]), bf16_to_f64(inp.k_ctx[sl]), bf16_to_f64(inp.v_ctx[sl]),
                       bf16_to_f64(inp.k_blk[sl]), bf16_to_f64(inp.v_blk[sl]), inp.ctx_lens[sl])
            done_bytes += decode_cost(1, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                      inp.ctx_lens[sl])["bytes"]
            units += 1
        else:
            nb = w.seq_len // w.block_size
            b = (n * 37) % nb
            sl = slice(0, 1)
            block_causal(bf16_to_f64(inp.q[sl]), bf16_to_f64(inp.k_ctx[sl]), bf16_to_f64(inp.v_ctx[sl]),
                         bf16_to_f64(inp.k_blk[sl]), bf16_to_f64(inp.v_blk[sl]), w.block_size, blocks=[b])
            L = w.block_size * b
            done_bytes += decode_cost(1, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim, [L])["bytes"]
            units += 1
        n += 1
    el = time.perf_counter() - t0
    what = "sequences" if w.kind == "decode" else "blocks of sequence 0"
    return done_bytes / el / 1e9, f"{units} {what} of the workload in {el:.1f} s", threads, el


def run_reference(args):
    # Under torchrun only rank 0 times the oracle; the others exit without work.
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    from two_tower_block_b200.workloads import WORKLOADS, make_workload
    w = WORKLOADS[args.workload]
    inp = make_workload(args.workload)
    per_step = max(1.0, min(8.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(args.workload, inp, per_step / 4)
    vals = []
    t_all = 0.0
    desc = ""
    threads = 1
    for _ in range(args.steps):
        v, desc, threads, el = oracle_sample(args.workload, inp, per_step)
        vals.append(v)
        t_all += el
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * t_all / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": w.describe(),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: {desc}"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- native arm --
def roofline_of(wid, cost, k_ms, kname, peaks, batch_override=0):
    """Roofline record of the dominant (attention) kernel of one workload: algorithmic bytes
    (decode, HBM-bound) or flops (block-causal, tensor-bound) per launch over its average
    event-timed duration."""
    from two_tower_block_b200.workloads import WORKLOADS
    traffic = None if batch_override else recorded_traffic(kname, wid)
    if WORKLOADS[wid].kind == "decode":
        achieved = cost["bytes"] / (k_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "kernel": f"attn_{kname}", "kernel_ms": round(k_ms, 5),
                "peak_source": peaks["source"] + " (hbm_gbs, copy)"}
    ach_t = cost["flops"] / (k_ms * 1e-3) / 1e12
    pk = peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]
    return {"bound": "tensor", "achieved": round(ach_t, 2), "peak": pk, "unit": "TFLOP/s",
            "frac": round(ach_t / pk, 4), "traffic": traffic,
            "kernel": f"attn_{kname}", "kernel_ms": round(k_ms, 5),
            "peak_source": peaks["source"] + " (bf16_tflops_sustained, cuBLAS)"}


class Measured:
    """One workload resident on the device: its plan, rotating input copies and timings."""

    def __init__(self, wid, args, dev, kernel, local):
        import torch
        from two_tower_block_b200 import ops
        from two_tower_block_b200.workloads import WORKLOADS, make_workload
        self.wid, self.w = wid, WORKLOADS[wid]
        self.args_batch = args.batch
        if args.batch:
            import dataclasses
            self.w = dataclasses.replace(self.w, batch=args.batch)
        w = self.w
        self.inp = make_workload(wid, batch=args.batch or None)
        self.cost = workload_cost(wid, self.inp)
        self.l2 = torch.cuda.get_device_properties(dev).L2_cache_size

        def to_dev(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
        self.to_dev = to_dev
        base = [to_dev(self.inp.q), to_dev(self.inp.k_ctx), to_dev(self.inp.v_ctx), to_dev(self.inp.k_blk),
                to_dev(self.inp.v_blk)]
        self.in_bytes = sum(t.numel() * 2 for t in base)
        self.n_copies = max(1, math.ceil(2.0 * self.l2 / self.in_bytes) + 1)
        self.copies = [base] + [[t.clone() for t in base] for _ in range(self.n_copies - 1)]
        if w.kind == "decode":
            self.lens = torch.from_numpy(self.inp.ctx_lens).to(dev)
            self.plan = ops.Plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                 ctx_capacity=w.ctx, kernel=kernel, num_ctas=args.num_ctas, device=local)
            self.out = torch.empty((w.batch, w.block_size, w.num_q_heads, w.head_dim), dtype=torch.float32,
                                   device=dev)
            self.lse = torch.empty((w.batch, w.num_q_heads, w.block_size), dtype=torch.float32, device=dev)
        else:
            self.lens = None
            self.plan = ops.Plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                 seq_len=w.seq_len, kernel=kernel, num_ctas=args.num_ctas, device=local)
            self.out = torch.empty((w.batch, w.seq_len, w.num_q_heads, w.head_dim), dtype=torch.float32,
                                   device=dev)
            self.lse = torch.empty((w.batch, w.num_q_heads, w.seq_len), dtype=torch.float32, device=dev)
        self.info = self.plan.info()
        kname = {1: "tcgen05", 2: "mma_sync"}[self.info.kernel]
        if self.info.kernel == 1 and self.info.variant in (2, 3):   # the selectable forms have their own sources
            kname = {2: "tcgen05_pt", 3: "tcgen05_2sm"}[self.info.variant]
        self.kname = kname

    def step(self, i):
        c = self.copies[i % self.n_copies]
        if self.w.kind == "decode":
            self.plan.block_attn(c[0], c[1], c[2], c[3], c[4], self.lens, out=self.out, lse=self.lse)
        else:
            self.plan.block_attn_block_causal(c[0], c[1], c[2], c[3], c[4], out=self.out, lse=self.lse)

    def time(self, args, pg, dev, before_timed=None):
        """W warm-up steps, then K timed steps (graph replay unless --no-graph) between a barrier and a
        synchronize on both sides; then the same K steps again with the library's per-kernel events."""
        import torch
        stream = torch.cuda.current_stream()
        for i in range(max(3, args.warmup)):
            self.step(i)
        self.plan.check()
        # the K timed steps are captured in one CUDA graph (rotating over the input copies) and
        # replayed once, so the host's launch overhead is not in the timed region
        graph = None
        if not args.no_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for i in range(args.steps):
                    self.step(i)
            graph.replay()
            torch.cuda.synchronize()
        if before_timed:
            before_timed()
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for i in range(args.steps):
                self.step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        ms_total = e0.elapsed_time(e1)
        # per-kernel durations of the same steps, from events the library records on the launching
        # stream; with graphs the profiled steps are captured in a graph too (the event records become
        # graph nodes), so the kernels are timed as the steps run
        self.plan.profile(True)
        if not args.no_graph:
            pgraph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(pgraph):
                for i in range(args.steps):
                    self.step(i)
            pgraph.replay()
            torch.cuda.synchronize()
            del pgraph
        else:
            for i in range(args.steps):
                self.step(i)
        torch.cuda.synchronize()
        n_k, ms_k = self.plan.profile_read(0)
        n_c, ms_c = self.plan.profile_read(1) if self.info.num_ctas > 1 else (0, 0.0)
        self.plan.profile(False)
        self.plan.check()
        self.graphs_used = graph is not None
        del graph
        self.ms_step = max_over_ranks(pg, ms_total, dev) / args.steps
        self.k_ms = ms_k / max(n_k, 1)
        if n_c == 0 and n_k == args.steps:
            # one launch per step (the combine runs in the kernel's tail): the step's own time bounds
            # the kernel's, while the profiled launches also carry the event records' scheduling gaps
            self.k_ms = min(self.k_ms, self.ms_step)
        self.c_ms = ms_c / max(n_c, 1) if n_c else None
        self.launches_per_step = (n_k + n_c) // max(args.steps, 1)

    def record(self, world, peaks):
        value = replica_rate(world, self.cost["bytes"], self.ms_step) / 1e9
        tflops = replica_rate(world, self.cost["flops"], self.ms_step) / 1e12
        return {"workload": self.w.name, "value": round(value, 3), "unit": "GB/s",
                "ms_per_step": round(self.ms_step, 5), "tflops": round(tflops, 2),
                "alg_bytes": int(self.cost["bytes"]), "flops": int(self.cost["flops"]),
                "roofline": roofline_of(self.wid, self.cost, self.k_ms, self.kname, peaks, self.args_batch),
                "combine_kernel_ms": round(self.c_ms, 5) if self.c_ms else None,
                "launches_per_step": self.launches_per_step, "num_ctas": self.info.num_ctas,
                "l2": "inputs rotate over %d copies (%.0f MB) > 2x L2 (%d MB)" % (
                    self.n_copies, self.n_copies * self.in_bytes / 1e6, self.l2 // 2**20)}

    def free(self):
        self.plan.close()
        del self.copies, self.out, self.lse


def measure_backward(m, dev):
    """Block-causal backward at a training workload's shape: device time of its kernel."""
    import torch
    w, plan, c0 = m.w, m.plan, m.copies[0]
    bout = torch.empty((w.batch, w.seq_len, w.num_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    blse = torch.empty((w.batch, w.num_q_heads, w.seq_len), dtype=torch.float32, device=dev)
    plan.block_attn_block_causal(c0[0], c0[1], c0[2], c0[3], c0[4], out=bout, lse=blse)
    dout = torch.empty_like(bout).normal_().to(torch.bfloat16)
    dq = torch.empty_like(bout)
    dkb = torch.empty((w.batch, w.seq_len, w.num_kv_heads, w.head_dim), dtype=torch.float32, device=dev)
    dvb = torch.empty_like(dkb)
    for _ in range(2):
        plan.block_causal_backward(c0[0], c0[1], c0[2], c0[3], c0[4], bout, blse, dout, dq, dkb, dvb)
    torch.cuda.synchronize()
    plan.profile(True)
    n_b = 3
    for _ in range(n_b):
        plan.block_causal_backward(c0[0], c0[1], c0[2], c0[3], c0[4], bout, blse, dout, dq, dkb, dvb)
    torch.cuda.synchronize()
    nb_l, ms_b = plan.profile_read(2)
    plan.profile(False)
    plan.check()
    ms_b /= max(nb_l, 1)
    # recompute S, dP and dQ over every visible key (3 x 2D flops per row and key),
    # dK and dV over the block's own keys (2 x 2D per row and block key)
    rows_keys = m.cost["flops"] / (4 * w.head_dim)
    rows_blk = w.batch * w.num_q_heads * w.seq_len * w.block_size
    bflops = 6 * w.head_dim * rows_keys + 4 * w.head_dim * rows_blk
    pkk = load_peaks()
    pk = pkk["bf16_tflops_sustained"] or pkk["bf16_tflops"]
    del bout, blse, dout, dq, dkb, dvb
    # the tcgen05 backward runs on sm_100 plans with S <= 32 unless TT_BWD_KERNEL=mma_sync
    tc = m.info.kernel == 1 and w.block_size <= 32 and os.environ.get("TT_BWD_KERNEL") != "mma_sync"
    return {"kernel": "attn_bwd_tc" if tc else "attn_bwd (mma.sync)", "ms": round(ms_b, 4),
            "tflops": round(bflops / (ms_b * 1e-3) / 1e12, 2),
            "frac_of_sustained_bf16": round(bflops / (ms_b * 1e-3) / 1e12 / pk, 4), "launches": nb_l,
            "traffic": recorded_traffic("bwd_tc", m.wid) if tc and not m.args_batch else None}


def run_native(args):
    import torch
    world, rank, local, pg = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from two_tower_block_b200 import ops
    kernel = {"auto": ops.KERNEL_AUTO, "tcgen05": ops.KERNEL_TCGEN05, "mma_sync": ops.KERNEL_MMA_SYNC}[args.kernel]
    peaks = load_peaks()

    clocks = ClockSampler(local)
    started = []

    def start_clocks():
        if not started:
            clocks.start()
            time.sleep(0.3)  # let the sampler attach before the first timed region
            started.append(1)

    # the other workloads first, each timed the same way and freed before the next
    extra = []
    extra_ids = [] if args.only else [x for x in (2, 3, 4, 5) if x != args.workload]
    bwd = None
    for wid in extra_ids:
        m = Measured(wid, args, dev, kernel, local)
        m.time(args, pg, dev, before_timed=start_clocks)
        extra.append(m.record(world, peaks))
        if m.w.kind == "causal" and not args.no_backward:
            bwd = measure_backward(m, dev)
            extra[-1]["backward"] = bwd
        m.free()
        del m
        torch.cuda.empty_cache()

    m = Measured(args.workload, args, dev, kernel, local)
    w, inp, cost, plan, info = m.w, m.inp, m.cost, m.plan, m.info
    m.time(args, pg, dev, before_timed=start_clocks)
    ck = clocks.stop()
    stream = torch.cuda.current_stream()
    ms_step = m.ms_step
    out, lse = m.out, m.lse

    # ---- end to end through the host-buffer entry (decode workloads) ----
    e2e = None
    if w.kind == "decode" and not args.no_e2e:
        hplan = ops.Plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, ctx_capacity=w.ctx,
                         kernel=kernel, num_ctas=args.num_ctas, host_io=True, device=local)

        def pinned(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()
        hin = [pinned(inp.q), pinned(inp.k_ctx), pinned(inp.v_ctx), pinned(inp.k_blk), pinned(inp.v_blk),
               torch.from_numpy(inp.ctx_lens).pin_memory()]
        hout = torch.empty(tuple(out.shape), dtype=torch.float32).pin_memory()
        hlse = torch.empty(tuple(lse.shape), dtype=torch.float32).pin_memory()
        for _ in range(2):
            hplan.block_attn_host(*hin, hout, hlse)
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 20))
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(n_e2e):
            hplan.block_attn_host(*hin, hout, hlse)
        a1.record(stream)
        torch.cuda.synchronize()
        hplan.check()
        ms_e2e = max_over_ranks(pg, a0.elapsed_time(a1) / n_e2e, dev)
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = hout.numel() * 4 + hlse.numel() * 4
        e2e = {"value": round(world * cost["bytes"] / (ms_e2e * 1e-3) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms_e2e, 4),
               "steps": n_e2e}
        hplan.close()
        del hin, hout, hlse

    # ---- the same decode over a paged cache: pages of --page-size rows in a shuffled pool ----
    paged = None
    if w.kind == "decode" and not args.no_paged:
        from two_tower_block_b200.workloads import make_paged
        P = args.page_size
        pc = make_paged(inp, P, seed=w.seed, spare_pages=0, fill_bits=0)
        ptab = torch.from_numpy(pc.page_table).to(dev)
        pbase = [m.to_dev(pc.k_pages), m.to_dev(pc.v_pages)]
        del pc
        pcopies = [pbase] + [[t.clone() for t in pbase] for _ in range(m.n_copies - 1)]
        pplan = ops.Plan(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, ctx_capacity=0,
                         kernel=kernel, num_ctas=args.num_ctas, device=local)

        def pstep(i):
            c, pk = m.copies[i % m.n_copies], pcopies[i % m.n_copies]
            pplan.block_attn_paged(c[0], pk[0], pk[1], ptab, c[3], c[4], m.lens, out=out, lse=lse)
        for i in range(max(3, args.warmup)):
            pstep(i)
        pplan.check()
        pgraph = None
        if not args.no_graph:
            pgraph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(pgraph):
                for i in range(args.steps):
                    pstep(i)
            pgraph.replay()
        torch.cuda.synchronize()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        if pgraph is not None:
            pgraph.replay()
        else:
            for i in range(args.steps):
                pstep(i)
        p1.record(stream)
        torch.cuda.synchronize()
        pplan.profile(True)   # profiled the same way as the contiguous steps (in a graph when graphs are on)
        if pgraph is not None:
            ppgraph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(ppgraph):
                for i in range(args.steps):
                    pstep(i)
            ppgraph.replay()
            torch.cuda.synchronize()
            del ppgraph
        else:
            for i in range(args.steps):
                pstep(i)
        torch.cuda.synchronize()
        n_pk, ms_pk = pplan.profile_read(0)
        n_pc, _ = pplan.profile_read(1) if info.num_ctas > 1 else (0, 0.0)
        pplan.profile(False)
        pplan.check()
        ms_pstep = max_over_ranks(pg, p0.elapsed_time(p1) / args.steps, dev)
        pk_ms = ms_pk / max(n_pk, 1)
        tbytes = int(sum(-(-int(L) // P) for L in inp.ctx_lens)) * 4 * w.num_kv_heads   # table entries read
        pbytes = cost["bytes"] + tbytes
        paged = {"page_size": P, "pool_pages": int(pbase[0].shape[0]), "ms_per_step": round(ms_pstep, 5),
                 "value": round(replica_rate(world, pbytes, ms_pstep) / 1e9, 3), "unit": "GB/s",
                 "kernel_ms": round(pk_ms, 5), "kernel_gbs": round(pbytes / (pk_ms * 1e-3) / 1e9, 2),
                 "kernel_time_vs_contiguous": round(pk_ms / m.k_ms, 4),
                 "launches_per_step": (n_pk + n_pc) // max(args.steps, 1)}
        del pgraph, pcopies, pbase
        pplan.close()

    if w.kind == "causal" and not args.no_backward:
        bwd = measure_backward(m, dev)

    # ---- committed-block cache update at this workload's shape (decode only) ----
    kv_app = None
    if w.kind == "decode":
        B_, S_, H_, D_ = w.batch, w.block_size, w.num_kv_heads, w.head_dim
        aplan = ops.Plan(B_, w.num_q_heads, H_, D_, S_, ctx_capacity=2 * S_, device=local)
        k_new = torch.empty((B_, S_, H_, D_), dtype=torch.bfloat16, device=dev).normal_()
        v_new = torch.empty_like(k_new).normal_()
        kc = torch.zeros((B_, H_, 2 * S_, D_), dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        zl = torch.zeros((B_,), dtype=torch.int32, device=dev)
        for _ in range(3):
            aplan.kv_append(k_new, v_new, kc, vc, zl, advance=False)
        # device time: n_app calls replay from one graph, so the host's call overhead is not timed
        n_app = 50
        ag = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ag):
            for _ in range(n_app):
                aplan.kv_append(k_new, v_new, kc, vc, zl, advance=False)
        ag.replay()
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        ag.replay()
        b1.record(stream)
        torch.cuda.synchronize()
        aplan.check()
        us = b0.elapsed_time(b1) * 1e3 / n_app
        nbytes = 4 * B_ * S_ * H_ * D_ * 2       # K and V: read the new rows, write them into the cache
        kv_app = {"us_per_call": round(us, 3), "bytes": nbytes, "gbs": round(nbytes / (us * 1e-6) / 1e9, 2),
                  "launches": n_app}
        del ag
        aplan.close()

    # ---- confidence-unmasking step over a 131072-entry vocabulary at the block shape ----
    unmask = None
    if w.kind == "decode":
        Vv = 131072
        UB = 8   # eight sequences of S block positions (the decode batch of the L = 4096 workload)
        ubytes = UB * w.block_size * Vv * 2
        # the logits rotate over copies that together exceed twice the L2, like the attention inputs
        n_lg = max(1, math.ceil(2.0 * m.l2 / ubytes) + 1)
        lgs = [torch.empty((UB, w.block_size, Vv), dtype=torch.bfloat16, device=dev).normal_() for _ in range(n_lg)]
        tk = torch.full((UB, w.block_size), -1, dtype=torch.int32, device=dev)
        mk = torch.ones((UB, w.block_size), dtype=torch.uint8, device=dev)
        # standard-normal logits never reach 0.8 and min_one is off: every call scans every row
        for i in range(3):
            ops.confidence_unmask(lgs[i % n_lg], tk, mk, gamma=0.8, min_one=False)
        n_u = 54
        ug = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ug):
            for i in range(n_u):
                ops.confidence_unmask(lgs[i % n_lg], tk, mk, gamma=0.8, min_one=False)
        ug.replay()
        torch.cuda.synchronize()
        u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        u0.record(stream)
        ug.replay()
        u1.record(stream)
        torch.cuda.synchronize()
        us = u0.elapsed_time(u1) * 1e3 / n_u
        unmask = {"rows": UB * w.block_size, "vocab": Vv, "us_per_call": round(us, 3), "bytes": ubytes,
                  "gbs": round(ubytes / (us * 1e-6) / 1e9, 2),
                  "frac_hbm": round(ubytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4), "launches_per_call": 2,
                  "traffic": recorded_traffic("unmask", 0),
                  "l2": "logits rotate over %d copies (%.0f MB)" % (n_lg, n_lg * ubytes / 1e6)}
        del ug, lgs

    # ---- oracle CPU baseline (rank 0, N = 1 only) ----
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, desc, threads, el = oracle_sample(args.workload, inp, args.cpu_seconds)
        cpu = {"value": round(v, 5), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": desc + f"; host has {os.cpu_count()} logical CPUs"}

    if rank != 0:
        m.free()
        return 0
    rec = m.record(world, peaks)
    line = {
        "metric": METRIC, "value": rec["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(w.describe(), parallelism=f"replicas{world}", l2=rec["l2"],
                       timing=("the K steps in one CUDA graph, replayed once" if not args.no_graph
                               else "direct launches")),
        "tflops": rec["tflops"],
        "tensor_frac": round(rec["tflops"] / peaks["bf16_tflops"], 4),
        "roofline": rec["roofline"],
        "combine_kernel_ms": rec["combine_kernel_ms"],
        "gpu_launches": m.launches_per_step * args.steps,
        "kernel": m.kname,
        "num_ctas": info.num_ctas,
        "e2e": e2e,
        "workloads": extra,
        "kv_append": kv_app,
        "paged": paged,
        "backward": bwd,
        "unmask": unmask,
        "cpu_baseline": cpu,
        "clocks": ck,
    }
    m.free()
    print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
