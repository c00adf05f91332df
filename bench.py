#!/usr/bin/env python
"""Benchmark of the 2:4 sparse GEMM hot path in the decode regime.

Workload (one step): for M in {1, 8, 32, 128} and (N, K) in {(5120,5120),
(25600,5120), (5120,25600), (10240,5120)}: cast the bf16 activations X [M x K]
to E4M3 per token, then Y [M x N] = X * W^T with W pruned 2:4 along K and
stored as E4M3 values + metadata with one fp32 scale per output channel
(16 independent GEMMs).  The 16 casts run as one grouped launch and the 16
GEMMs as three grouped launches, one per token-count class (M in {1, 8}, 32,
128): 4 launches per step.  W ~ N(0, 0.02^2), X ~ N(0, 1), seeded.
Each of the 16 GEMMs reads its own copy of W (852 MB of distinct weights per
step, far above the 126 MB L2), so no weight is served from L2.

The step is captured once in a CUDA graph and replayed; timing is CUDA
events on the replay stream, max over ranks.  Under torchrun every rank runs
an independent replica (the path has no exchange step).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "2:4 sparse GEMM TFLOPS & GB/s, % of roofline, speedup vs in-build dense"
WORKLOAD = "decode-regime linear layers, e4m3 2:4 weights (per-channel scale), per-token e4m3 activations"
L2_NOTE = ("inputs larger than L2: every GEMM of a step reads its own weight copy "
           "(852 MB of distinct compressed weights per step vs 126 MB L2); no flush")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="sp24", choices=["sp24", "reference"])
    p.add_argument("--manifest", default="", help="write the tactic audit manifest here")
    p.add_argument("--cpu-rows", type=int, default=256,
                   help="weight rows per GEMM in the single-thread CPU-baseline sample")
    p.add_argument("--no-configs", action="store_true",
                   help="leave the other workloads' rows (prefill, activations, hybrid) out of the line")
    p.add_argument("--config", default="decode",
                   choices=["decode", "tiny", "prefill", "activation", "hybrid", "prune", "nvfp4"],
                   help="decode (default): the headline step line.  The others time the other "
                        "workloads of the hot path, one JSON line each, eager calls with an L2 "
                        "flush before every timed call")
    p.add_argument("--case", default="",
                   help="M,N,K[,bf16|e4m3[,sparse|dense|hybrid]]: time one GEMM of the decode/prefill "
                        "family in isolation (used for profiler captures) instead of the step; hybrid = "
                        "e4m3 2:4 weights with 25%% dense 128 x 128 tiles; "
                        "group:M1,M2,...: one grouped launch of the decode GEMMs for those M")
    return p.parse_args()


def gemm_list():
    from semi_structured_sparse_02_b200 import inputs
    return [(M, N, K) for M in inputs.DECODE_M for (N, K) in inputs.DECODE_NK]


def gemm_bytes(M, N, K):
    """Algorithmic HBM bytes of one sparse e4m3 GEMM: W values (K/2 bytes per
    row) + metadata (K/8) + W scales, X codes + scales, Y (bf16)."""
    return N * K // 2 + N * K // 8 + 4 * N + M * K + 4 * M + 2 * M * N


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_step_traffic.md")
GEMM_SOURCE = os.path.join(ROOT, "semi_structured_sparse_02_b200", "csrc", "gemm.cuh")


def recorded_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current GEMM source (else None)."""
    import hashlib
    import re
    if not os.path.exists(TRAFFIC_FILE):
        return None
    txt = open(TRAFFIC_FILE).read()
    sha = re.search(r"gemm_source_sha256:\s*([0-9a-f]{64})", txt)
    val = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", txt)
    if not sha or not val:
        return None
    if hashlib.sha256(open(GEMM_SOURCE, "rb").read()).hexdigest() != sha.group(1):
        return None
    return int(val.group(1))


def quant_bytes(M, K):
    return 2 * M * K + M * K + 4 * M


def dense_gemm_bytes(M, N, K):
    return N * K + 4 * N + M * K + 4 * M + 2 * M * N


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock and throttle-reason samples (every 100 ms) with their
    timestamps, so that each timed window gets the samples taken inside it."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        import torch
        props = torch.cuda.get_device_properties(device_index)
        self.bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        self.proc = None
        self.lines = []
        self.samples = []  # (epoch seconds, sm MHz, max MHz, set of active reasons)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.proc = None
        self.lines = [ln for ln in out.splitlines() if ln.strip()]
        self.samples = []
        import datetime
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = float("nan")
            active = {n for n, v in zip(self.REASONS, f[4:8]) if v.lower() == "active"}
            self.samples.append((ts, sm, mx, active))

    def summary(self, t0=None, t1=None):
        """Median SM clock, max clock and the reasons seen, over the samples
        taken between wall-clock times t0 and t1 (all samples by default)."""
        sel = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not sel and self.samples and all(x[0] != x[0] for x in self.samples):
            sel = self.samples  # no parseable timestamps: the whole record
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for x in sel:
            reasons |= x[3]
        return {"sm_mhz": statistics.median(x[1] for x in sel), "sm_max_mhz": max(x[2] for x in sel),
                "reasons": sorted(reasons), "samples": len(sel)}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def run_product(args, rank, world, local_rank):
    import torch

    from semi_structured_sparse_02_b200 import inputs, manifest, replicas, sp24

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    sp24.lib()  # raises if the CUDA library is missing
    gemms = gemm_list()
    shapes = sorted(set((N, K) for _, N, K in gemms))

    # weights: prune + compress once per shape on the GPU, then one copy per GEMM
    base = {}
    for (N, K) in shapes:
        Wb = inputs.normal_bf16((N, K), 0.02, seed=N + K)
        W = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).to(dev)
        vals = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
        meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
        wsc = torch.empty(N, dtype=torch.float32, device=dev)
        sp24.prune_compress(W, sp24.E4M3, vals, meta, row_scales=wsc)
        dq = torch.empty(N, K, dtype=torch.uint8, device=dev)
        dsc = torch.empty(N, dtype=torch.float32, device=dev)
        sp24.quantize_e4m3_rows(W, dq, dsc)
        base[(N, K)] = (vals, meta, wsc, dq, dsc)
        del W
    torch.cuda.synchronize()

    # activations and outputs live in single staging buffers (one copy each way for e2e)
    x_elems = sum(M * K for M, _, K in gemms)
    y_elems = sum(M * N for M, N, _ in gemms)
    X_all = torch.empty(x_elems, dtype=torch.bfloat16, device=dev)
    Y_all = torch.empty(y_elems, dtype=torch.bfloat16, device=dev)
    Yd_all = torch.empty(y_elems, dtype=torch.bfloat16, device=dev)
    inst = []
    xo = yo = 0
    for i, (M, N, K) in enumerate(gemms):
        X = X_all[xo:xo + M * K].view(M, K)
        X.copy_(torch.from_numpy(inputs.normal_bf16((M, K), 1.0, seed=1000 + i).view(np.int16))
                .view(torch.bfloat16))
        Y = Y_all[yo:yo + M * N].view(M, N)
        Yd = Yd_all[yo:yo + M * N].view(M, N)
        xo += M * K
        yo += M * N
        vals, meta, wsc, dq, dsc = (t.clone() for t in base[(N, K)])  # distinct copy per GEMM
        xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
        xs = torch.empty(M, dtype=torch.float32, device=dev)
        # the weights are static: the GEMM may stream them during the upstream kernel
        a_sp = sp24.gemm_args(xq, vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs, w_scales=wsc,
                              flags=sp24.GEMM_W_STATIC)
        n = sp24.gemm_workspace_bytes(a_sp)
        if n:
            sp24.set_workspace(a_sp, torch.zeros(n, dtype=torch.uint8, device=dev))
        a_dn = sp24.gemm_args(xq, dq, Yd, K, sp24.DENSE, x_scales=xs, w_scales=dsc,
                              flags=sp24.GEMM_W_STATIC)
        n = sp24.gemm_workspace_bytes(a_dn)
        if n:
            sp24.set_workspace(a_dn, torch.zeros(n, dtype=torch.uint8, device=dev))
        inst.append(dict(M=M, N=N, K=K, X=X, xq=xq, xs=xs, a_sp=a_sp, a_dn=a_dn, W=(vals, meta, wsc)))
    del base
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    # the per-token e4m3 casts of the 16 independent activation matrices run
    # as one grouped launch; then the 16 GEMMs run as one grouped launch per
    # tactic (each problem multiplies its own token-tile width inside the
    # widest one).  Launches are chained by programmatic dependent launch, each
    # streaming its weights while the previous kernel drains.
    quant_all = sp24.QuantGroup([(it["X"], it["xq"], it["xs"]) for it in inst])

    def make_groups(pick, items=None, by_class=False):
        """Grouped launches for the tactic pick(it) of every GEMM, one per
        tactic (or, with by_class, one per tactic and token-count class).  The
        GEMMs are independent and all their inputs come from the cast before
        the first group, so every group after the first is marked as following
        an independent GEMM launch: its CTAs start as SMs free up instead of
        waiting for the previous group to finish."""
        by = {}
        for it in (inst if items is None else items):
            t = pick(it)
            a = it["a_sp"] if t == "sparse" else it["a_dn"]
            by.setdefault((t, sp24.m_class(it["M"]) if by_class else 0), []).append(a)
        return [sp24.GemmGroup(v, after_independent=i > 0) for i, (_, v) in enumerate(sorted(by.items()))]

    groups = {"sparse": make_groups(lambda it: "sparse"), "dense": make_groups(lambda it: "dense")}
    # the same 16 GEMMs as three launches, one per token-count class
    # (M in {1, 8}, 32, 128), each with its own token-tile width, for comparison
    groups["sparse_by_class"] = make_groups(lambda it: "sparse", by_class=True)
    groups["dense_by_class"] = make_groups(lambda it: "dense", by_class=True)

    def step(kind):
        quant_all()
        if kind == "ungrouped":
            for it in inst:
                sp24.gemm(it["a_sp"])
            return
        for grp in groups[kind]:
            grp()

    def gemm_only():
        for grp in groups["sparse"]:
            grp()

    # tactic selection per GEMM (untimed), on the benchmark stream
    with torch.cuda.stream(stream):
        step("sparse")  # quantized X in place for the selector
        records = {}
        for it in inst:
            r = sp24.select_tactic(it["a_sp"], it["a_dn"], warmup=3, iters=15, stream=stream)
            it["tactic"] = r["selected"]
            records["M%d_N%d_K%d" % (it["M"], it["N"], it["K"])] = r
    man = manifest.build_manifest(records, revision="synthetic-seeded")
    if args.manifest and rank == 0:
        with open(args.manifest, "w") as f:
            f.write(manifest.dumps(man))
    groups["selected"] = make_groups(lambda it: it["tactic"])

    # eager warm-up (sets kernel attributes), then capture the graphs
    kinds = ("sparse", "dense", "selected", "ungrouped", "sparse_by_class", "dense_by_class", "gemm_only")
    with torch.cuda.stream(stream):
        for kind in kinds[:-1]:
            step(kind)
        gemm_only()
    torch.cuda.synchronize()
    graphs = {}
    launches = {}
    for kind in kinds:
        g = torch.cuda.CUDAGraph()
        c0 = sp24.launch_count()
        with torch.cuda.graph(g, stream=stream):
            if kind == "gemm_only":
                gemm_only()
            else:
                step(kind)
        launches[kind] = sp24.launch_count() - c0
        graphs[kind] = g
    torch.cuda.synchronize()

    barrier = replicas.barrier

    def time_graph(g, steps, warmup, nvtx=None):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            if nvtx:
                torch.cuda.nvtx.range_push(nvtx)
            e0.record(stream)
            for _ in range(steps):
                g.replay()
            e1.record(stream)
            if nvtx:
                torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        barrier()
        return replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)

    K_steps, W_warm = args.steps, args.warmup
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    t_wall0 = time.perf_counter()
    ms_sparse = time_graph(graphs["sparse"], K_steps, W_warm, nvtx="sp24_timed_step")
    t_wall = time.perf_counter() - t_wall0
    # keep the GPU under the same load long enough for the clock record
    extra = 0
    if t_wall < 1.5:
        n_more = int(max(1, (1.5 - t_wall) / max(ms_sparse / K_steps / 1e3, 1e-6)))
        for _ in range(n_more):
            graphs["sparse"].replay()
        torch.cuda.synchronize()
        extra = n_more
    sampler.stop()
    clocks = sampler.summary()
    clocks["note"] = ("sampled over the timed replays" if extra == 0 else
                      "sampled over the timed replays plus %d more replays of the same step" % extra)

    # the GEMM launch alone (the roofline's kernel), right after the step under
    # the same load, as the median of three timed runs
    ms_gemm = float(np.median([time_graph(graphs["gemm_only"], K_steps, W_warm) for _ in range(3)]))
    ms_dense = time_graph(graphs["dense"], K_steps, W_warm)
    ms_sel = time_graph(graphs["selected"], K_steps, W_warm)
    ms_ungrouped = time_graph(graphs["ungrouped"], K_steps, W_warm)
    ms_cls = time_graph(graphs["sparse_by_class"], K_steps, W_warm)
    ms_cls_dense = time_graph(graphs["dense_by_class"], K_steps, W_warm)

    # End to end through the public API: every step copies its activations in
    # from pinned host memory and its outputs back out, eager calls.  The
    # steps are pipelined over two device buffer sets (activations, casts,
    # outputs; the weights are shared) on three streams, so that step i's
    # input copy, step i-1's compute and step i-2's output copy overlap.
    X_all1 = torch.empty_like(X_all)
    Y_all1 = torch.empty_like(Y_all)
    inst1 = []
    xo = yo = 0
    for it in inst:
        M, N, K = it["M"], it["N"], it["K"]
        X1 = X_all1[xo:xo + M * K].view(M, K)
        Y1 = Y_all1[yo:yo + M * N].view(M, N)
        xo += M * K
        yo += M * N
        xq1 = torch.empty(M, K, dtype=torch.uint8, device=dev)
        xs1 = torch.empty(M, dtype=torch.float32, device=dev)
        vals, meta, wsc = it["W"]
        inst1.append(dict(M=M, X=X1, xq=xq1, xs=xs1,
                          a_sp=sp24.gemm_args(xq1, vals, Y1, K, sp24.SPARSE, W_meta=meta, x_scales=xs1,
                                              w_scales=wsc, flags=sp24.GEMM_W_STATIC)))
    bufsets = [(X_all, Y_all, quant_all, groups["sparse"]),
               (X_all1, Y_all1, sp24.QuantGroup([(it["X"], it["xq"], it["xs"]) for it in inst1]),
                make_groups(lambda it: "sparse", inst1))]
    X_host = torch.empty(x_elems, dtype=torch.bfloat16, pin_memory=True)
    X_host.copy_(X_all.cpu())
    Y_host = [torch.empty(y_elems, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps_run(n):
        for i in range(n):
            b = i & 1
            Xd, Yd_, quant_b, groups_b = bufsets[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[b])   # step i-2 has consumed this input buffer
                Xd.copy_(X_host, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # step i-2's outputs have been copied out
                quant_b()
                for grp in groups_b:
                    grp()
                ev_cmp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b])
                Y_host[b].copy_(Yd_, non_blocking=True)
                ev_out[b].record(s_out)
        return (n - 1) & 1

    e2e_steps = max(3, min(K_steps, 50))
    e2e_steps_run(4)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    last = e2e_steps_run(e2e_steps)
    s_in.wait_event(ev_out[last])  # the last output copy (copies are in order on their stream)
    e1.record(s_in)
    torch.cuda.synchronize()
    ms_e2e = replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)
    # the same loop serialized on one stream (no overlap), for context
    e0s = torch.cuda.Event(enable_timing=True)
    e1s = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0s.record(stream)
        for _ in range(e2e_steps):
            X_all.copy_(X_host, non_blocking=True)
            step("sparse")
            Y_host[0].copy_(Y_all, non_blocking=True)
        e1s.record(stream)
    torch.cuda.synchronize()
    ms_e2e_serial = replicas.max_over_ranks(e0s.elapsed_time(e1s), device=dev)

    # accounting
    step_bytes = sum(gemm_bytes(M, N, K) + quant_bytes(M, K) for M, N, K in gemms)
    gemm_bytes_total = sum(gemm_bytes(M, N, K) for M, N, K in gemms)
    step_flops = sum(2.0 * M * N * K for M, N, K in gemms)
    t_step = ms_sparse / K_steps / 1e3
    value = replicas.aggregate_rate(step_bytes, t_step, world) / 1e9
    n_gemm_launches = launches["gemm_only"]
    t_gemm_launch = ms_gemm / K_steps / 1e3 / n_gemm_launches
    bytes_per_launch = gemm_bytes_total / n_gemm_launches
    peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(peaks_path):
        peaks = json.load(open(peaks_path))
        hbm_peak, peak_src = float(peaks["hbm_gbs"]), "measured"
    else:
        hbm_peak, peak_src = 6650.0, "fallback"
    achieved = bytes_per_launch / t_gemm_launch / 1e9
    e2e_value = replicas.aggregate_rate(step_bytes, ms_e2e / e2e_steps / 1e3, world) / 1e9
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": W_warm,
        "ms_per_step": round(ms_sparse / K_steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic (seeded numpy normal draws rounded to bf16)",
        "config": bench_config(world),
        "timing": "CUDA graph of one step replayed K times; CUDA events on the replay stream",
        "step": ("one grouped per-token e4m3 cast of the 16 activation matrices, then the 16 "
                 "GEMMs as %d grouped launch (token tiles of 16, 32 and 128 rows in one launch)"
                 % len(groups["sparse"])),
        "tflops": round(world * step_flops / t_step / 1e12, 3),
        "speedup_vs_dense": round(ms_dense / ms_sparse, 4),
        "ms_per_step_dense": round(ms_dense / K_steps, 5),
        "ms_per_step_selected": round(ms_sel / K_steps, 5),
        "ms_per_step_ungrouped": round(ms_ungrouped / K_steps, 5),
        "ms_per_step_by_token_class": round(ms_cls / K_steps, 5),
        "ms_per_step_dense_by_token_class": round(ms_cls_dense / K_steps, 5),
        "tactics": man["metrics"],
        "roofline": {
            "kernel": "k_gemm sparse e4m3 (tcgen05.mma.sp), one grouped launch of the 16 GEMMs",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": hbm_peak,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "traffic": recorded_traffic(),
            "bytes_per_launch": int(bytes_per_launch),
            "us_per_launch": round(t_gemm_launch * 1e6, 3),
        },
        "clocks": clocks,
        "e2e": {
            "value": round(e2e_value, 2),
            "unit": "GB/s",
            "h2d_bytes_per_step": x_elems * 2,
            "d2h_bytes_per_step": y_elems * 2,
            "ms_per_step": round(ms_e2e / e2e_steps, 5),
            "ms_per_step_serialized": round(ms_e2e_serial / e2e_steps, 5),
            "how": "eager public-API calls (one sp24_quantize_e4m3_rows_grouped + %d "
                   "sp24_gemm_grouped) with one pinned H2D copy of X and one D2H copy of Y per step, "
                   "pipelined over two device buffer sets on three streams (copy in / compute / copy out); "
                   "CUDA events, the last output copy included" % len(groups["sparse"]),
        },
        "gpu_launches": launches["sparse"] * K_steps,
    }
    if world == 1 and not args.no_configs:
        # the other workloads of the hot path, each with its own clock record
        out["configs"] = run_configs_compact(dev)
    if rank == 0:
        out["cpu_baseline"] = cpu_baseline(args.cpu_rows)
    return out


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def _oracle_prep(M, N, K, rows, seed):
    """Untimed preparation of one decode GEMM's sample for the oracle: `rows`
    weight rows pruned and cast to E4M3 (offline work), their dequantized
    kept values, and the bf16 activations."""
    from oracle import oracle as orc
    from semi_structured_sparse_02_b200 import inputs
    R = min(rows, N)
    Wb = inputs.normal_bf16((R, K), 0.02, seed=seed)
    vq, canon, wsc, _ = orc.prune_compress_e4m3(Wb)
    wv = orc.e4m3_decode(vq) * wsc.astype(np.float64)[:, None]
    Xb = inputs.normal_bf16((M, K), 1.0, seed=seed + 1)
    return R, wv, canon, Xb


def _oracle_call(Xb, wv, canon):
    """The oracle's per-call path: per-token E4M3 quantization of X,
    dequantization, fp64 sparse GEMM over the sample's weight rows."""
    from oracle import oracle as orc
    q, s = orc.quantize_rows_e4m3(Xb)
    Xh = orc.e4m3_decode(q) * s.astype(np.float64)[:, None]
    orc.gemm_sparse_f64(Xh, wv, canon)


def oracle_gemm_sample(M, N, K, rows, seed):
    """Seconds of the oracle's per-call path for one decode GEMM on `rows`
    weight rows (one thread), and the rows used."""
    R, wv, canon, Xb = _oracle_prep(M, N, K, rows, seed)
    t0 = time.perf_counter()
    _oracle_call(Xb, wv, canon)
    return time.perf_counter() - t0, R


def _cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_baseline(rows):
    """The C oracle on the host cores, on a bounded sample of the step: every
    decode GEMM on a slice of its weight rows, timed (a) on one thread and
    (b) on all the cores this process may use (one thread per core, each on
    its own 'rows'-row slice; the C calls release the interpreter lock).  The
    sampled time is scaled to the full N rows of each GEMM."""
    from concurrent.futures import ThreadPoolExecutor
    gemms = gemm_list()
    threads = _cpu_threads()
    t1 = t_all = 0.0
    b = 0
    for i, (M, N, K) in enumerate(gemms):
        dt, R = oracle_gemm_sample(M, N, K, rows, seed=7000 + i)
        t1 += dt * N / R
        b += gemm_bytes(M, N, K) + quant_bytes(M, K)
    # all cores: `threads` slices of `rows` rows per GEMM (capped at N rows)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for i, (M, N, K) in enumerate(gemms):
            n_sl = max(1, min(threads, N // rows))
            preps = list(ex.map(lambda j: _oracle_prep(M, N, K, rows, seed=7100 + 64 * i + j), range(n_sl)))
            t0 = time.perf_counter()
            list(ex.map(lambda pr: _oracle_call(pr[3], pr[1], pr[2]), preps))
            dt = time.perf_counter() - t0
            t_all += dt * N / sum(pr[0] for pr in preps)
    return {"value": round(b / t_all / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "single_thread_value": round(b / t1 / 1e9, 4), "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
            "sample": "all 16 decode GEMMs; one thread: %d weight rows each; all cores: %d threads, each on its own "
                      "%d-row slice (at most N rows per GEMM); time scaled by N / rows sampled; C oracle, fp64"
                      % (rows, threads, rows)}


def bench_config(world):
    """The 'config' object of the decode line (both arms)."""
    from semi_structured_sparse_02_b200 import inputs
    gemms = gemm_list()
    return {
        "workload": WORKLOAD,
        "gemms_per_step": len(gemms),
        "M": sorted(set(M for M, _, _ in gemms)),
        "NK": [list(s) for s in sorted(set((N, K) for _, N, K in gemms))],
        "parallelism": "replicas" if world > 1 else "single-gpu",
        "l2": L2_NOTE,
    }


def run_reference(args, world):
    """The reference arm: the CPU oracle, one thread, as it stands.  One step =
    one of the 16 decode GEMMs in turn on a 64-row slice of its weights; the
    line reports the measured time of those sampled steps and the throughput
    of the sampled work, with the full-size extrapolation labelled apart."""
    gemms = gemm_list()
    rows = 64
    for i in range(args.warmup):
        M, N, K = gemms[i % len(gemms)]
        oracle_gemm_sample(M, N, K, rows, seed=9000 + i)
    t = t_full = 0.0
    b = 0
    for i in range(args.steps):
        M, N, K = gemms[i % len(gemms)]
        dt, R = oracle_gemm_sample(M, N, K, rows, seed=9100 + i)
        t += dt
        t_full += dt * N / R
        b += gemm_bytes(M, R, K) + quant_bytes(M, K)
    value = b / t / 1e9
    cfg = bench_config(world)
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t / args.steps * 1e3, 3),
        "ms_per_full_gemm_extrapolated": round(t_full / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded numpy normal draws rounded to bf16)",
        "config": cfg,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "cpu_model": _cpu_model(),
                         "sample": "one step = one decode GEMM (the 16 in turn) on a %d-row slice of its weights; "
                                   "value = algorithmic bytes of the sampled work / its measured time" % rows},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_group_case(args):
    """One grouped launch of the decode GEMMs for the token counts listed after
    "group:" (e.g. group:1,8), e4m3 sparse weights marked static; eager calls,
    CUDA-event timing (for profiler captures)."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    dev = torch.device("cuda", 0)
    Ms = [int(v) for v in args.case.split(":", 1)[1].split(",")]
    keep, argl = [], []
    for M in Ms:
        for i, (N, K) in enumerate(inputs.DECODE_NK):
            W = torch.from_numpy(inputs.normal_bf16((N, K), 0.02, seed=N + K).view(np.int16)).view(
                torch.bfloat16).to(dev)
            X = torch.from_numpy(inputs.normal_bf16((M, K), 1.0, seed=M + i).view(np.int16)).view(
                torch.bfloat16).to(dev)
            vals = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
            meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
            wsc = torch.empty(N, dtype=torch.float32, device=dev)
            sp24.prune_compress(W, sp24.E4M3, vals, meta, row_scales=wsc)
            xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
            xs = torch.empty(M, dtype=torch.float32, device=dev)
            sp24.quantize_e4m3_rows(X, xq, xs)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            argl.append(sp24.gemm_args(xq, vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs, w_scales=wsc,
                                       flags=sp24.GEMM_W_STATIC))
            keep.append((W, X))
            del W
    del keep
    grp = sp24.GemmGroup(argl)
    t, _, _ = Timer(dev, args.steps, args.warmup, 0.0).calls(lambda: grp())
    byts = sum(gemm_bytes(a.M, a.N, a.K) for a in argl)
    print(json.dumps({"case": args.case, "gemms": len(argl), "us_median": round(t, 3),
                      "GBps": round(byts / t / 1e3, 1), "bytes": byts,
                      "workspace_bytes": grp.ws_bytes}), flush=True)


def run_other_case(args):
    """prune:N,K,bf16|e4m3 -- the weight prune / compress of N x K;
    act:M,N,K,bf16|e4m3|ingemm -- the online-activation path (prune of X every
    call, then the sparse GEMM; ingemm: the prune inside the GEMM kernel);
    nv:M,N,K,sparse|dense -- the NVFP4 GEMM (pairwise
    4:8 or dense), X cast to NVFP4 once; nvstep:sparse|dense -- the NVFP4
    decode step's 16 GEMMs as one grouped launch.  Eager calls, CUDA-event
    timing, L2 flushed before each call (for profiler captures)."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    dev = torch.device("cuda", 0)
    kind, rest = args.case.split(":", 1)
    f = rest.split(",")
    T = Timer(dev, args.steps, args.warmup, 0.0)
    if kind == "prune":
        N, K, e4 = int(f[0]), int(f[1]), (f[2] if len(f) > 2 else "bf16") == "e4m3"
        W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=N + K), dev)
        vals = torch.empty(N, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device=dev)
        meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
        sc = torch.empty(N, dtype=torch.float32, device=dev) if e4 else None
        t, _, _ = T.calls(lambda: sp24.prune_compress(W, sp24.E4M3 if e4 else sp24.BF16, vals, meta, row_scales=sc))
        byts = 2 * N * K + N * K * (1 if e4 else 2) // 2 + N * K // 8
        print(json.dumps({"case": args.case, "us_median": round(t, 3), "GBps": round(byts / t / 1e3, 1)}), flush=True)
    elif kind == "act":
        M, N, K, e4 = int(f[0]), int(f[1]), int(f[2]), (f[3] if len(f) > 3 else "bf16") == "e4m3"
        X = _bf16_dev(inputs.student_t_bf16((M, K), 3.0, seed=4), dev)
        W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=4), dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        if e4:
            Wq = torch.empty(N, K, dtype=torch.uint8, device=dev)
            wsc = torch.empty(N, dtype=torch.float32, device=dev)
            sp24.quantize_e4m3_rows(W, Wq, wsc)
            ws = torch.empty(sp24.activations_e4m3_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
            fn = lambda: sp24.prune_compress_activations_fused_e4m3(X, Wq, wsc, Y, workspace=ws)  # noqa: E731
        elif len(f) > 3 and f[3] == "ingemm":
            fn = lambda: sp24.prune_activations_in_gemm(X, W, Y)  # noqa: E731
        else:
            ws = torch.empty(sp24.activations_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
            fn = lambda: sp24.prune_compress_activations_fused(X, W, Y, workspace=ws)  # noqa: E731
        t, _, _ = T.calls(fn)
        print(json.dumps({"case": args.case, "us_median": round(t, 3),
                          "TFLOPS": round(2.0 * M * N * K / t / 1e6, 1)}), flush=True)
    elif kind == "nvstep":
        grp, byts = nvfp4_step_group(dev, (f[0] if f else "sparse") == "sparse")
        t, _, _ = T.calls(lambda: grp())
        print(json.dumps({"case": args.case, "us_median": round(t, 3), "GBps": round(byts / t / 1e3, 1),
                          "bytes": int(byts), "workspace_bytes": grp.ws_bytes}), flush=True)
    elif kind == "nv":
        M, N, K = int(f[0]), int(f[1]), int(f[2])
        sparse = (f[3] if len(f) > 3 else "sparse") == "sparse"
        blk = 32 if sparse else 16
        W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=N + K), dev)
        X = _bf16_dev(inputs.normal_bf16((M, K), 1.0, seed=M), dev)
        xc = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        xs = torch.empty(sp24.nvfp4_scales_bytes(M, K, blk), dtype=torch.uint8, device=dev)
        xts = torch.empty(1, dtype=torch.float32, device=dev)
        sp24.quantize_nvfp4(X, blk, xc, xs, xts)
        wts = torch.empty(1, dtype=torch.float32, device=dev)
        ws_ = torch.empty(sp24.nvfp4_scales_bytes(N, K, blk), dtype=torch.uint8, device=dev)
        meta = None
        if sparse:
            wv = torch.empty(N, K // 4, dtype=torch.uint8, device=dev)
            meta = torch.empty(sp24.nvfp4_48_meta_bytes(N, K), dtype=torch.uint8, device=dev)
            sp24.prune_compress_nvfp4_48(W, wv, meta, ws_, wts)
        else:
            wv = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
            sp24.quantize_nvfp4(W, 16, wv, ws_, wts)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        a = sp24.nvfp4_gemm_args(xc, xs, xts, wv, ws_, wts, Y, K, sp24.SPARSE if sparse else sp24.DENSE, W_meta=meta)
        n = sp24.gemm_nvfp4_workspace_bytes(a)
        if n:
            wsp = torch.zeros(n, dtype=torch.uint8, device=dev)
            a.workspace, a.workspace_bytes = wsp.data_ptr(), n
            a._keep.append(wsp)
        t, _, _ = T.calls(lambda: sp24.gemm_nvfp4(a))
        wbytes = N * K * (0.25 + 1 / 16 + 1 / 32) if sparse else N * K * (0.5 + 1 / 16)
        byts = wbytes + M * K * (0.5 + 1 / blk) + 2 * M * N
        print(json.dumps({"case": args.case, "us_median": round(t, 3), "GBps": round(byts / t / 1e3, 1),
                          "TFLOPS": round(2.0 * M * N * K / t / 1e6, 1), "workspace_bytes": n}), flush=True)
    else:
        raise SystemExit("unknown case kind %r" % kind)


def run_case(args):
    """One GEMM shape, eager calls, CUDA-event timing (for profiler captures)."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    if args.case.startswith("group:"):
        run_group_case(args)
        return
    if args.case.split(":", 1)[0] in ("prune", "act", "nv", "nvstep"):
        run_other_case(args)
        return
    f = args.case.split(",")
    M, N, K = int(f[0]), int(f[1]), int(f[2])
    e4 = (f[3] if len(f) > 3 else "e4m3") == "e4m3"
    tactic = f[4] if len(f) > 4 else "sparse"
    assert tactic in ("sparse", "dense", "hybrid"), tactic
    hybrid = tactic == "hybrid"  # 2:4 weights with 25% dense 128 x 128 tiles (seeded), e4m3 only
    assert e4 or not hybrid, "hybrid tiles are e4m3"
    sparse = tactic != "dense"
    dev = torch.device("cuda", 0)
    W = torch.from_numpy(inputs.normal_bf16((N, K), 0.02, seed=N + K).view(np.int16)).view(
        torch.bfloat16).to(dev)
    X = torch.from_numpy(inputs.normal_bf16((M, K), 1.0, seed=M).view(np.int16)).view(
        torch.bfloat16).to(dev)
    wsc = xs = meta = mask = dense = None
    if sparse:
        Wv = torch.empty(N, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device=dev)
        meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
        wsc = torch.empty(N, dtype=torch.float32, device=dev) if e4 else None
        if hybrid:
            mask = torch.from_numpy(inputs.hybrid_mask(N, K, seed=0)).to(dev)
            dense = torch.empty(N, K, dtype=torch.uint8, device=dev)
        sp24.prune_compress(W, sp24.E4M3 if e4 else sp24.BF16, Wv, meta, row_scales=wsc, tile_mask=mask,
                            dense_tiles=dense)
    elif e4:
        Wv = torch.empty(N, K, dtype=torch.uint8, device=dev)
        wsc = torch.empty(N, dtype=torch.float32, device=dev)
        sp24.quantize_e4m3_rows(W, Wv, wsc)
    else:
        Wv = W
    if e4:
        Xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
        xs = torch.empty(M, dtype=torch.float32, device=dev)
        sp24.quantize_e4m3_rows(X, Xq, xs)
    else:
        Xq = X
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    a = sp24.gemm_args(Xq, Wv, Y, K, sp24.SPARSE if sparse else sp24.DENSE, W_meta=meta,
                       x_scales=xs, w_scales=wsc, tile_mask=mask, W_dense_tiles=dense)
    n = sp24.gemm_workspace_bytes(a)
    if n:
        sp24.set_workspace(a, torch.zeros(n, dtype=torch.uint8, device=dev))
    t, _, _ = Timer(dev, args.steps, args.warmup, 0.0).calls(lambda: sp24.gemm(a))  # L2 flushed per call
    eb = 1 if e4 else 2
    wbytes = N * K * eb // 2 + N * K // 8 if sparse else N * K * eb
    if hybrid:  # a dense tile reads its dense form instead of its (zero) compressed slots
        wbytes = int(0.75 * wbytes + 0.25 * N * K)
    byts = wbytes + M * K * eb + 2 * M * N
    print(json.dumps({"case": args.case, "us_median": round(t, 3), "GBps": round(byts / t / 1e3, 1),
                      "TFLOPS": round(2.0 * M * N * K / t / 1e6, 2),
                      "workspace_bytes": n}), flush=True)


# ---------------------------------------------------------------------------
# the other workloads (--config): one JSON line each
# ---------------------------------------------------------------------------
def _peaks():
    """(HBM GB/s, dense bf16 TFLOP/s burst, sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        pk = json.load(open(path))
        return (float(pk["hbm_gbs"]), float(pk["bf16_tflops"]),
                float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def _flush_l2(buf):
    """Evicts L2 by reading a buffer twice its size.  A read leaves clean lines
    behind; a memset would leave ~126 MB of dirty lines whose write-back
    lands inside the next timed call."""
    buf.max()


class Timer:
    """Device timing of eager calls for the per-workload lines: every timed
    call follows an L2 flush, all reps are enqueued before one synchronize
    (the device waits while the host enqueues, so no host launch latency lands
    between a call's events), and the reps grow until the timed calls span at
    least `min_s` seconds, so that the clock sampler (100 ms period) has
    samples inside each timed window."""

    def __init__(self, dev, reps, warm, min_s):
        import torch
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.reps, self.warm, self.min_s = reps, warm, min_s
        self.hbm, self.bf16_tf, self.bf16_tf_sus, self.peak_src = _peaks()

    def peak(self, sparse, e4):
        # dense-equivalent flops; sparse peaks are twice the dense ones, e4m3
        # twice bf16 (nominal ratios), all from the measured dense bf16 burst
        return self.bf16_tf * (2 if sparse else 1) * (2 if e4 else 1)

    def calls(self, fn):
        """(median us, min us, (t0, t1) wall-clock window of the timed calls)."""
        import torch
        for _ in range(self.warm):
            fn()
        torch.cuda.synchronize()
        reps = self.reps
        if self.min_s > 0:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(3):
                _flush_l2(self.flush)
                fn()
            e1.record()
            torch.cuda.synchronize()
            per = max(e0.elapsed_time(e1) / 3e3, 1e-6)  # seconds per flushed call
            reps = int(min(max(reps, self.min_s / per), 4000))
        t0 = time.time()
        torch.cuda._sleep(200_000 * reps)
        ev = []
        for _ in range(reps):
            _flush_l2(self.flush)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            ev.append((e0, e1))
        torch.cuda.synchronize()
        t1 = time.time()
        ts = [a.elapsed_time(b) * 1e3 for a, b in ev]
        return float(np.median(ts)), float(np.min(ts)), (t0, t1)

    def graph(self, graphs, stream):
        """us per replay of a list of CUDA graphs replayed round-robin (their
        weights together exceed L2, so no flush), and the window."""
        import torch
        for _ in range(max(self.warm, 3)):
            for g in graphs:
                g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(4):
                for g in graphs:
                    g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        per = max(e0.elapsed_time(e1) / 1e3 / (4 * len(graphs)), 1e-7)
        n = int(min(max(20, self.min_s / per / len(graphs)), 2000))
        t0 = time.time()
        with torch.cuda.stream(stream):
            torch.cuda._sleep(100_000 * n * len(graphs))
            e0.record(stream)
            for _ in range(n):
                for g in graphs:
                    g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        t1 = time.time()
        return e0.elapsed_time(e1) * 1e3 / (n * len(graphs)), (t0, t1)


def _win(*ws):
    return (min(w[0] for w in ws), max(w[1] for w in ws))


def _bf16_dev(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def _roofline(flops, byts, t_us, tflops_peak, hbm):
    t_roof = max(flops / (tflops_peak * 1e12), byts / (hbm * 1e9)) * 1e6
    bound = "tensor" if flops / (tflops_peak * 1e12) >= byts / (hbm * 1e9) else "hbm"
    return dict(bound=bound, t_roofline_us=round(t_roof, 3), frac=round(t_roof / t_us, 4))


class _Linear:
    """One linear layer's device operands in every form the suite times."""

    def __init__(self, W_bits, M, e4, dev, x_seed, mask=None, X_bits=None):
        import torch

        from semi_structured_sparse_02_b200 import inputs, sp24
        N, K = W_bits.shape
        self.M, self.N, self.K, self.e4 = M, N, K, e4
        W = _bf16_dev(W_bits, dev)
        X = _bf16_dev(inputs.normal_bf16((M, K), 1.0, seed=x_seed) if X_bits is None else X_bits, dev)
        vdt = torch.uint8 if e4 else torch.bfloat16
        self.vals = torch.empty(N, K // 2, dtype=vdt, device=dev)
        self.meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
        self.wsc = torch.empty(N, dtype=torch.float32, device=dev) if e4 else None
        self.mask = self.dense_tiles = None
        if mask is not None:
            self.mask = torch.from_numpy(mask).to(dev)
            self.dense_tiles = torch.empty(N, K, dtype=torch.uint8, device=dev)
        sp24.prune_compress(W, sp24.E4M3 if e4 else sp24.BF16, self.vals, self.meta,
                            row_scales=self.wsc, tile_mask=self.mask, dense_tiles=self.dense_tiles)
        if e4:
            self.wd = torch.empty(N, K, dtype=torch.uint8, device=dev)
            self.wdsc = torch.empty(N, dtype=torch.float32, device=dev)
            sp24.quantize_e4m3_rows(W, self.wd, self.wdsc)
            self.x = torch.empty(M, K, dtype=torch.uint8, device=dev)
            self.xs = torch.empty(M, dtype=torch.float32, device=dev)
            sp24.quantize_e4m3_rows(X, self.x, self.xs)
        else:
            self.wd, self.wdsc, self.x, self.xs = W, None, X, None
        del W, X
        self.Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        self.sp = sp24.gemm_args(self.x, self.vals, self.Y, K, sp24.SPARSE, W_meta=self.meta,
                                 x_scales=self.xs, w_scales=self.wsc, tile_mask=self.mask,
                                 W_dense_tiles=self.dense_tiles)
        self.dn = sp24.gemm_args(self.x, self.wd, self.Y, K, sp24.DENSE, x_scales=self.xs,
                                 w_scales=self.wdsc)
        for a in (self.sp, self.dn):
            n = sp24.gemm_workspace_bytes(a)
            if n:
                sp24.set_workspace(a, torch.zeros(n, dtype=torch.uint8, device=dev))

    def weight_bytes(self, sparse):
        eb = 1 if self.e4 else 2
        N, K = self.N, self.K
        if not sparse:
            return N * K * eb
        if self.mask is not None:  # dense tiles read their dense form, sparse ones values + metadata
            f = float(self.mask.float().mean().item())
            return int(f * N * K * eb + (1 - f) * (N * K * eb // 2 + N * K // 8))
        return N * K * eb // 2 + N * K // 8

    def bytes(self, sparse):
        eb = 1 if self.e4 else 2
        M, N, K = self.M, self.N, self.K
        return self.weight_bytes(sparse) + (4 * N if self.e4 else 0) + M * K * eb + \
            (4 * M if self.e4 else 0) + 2 * M * N


def _gemm_row(L, label, T, select=False, extra=None):
    """Sparse and dense call of one layer, timed; roofline fractions against
    the measured peaks; optionally the tactic selector's pick."""
    from semi_structured_sparse_02_b200 import sp24
    t_sp, _, w1 = T.calls(lambda: sp24.gemm(L.sp))
    t_dn, _, w2 = T.calls(lambda: sp24.gemm(L.dn))
    F = 2.0 * L.M * L.N * L.K
    r = dict(gemm=label, M=L.M, N=L.N, K=L.K, dtype="e4m3" if L.e4 else "bf16",
             us_sparse=round(t_sp, 2), us_dense=round(t_dn, 2),
             tflops_sparse=round(F / t_sp / 1e6, 1), tflops_dense=round(F / t_dn / 1e6, 1),
             gbs_sparse=round(L.bytes(True) / t_sp / 1e3, 1),
             speedup_vs_dense=round(t_dn / t_sp, 3),
             roofline_sparse=_roofline(F, L.bytes(True), t_sp, T.peak(True, L.e4), T.hbm),
             roofline_dense=_roofline(F, L.bytes(False), t_dn, T.peak(False, L.e4), T.hbm),
             _win=_win(w1, w2))
    if select:
        rec = sp24.select_tactic(L.sp, L.dn, warmup=3, iters=15)
        r["selected"] = rec["selected"]
        r["reason"] = rec["reason"]
        r["_rec"] = rec
    if extra:
        r.update(extra)
    print(json.dumps({k: v for k, v in r.items() if not k.startswith("_")}), file=sys.stderr, flush=True)
    return r


def cfg_tiny(dev, T):
    from semi_structured_sparse_02_b200 import inputs
    X, W = inputs.tiny(0)
    L = _Linear(W, 16, False, dev, 0, X_bits=X)
    return [_gemm_row(L, "tiny", T, select=True)]


def cfg_prefill(dev, T, Ms, dtypes=(False, True)):
    import torch

    from semi_structured_sparse_02_b200 import inputs
    rows = []
    for i, (N, K) in enumerate(inputs.PREFILL_NK):
        W = inputs.weights_with_outliers(N, K, seed=3 + i)
        for M in Ms:
            Xb = inputs.normal_bf16((M, K), 1.0, seed=3000 + M + i)
            for e4 in dtypes:
                L = _Linear(W, M, e4, dev, x_seed=0, X_bits=Xb)
                rows.append(_gemm_row(L, "prefill", T, select=True))
                del L
                torch.cuda.empty_cache()
    return rows


def cfg_activation(dev, T):
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    M, K, N = inputs.ACT_SHAPE["M"], inputs.ACT_SHAPE["K"], inputs.ACT_SHAPE["N"]
    X = _bf16_dev(inputs.student_t_bf16((M, K), 3.0, seed=4), dev)
    W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=4), dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(sp24.activations_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
    F = 2.0 * M * N * K
    rows = []
    t_f, _, w1 = T.calls(lambda: sp24.prune_compress_activations_fused(X, W, Y, workspace=ws))
    dn = sp24.gemm_args(X, W, Y, K, sp24.DENSE)
    t_d, _, w2 = T.calls(lambda: sp24.gemm(dn))
    byts = 2 * M * K + 1.125 * M * K + 1.125 * M * K + 2 * N * K + 2 * M * N
    rows.append(dict(gemm="activation", M=M, N=N, K=K, dtype="bf16",
                     us_fused=round(t_f, 2), us_dense=round(t_d, 2),
                     tflops_fused=round(F / t_f / 1e6, 1), tflops_dense=round(F / t_d / 1e6, 1),
                     speedup_vs_dense=round(t_d / t_f, 3),
                     roofline_fused=_roofline(F, byts, t_f, T.peak(True, False), T.hbm),
                     roofline_dense=_roofline(F, 2 * M * K + 2 * N * K + 2 * M * N, t_d,
                                              T.peak(False, False), T.hbm),
                     selected="sparse" if t_f < t_d else "dense", _win=_win(w1, w2),
                     note="fused = prune+compress of X every call, then the sparse GEMM with X as "
                          "the sparse operand; dense = the in-build dense GEMM on unpruned X"))
    # the prune inside the GEMM kernel (no compressed X in HBM)
    t_g, _, w3 = T.calls(lambda: sp24.prune_activations_in_gemm(X, W, Y))
    rows.append(dict(gemm="activation_in_gemm", M=M, N=N, K=K, dtype="bf16",
                     us_fused=round(t_g, 2), us_dense=round(t_d, 2), us_two_kernel=round(t_f, 2),
                     tflops_fused=round(F / t_g / 1e6, 1), speedup_vs_dense=round(t_d / t_g, 3),
                     speedup_vs_two_kernel=round(t_f / t_g, 3),
                     roofline_fused=_roofline(F, 2 * M * K + 2 * N * K + 2 * M * N, t_g, T.peak(True, False), T.hbm),
                     selected="sparse" if t_g < t_d else "dense", _win=_win(w3, w2),
                     note="X pruned and compressed in shared memory by converter warps of the CTA-pair GEMM "
                          "(re-pruned for every 256-row block of W), no compressed X in HBM"))
    # the same at the FP8 floor: X pruned and cast to e4m3 per token every call, W e4m3 per channel
    Wq = torch.empty(N, K, dtype=torch.uint8, device=dev)
    wsc = torch.empty(N, dtype=torch.float32, device=dev)
    sp24.quantize_e4m3_rows(W, Wq, wsc)
    ws8 = torch.empty(sp24.activations_e4m3_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
    t_f8, _, w1 = T.calls(lambda: sp24.prune_compress_activations_fused_e4m3(X, Wq, wsc, Y, workspace=ws8))
    Xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
    xsc = torch.empty(M, dtype=torch.float32, device=dev)
    dn8 = sp24.gemm_args(Xq, Wq, Y, K, sp24.DENSE, x_scales=xsc, w_scales=wsc)

    def dense8():
        sp24.quantize_e4m3_rows(X, Xq, xsc)
        sp24.gemm(dn8)
    t_d8, _, w2 = T.calls(dense8)
    byts8 = 2 * M * K + (0.625 * M * K + 4 * M) * 2 + N * K + 4 * N + 2 * M * N
    rows.append(dict(gemm="activation_e4m3", M=M, N=N, K=K, dtype="e4m3",
                     us_fused=round(t_f8, 2), us_dense=round(t_d8, 2),
                     tflops_fused=round(F / t_f8 / 1e6, 1), tflops_dense=round(F / t_d8 / 1e6, 1),
                     speedup_vs_dense=round(t_d8 / t_f8, 3),
                     roofline_fused=_roofline(F, byts8, t_f8, T.peak(True, True), T.hbm),
                     roofline_dense=_roofline(F, 3 * M * K + N * K + 2 * M * N, t_d8, T.peak(False, True), T.hbm),
                     selected="sparse" if t_f8 < t_d8 else "dense", _win=_win(w1, w2),
                     note="fused = prune + per-token e4m3 cast of X every call, then the e4m3 sparse GEMM "
                          "with X as the sparse operand; dense = per-token e4m3 cast of unpruned X plus the "
                          "in-build dense e4m3 GEMM"))
    for r in rows:
        print(json.dumps({k: v for k, v in r.items() if not k.startswith("_")}), file=sys.stderr, flush=True)
    return rows


def cfg_hybrid(dev, T, Ms):
    """Each GEMM of the hybrid block alone (25% dense 128 x 128 tiles, e4m3),
    with the tactic selector's pick; returns (rows, selector records)."""
    import torch

    from semi_structured_sparse_02_b200 import inputs
    rows, records = [], {}
    for gi, (name, N, K) in enumerate(inputs.HYBRID_NK):
        W = inputs.normal_bf16((N, K), 0.02, seed=5 + gi)
        mask = inputs.hybrid_mask(N, K, seed=gi)
        for M in Ms:
            L = _Linear(W, M, True, dev, x_seed=5000 + M + gi, mask=mask)
            r = _gemm_row(L, name, T, select=True, extra=dict(dense_tiles=0.25))
            records["%s_M%d" % (name, M)] = r.pop("_rec")
            rows.append(r)
            del L
            torch.cuda.empty_cache()
    return rows, records


def cfg_hybrid_block(dev, T, Ms):
    """The hybrid block as one step per token count: the per-token e4m3 cast
    of the four projections' activations (one grouped launch), then the four
    GEMMs (qkv, o, gate_up, down) as one grouped launch, captured in a CUDA
    graph; against the same step on dense e4m3 weights.  Two copies of the
    block's weights (hybrid: 2 x 139 MB, dense: 2 x 193 MB) are replayed in
    turn, so no weight is served from L2."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    copies = []
    for c in range(2):
        ws = []
        for gi, (name, N, K) in enumerate(inputs.HYBRID_NK):
            if c == 0:
                Wd = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=5 + gi), dev)
                mask = torch.from_numpy(inputs.hybrid_mask(N, K, seed=gi)).to(dev)
                vals = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
                meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
                wsc = torch.empty(N, dtype=torch.float32, device=dev)
                dense_form = torch.empty(N, K, dtype=torch.uint8, device=dev)
                sp24.prune_compress(Wd, sp24.E4M3, vals, meta, row_scales=wsc, tile_mask=mask,
                                    dense_tiles=dense_form)
                wq = torch.empty(N, K, dtype=torch.uint8, device=dev)
                wqs = torch.empty(N, dtype=torch.float32, device=dev)
                sp24.quantize_e4m3_rows(Wd, wq, wqs)
                del Wd
                ws.append((vals, meta, wsc, mask, dense_form, wq, wqs))
            else:
                ws.append(tuple(t.clone() for t in copies[0][gi]))
        copies.append(ws)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    rows = []
    byts_h = sum(int(0.25 * N * K + 0.75 * (N * K // 2 + N * K // 8)) for _, N, K in inputs.HYBRID_NK)
    byts_d = sum(N * K for _, N, K in inputs.HYBRID_NK)
    for M in Ms:
        Xs, xqs, xss, Ys = [], [], [], []
        for gi, (name, N, K) in enumerate(inputs.HYBRID_NK):
            Xs.append(_bf16_dev(inputs.normal_bf16((M, K), 1.0, seed=5000 + M + gi), dev))
            xqs.append(torch.empty(M, K, dtype=torch.uint8, device=dev))
            xss.append(torch.empty(M, dtype=torch.float32, device=dev))
            Ys.append(torch.empty(M, N, dtype=torch.bfloat16, device=dev))
        quant = sp24.QuantGroup(list(zip(Xs, xqs, xss)))
        graphs = {"hybrid": [], "dense": []}
        launches = {}
        for kind in ("hybrid", "dense"):
            for c in range(2):
                al = []
                for gi, (name, N, K) in enumerate(inputs.HYBRID_NK):
                    vals, meta, wsc, mask, dense_form, wq, wqs = copies[c][gi]
                    if kind == "hybrid":
                        al.append(sp24.gemm_args(xqs[gi], vals, Ys[gi], K, sp24.SPARSE, W_meta=meta,
                                                 x_scales=xss[gi], w_scales=wsc, tile_mask=mask,
                                                 W_dense_tiles=dense_form, flags=sp24.GEMM_W_STATIC))
                    else:
                        al.append(sp24.gemm_args(xqs[gi], wq, Ys[gi], K, sp24.DENSE, x_scales=xss[gi],
                                                 w_scales=wqs, flags=sp24.GEMM_W_STATIC))
                grp = sp24.GemmGroup(al)
                with torch.cuda.stream(stream):
                    quant()
                    grp()
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                c0 = sp24.launch_count()
                with torch.cuda.graph(g, stream=stream):
                    quant()
                    grp()
                launches[kind] = sp24.launch_count() - c0
                g._keep = (grp, al)
                graphs[kind].append(g)
        t_h, w1 = T.graph(graphs["hybrid"], stream)
        t_d, w2 = T.graph(graphs["dense"], stream)
        xb = sum(3 * M * K + 4 * M for _, _, K in inputs.HYBRID_NK)
        yb = sum(2 * M * N for _, N, _ in inputs.HYBRID_NK)
        F = sum(2.0 * M * N * K for _, N, K in inputs.HYBRID_NK)
        sc = sum(4 * N for _, N, _ in inputs.HYBRID_NK)
        bh, bd = byts_h + xb + yb + sc, byts_d + xb + yb + sc
        rows.append(dict(block_step=M, gemms=4, launches_per_step=launches["hybrid"],
                         us_hybrid=round(t_h, 2), us_dense=round(t_d, 2), speedup_vs_dense=round(t_d / t_h, 3),
                         gbs_hybrid=round(bh / t_h / 1e3, 1), gbs_dense=round(bd / t_d / 1e3, 1),
                         bytes_ratio=round(bh / bd, 4),
                         roofline_hybrid=_roofline(F, bh, t_h, T.peak(True, True), T.hbm),
                         roofline_dense=_roofline(F, bd, t_d, T.peak(False, True), T.hbm),
                         selected="hybrid" if t_h < t_d else "dense", _win=_win(w1, w2)))
        print(json.dumps({k: v for k, v in rows[-1].items() if not k.startswith("_")}), file=sys.stderr,
              flush=True)
        for gl in graphs.values():
            for g in gl:
                g.reset()
        del graphs
    return rows


def cfg_nvfp4(dev, T, shapes):
    """Pairwise 4:8 sparse NVFP4 against dense NVFP4 (the Blackwell sparse FP4
    format, 2:4-versus-quantization paper section 6.2) on linear-layer
    shapes: W pruned and cast offline, X cast to NVFP4 once (outside the
    timed call), the block-scaled GEMM timed.  Peaks: FP4 4x the measured
    bf16 dense figure, sparse 2x that (nominal ratios)."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    rows = []
    stream = torch.cuda.Stream(device=dev)

    def streamed(a, tensors, tactic):
        """us per call when the calls run back to back in a CUDA graph over
        distinct copies of the weights that together exceed L2 (no flush):
        the regime of a decode step, where each layer's weights stream once."""
        xc, xs, xts, wv, wsc, wts, meta, Y, K_ = tensors
        wbytes = wv.numel() + wsc.numel() + (meta.numel() if meta is not None else 0)
        C = int(min(8, max(2, -(-256_000_000 // wbytes))))
        al = []
        for _ in range(C):
            m2 = meta.clone() if meta is not None else None
            # static weights, as in a decode step: each call streams its
            # weights while the previous call drains
            a2 = sp24.nvfp4_gemm_args(xc, xs, xts, wv.clone(), wsc.clone(), wts, Y, K_, tactic, W_meta=m2,
                                      flags=sp24.GEMM_W_STATIC)
            n2 = sp24.gemm_nvfp4_workspace_bytes(a2)
            if n2:
                w2 = torch.zeros(n2, dtype=torch.uint8, device=dev)
                a2.workspace, a2.workspace_bytes = w2.data_ptr(), n2
                a2._keep.append(w2)
            al.append(a2)
        with torch.cuda.stream(stream):
            for a2 in al:
                sp24.gemm_nvfp4(a2, stream=stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for a2 in al:
                sp24.gemm_nvfp4(a2, stream=stream)
        g._keep = al
        t, w = T.graph([g], stream)
        return t / C, w, C

    for (M, N, K) in shapes:
        W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=N + K), dev)
        X = _bf16_dev(inputs.normal_bf16((M, K), 1.0, seed=M + K), dev)
        ops = {}
        keep = {}
        for sparse in (True, False):
            blk = 32 if sparse else 16
            xc = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
            xs = torch.empty(sp24.nvfp4_scales_bytes(M, K, blk), dtype=torch.uint8, device=dev)
            xts = torch.empty(1, dtype=torch.float32, device=dev)
            sp24.quantize_nvfp4(X, blk, xc, xs, xts)
            wts = torch.empty(1, dtype=torch.float32, device=dev)
            wsc = torch.empty(sp24.nvfp4_scales_bytes(N, K, blk), dtype=torch.uint8, device=dev)
            meta = None
            if sparse:
                wv = torch.empty(N, K // 4, dtype=torch.uint8, device=dev)
                meta = torch.empty(sp24.nvfp4_48_meta_bytes(N, K), dtype=torch.uint8, device=dev)
                sp24.prune_compress_nvfp4_48(W, wv, meta, wsc, wts)
            else:
                wv = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
                sp24.quantize_nvfp4(W, 16, wv, wsc, wts)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            a = sp24.nvfp4_gemm_args(xc, xs, xts, wv, wsc, wts, Y, K, sp24.SPARSE if sparse else sp24.DENSE,
                                     W_meta=meta)
            n = sp24.gemm_nvfp4_workspace_bytes(a)
            if n:
                wsp = torch.zeros(n, dtype=torch.uint8, device=dev)
                a.workspace, a.workspace_bytes = wsp.data_ptr(), n
                a._keep.append(wsp)
            ops[sparse] = a
            keep[sparse] = (xc, xs, xts, wv, wsc, wts, meta, Y, K)
        t_sp, _, w1 = T.calls(lambda: sp24.gemm_nvfp4(ops[True]))
        t_dn, _, w2 = T.calls(lambda: sp24.gemm_nvfp4(ops[False]))
        extra = {}
        if M <= 128:
            ts_sp, w3, c_sp = streamed(ops[True], keep[True], sp24.SPARSE)
            ts_dn, w4, c_dn = streamed(ops[False], keep[False], sp24.DENSE)
        F = 2.0 * M * N * K
        b_sp = N * K * (0.25 + 1 / 16 + 1 / 32) + M * K * (0.5 + 1 / 32) + 2 * M * N
        b_dn = N * K * (0.5 + 1 / 16) + M * K * (0.5 + 1 / 16) + 2 * M * N
        rows.append(dict(gemm="nvfp4", M=M, N=N, K=K, dtype="nvfp4",
                         us_sparse=round(t_sp, 2), us_dense=round(t_dn, 2),
                         tflops_sparse=round(F / t_sp / 1e6, 1), tflops_dense=round(F / t_dn / 1e6, 1),
                         gbs_sparse=round(b_sp / t_sp / 1e3, 1), gbs_dense=round(b_dn / t_dn / 1e3, 1),
                         speedup_vs_dense=round(t_dn / t_sp, 3),
                         selected="sparse" if t_sp < t_dn else "dense",
                         roofline_sparse=_roofline(F, b_sp, t_sp, 8 * T.bf16_tf, T.hbm),
                         roofline_dense=_roofline(F, b_dn, t_dn, 4 * T.bf16_tf, T.hbm),
                         _win=_win(w1, w2)))
        if M <= 128:
            rows[-1].update(us_sparse_streamed=round(ts_sp, 2), us_dense_streamed=round(ts_dn, 2),
                            gbs_sparse_streamed=round(b_sp / ts_sp / 1e3, 1),
                            speedup_vs_dense_streamed=round(ts_dn / ts_sp, 3),
                            roofline_sparse_streamed=_roofline(F, b_sp, ts_sp, 8 * T.bf16_tf, T.hbm),
                            streamed_copies=[c_sp, c_dn],
                            streamed_how="CUDA graph of back-to-back calls over distinct weight copies "
                                         "together larger than L2, no flush (a decode step's regime); "
                                         "us per call")
            rows[-1]["_win"] = _win(w1, w2, w3, w4)
        print(json.dumps({k: v for k, v in rows[-1].items() if not k.startswith("_")}), file=sys.stderr,
              flush=True)
        del ops, keep, W, X
        torch.cuda.empty_cache()
    return rows


def nvfp4_step_group(dev, sparse, Wb=None):
    """The decode step's 16 GEMMs (M in 1, 8, 32, 128 times the four weight
    shapes) in NVFP4 as one sp24_gemm_nvfp4_grouped launch: pairwise 4:8 or
    dense, every GEMM with its own copy of its weights (together larger than
    L2), X cast to NVFP4 beforehand, weights marked static.  Returns the group
    and the step's algorithmic bytes."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    gemms = [(M, N, K) for M in inputs.DECODE_M for (N, K) in inputs.DECODE_NK]
    if Wb is None:
        Wb = {(N, K): inputs.normal_bf16((N, K), 0.02, seed=N + K) for (N, K) in inputs.DECODE_NK}
    blk = 32 if sparse else 16
    base = {}
    for (N, K) in inputs.DECODE_NK:
        W = _bf16_dev(Wb[(N, K)], dev)
        wts = torch.empty(1, dtype=torch.float32, device=dev)
        wsc = torch.empty(sp24.nvfp4_scales_bytes(N, K, blk), dtype=torch.uint8, device=dev)
        if sparse:
            wv = torch.empty(N, K // 4, dtype=torch.uint8, device=dev)
            meta = torch.empty(sp24.nvfp4_48_meta_bytes(N, K), dtype=torch.uint8, device=dev)
            sp24.prune_compress_nvfp4_48(W, wv, meta, wsc, wts)
        else:
            wv = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
            meta = None
            sp24.quantize_nvfp4(W, 16, wv, wsc, wts)
        base[(N, K)] = (wv, meta, wsc, wts)
        del W
    al, b = [], 0
    for i, (M, N, K) in enumerate(gemms):
        wv, meta, wsc, wts = base[(N, K)]
        wv, wsc = wv.clone(), wsc.clone()  # a distinct weight copy per GEMM
        meta = meta.clone() if meta is not None else None
        X = _bf16_dev(inputs.normal_bf16((M, K), 1.0, seed=2000 + i), dev)
        xc = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        xs = torch.empty(sp24.nvfp4_scales_bytes(M, K, blk), dtype=torch.uint8, device=dev)
        xts = torch.empty(1, dtype=torch.float32, device=dev)
        sp24.quantize_nvfp4(X, blk, xc, xs, xts)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        al.append(sp24.nvfp4_gemm_args(xc, xs, xts, wv, wsc, wts, Y, K, sp24.SPARSE if sparse else sp24.DENSE,
                                       W_meta=meta, flags=sp24.GEMM_W_STATIC))
        b += (N * K * (0.25 + 1 / 16 + 1 / 32) if sparse else N * K * (0.5 + 1 / 16)) + \
            M * K * (0.5 + 1 / blk) + 2 * M * N
    return sp24.Nvfp4GemmGroup(al), b


def cfg_nvfp4_step(dev, T):
    """The NVFP4 decode step (nvfp4_step_group), pairwise 4:8 against dense,
    timed as CUDA-graph replays of the one launch."""
    import torch

    from semi_structured_sparse_02_b200 import inputs
    gemms = [(M, N, K) for M in inputs.DECODE_M for (N, K) in inputs.DECODE_NK]
    stream = torch.cuda.Stream(device=dev)
    times, wins, byts = {}, {}, {}
    F = sum(2.0 * M * N * K for M, N, K in gemms)
    Wb = {(N, K): inputs.normal_bf16((N, K), 0.02, seed=N + K) for (N, K) in inputs.DECODE_NK}
    for sparse in (True, False):
        grp, byts[sparse] = nvfp4_step_group(dev, sparse, Wb)
        with torch.cuda.stream(stream):
            grp(stream=stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            grp(stream=stream)
        g._keep = grp
        times[sparse], wins[sparse] = T.graph([g], stream)
        del g, grp
        torch.cuda.empty_cache()
    del Wb
    t_sp, t_dn = times[True], times[False]
    row = dict(gemm="nvfp4_step", gemms=len(gemms), dtype="nvfp4", us_sparse=round(t_sp, 2), us_dense=round(t_dn, 2),
               gbs_sparse=round(byts[True] / t_sp / 1e3, 1), gbs_dense=round(byts[False] / t_dn / 1e3, 1),
               weight_mb_sparse=round(byts[True] / 1e6, 1), weight_mb_dense=round(byts[False] / 1e6, 1),
               speedup_vs_dense=round(t_dn / t_sp, 3), selected="sparse" if t_sp < t_dn else "dense",
               roofline_sparse=_roofline(F, byts[True], t_sp, 8 * T.bf16_tf, T.hbm),
               roofline_dense=_roofline(F, byts[False], t_dn, 4 * T.bf16_tf, T.hbm),
               _win=_win(wins[True], wins[False]),
               note="one grouped launch of the 16 decode GEMMs per tactic, CUDA-graph replays, distinct weight "
                    "copies per GEMM (larger than L2 together); X cast outside the timed launch")
    print(json.dumps({k: v for k, v in row.items() if not k.startswith("_")}), file=sys.stderr, flush=True)
    return [row]


NVFP4_SHAPES = [(8, N, K) for N, K in [(5120, 5120), (25600, 5120), (5120, 25600), (10240, 5120)]] + \
    [(128, 5120, 25600), (8192, 4096, 4096), (8192, 12288, 4096)]


def cfg_prune(dev, T):
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    shapes = [("decode", N, K, True) for N, K in inputs.DECODE_NK] + \
             [("prefill", N, K, False) for N, K in inputs.PREFILL_NK] + \
             [("hybrid", N, K, True) for _, N, K in inputs.HYBRID_NK]
    rows = []
    for name, N, K, e4 in shapes:
        W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=N + K), dev)
        vals = torch.empty(N, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device=dev)
        meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
        sc = torch.empty(N, dtype=torch.float32, device=dev) if e4 else None
        t, _, w = T.calls(lambda: sp24.prune_compress(W, sp24.E4M3 if e4 else sp24.BF16, vals, meta, row_scales=sc))
        # algorithmic: read bf16 W once, write values + metadata (+ scales)
        byts = 2 * N * K + N * K * (1 if e4 else 2) // 2 + N * K // 8 + (4 * N if e4 else 0)
        rows.append(dict(weights=name, N=N, K=K, out="e4m3" if e4 else "bf16", us=round(t, 2),
                         gbs=round(byts / t / 1e3, 1), frac_hbm=round(byts / t / 1e3 / T.hbm, 4), _win=w))
        # the 2:4 energy-loss diagnostic on the same weights: reads 2 B per element
        share = torch.empty(N, dtype=torch.float64, device=dev)
        sums = torch.empty(2, dtype=torch.float64, device=dev)
        te, _, w = T.calls(lambda: sp24.energy_loss(W, share, sums))
        eb_ = 2 * N * K + 8 * N
        rows.append(dict(energy_loss=name, N=N, K=K, us=round(te, 2), gbs=round(eb_ / te / 1e3, 1),
                         frac_hbm=round(eb_ / te / 1e3 / T.hbm, 4), e24=round(float(sums[0] / sums[1]), 5),
                         _win=w))
        del share, sums, W, vals, meta, sc
    return rows


def _finish_rows(rows, sampler):
    """Replaces each row's timing window by the clock record taken inside it."""
    for r in rows:
        w = r.pop("_win", None)
        r.pop("_rec", None)
        if w is not None:
            c = sampler.summary(*w)
            r["clocks"] = {"sm_mhz": c["sm_mhz"], "reasons": c["reasons"], "samples": c["samples"]}
    return rows


def run_config(args):
    """Times one of the non-headline workloads and prints one JSON line; every
    row carries the clock record sampled during its timed calls."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, manifest, sp24
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sp24.lib()
    T = Timer(dev, reps=max(5, min(args.steps, 30)), warm=max(3, args.warmup), min_s=0.25)
    out = {"config": args.config, "unit_note": "us = median device time per call (CUDA events), "
           "L2 flushed before every call (block steps: graph replays over weights larger than L2); "
           "TFLOPS = 2*M*N*K / t (dense-equivalent)",
           "peaks": {"hbm_gbs": T.hbm, "bf16_dense_tflops": T.bf16_tf, "source": T.peak_src,
                     "sparse": "2x dense (2:4), e4m3 2x bf16 (nominal ratios)"}}
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    rows = []
    if args.config == "tiny":
        rows = cfg_tiny(dev, T)
    elif args.config == "prefill":
        rows = cfg_prefill(dev, T, inputs.PREFILL_M)
    elif args.config == "hybrid":
        rows, records = cfg_hybrid(dev, T, inputs.HYBRID_M)
        rows += cfg_hybrid_block(dev, T, [1, 16, 256])
        out["tactics"] = manifest.build_manifest(records, revision="synthetic-seeded")["metrics"]
    elif args.config == "activation":
        rows = cfg_activation(dev, T)
    elif args.config == "prune":
        rows = cfg_prune(dev, T)
    elif args.config == "nvfp4":
        rows = cfg_nvfp4_step(dev, T) + cfg_nvfp4(dev, T, NVFP4_SHAPES)
    time.sleep(0.2)
    sampler.stop()
    out["rows"] = _finish_rows(rows, sampler)
    out["clocks"] = sampler.summary()
    print(json.dumps(out), flush=True)


def run_configs_compact(dev):
    """The other workloads in brief, for the default bench line: prefill at
    16384 tokens (every weight shape, bf16 and e4m3), the online-activation
    paths (bf16 and FP8), the hybrid block's GEMMs alone at 1 and 4096 tokens,
    the hybrid block step at 1, 16 and 256 tokens, the tiny case, and
    pairwise 4:8 NVFP4 against dense NVFP4 at two decode shapes and one
    prefill shape.  Each
    row: sparse and dense device time, roofline fraction against the measured
    peaks, the selected tactic, and the clocks sampled during its timing."""
    import torch

    from semi_structured_sparse_02_b200 import manifest
    T = Timer(dev, reps=10, warm=3, min_s=0.2)
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    time.sleep(0.3)
    t_start = time.time()
    out = {}
    out["prefill"] = cfg_prefill(dev, T, [16384])
    torch.cuda.empty_cache()
    out["activation"] = cfg_activation(dev, T)
    torch.cuda.empty_cache()
    out["hybrid"], records = cfg_hybrid(dev, T, [1, 4096])
    torch.cuda.empty_cache()
    out["hybrid_block"] = cfg_hybrid_block(dev, T, [1, 16, 256])
    torch.cuda.empty_cache()
    out["tiny"] = cfg_tiny(dev, T)
    torch.cuda.empty_cache()
    out["nvfp4"] = cfg_nvfp4_step(dev, T) + cfg_nvfp4(dev, T, [(8, 25600, 5120), (128, 5120, 25600), (8192, 4096, 4096)])
    time.sleep(0.2)
    sampler.stop()
    keep = ("gemm", "gemms", "block_step", "M", "N", "K", "dtype", "us_sparse", "us_dense", "us_fused", "us_hybrid",
            "tflops_sparse", "tflops_fused", "speedup_vs_dense", "selected", "reason", "clocks")
    for name, rows in out.items():
        _finish_rows(rows, sampler)
        for r in rows:
            for k in ("roofline_sparse", "roofline_fused", "roofline_hybrid"):
                if k in r:
                    r["frac"] = r[k]["frac"]
                    r["bound"] = r[k]["bound"]
            if "roofline_dense" in r:
                r["frac_dense"] = r["roofline_dense"]["frac"]
            if "roofline_sparse_streamed" in r:
                r["frac_streamed"] = r["roofline_sparse_streamed"]["frac"]
            for k in list(r):
                if k not in keep and k not in ("frac", "bound", "frac_dense", "frac_streamed", "us_sparse_streamed",
                                               "us_dense_streamed", "speedup_vs_dense_streamed"):
                    del r[k]
    out["hybrid_tactics"] = manifest.build_manifest(records, revision="synthetic-seeded")["metrics"]
    out["clocks"] = sampler.summary()
    out["seconds"] = round(time.time() - t_start, 1)
    out["how"] = ("eager calls with an L2 flush (a 256 MB read) before each, median of >= 0.2 s of timed calls "
                  "per figure (block steps, and the *_streamed NVFP4 decode figures: CUDA-graph replays over "
                  "weight copies together larger than L2, no flush); "
                  "frac = roofline time max(flops/peak, bytes/HBM) / measured time, peaks from "
                  "MEASURED_PEAKS.json (sparse 2x dense, e4m3 2x bf16)")
    return out


def main():
    args = parse()
    if args.case:
        run_case(args)
        return
    if args.config != "decode":
        run_config(args)
        return
    from semi_structured_sparse_02_b200 import replicas
    rank, world, local_rank = replicas.env_ranks()
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, world)
        return
    if world > 1:
        import torch
        torch.cuda.set_device(local_rank)
        replicas.init("nccl", local_rank)
    out = run_product(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        replicas.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
