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
                   help="weight rows per GEMM in the CPU-baseline sample")
    p.add_argument("--config", default="decode",
                   choices=["decode", "tiny", "prefill", "activation", "hybrid", "prune"],
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
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        props = torch.cuda.get_device_properties(device_index)
        self.bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        self.proc = None
        self.lines = []

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
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


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
        inst.append(dict(M=M, N=N, K=K, X=X, xq=xq, xs=xs, a_sp=a_sp, a_dn=a_dn))
    del base
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    # the per-token e4m3 casts of the 16 independent activation matrices run
    # as one grouped launch; then the GEMMs run as grouped launches, one per
    # (tactic, token-count class): M in {1, 8} share one, M = 32 and M = 128
    # one each.  Launches are chained by programmatic dependent launch, each
    # streaming its weights while the previous kernel drains.
    quant_all = sp24.QuantGroup([(it["X"], it["xq"], it["xs"]) for it in inst])

    def make_groups(pick):
        """Grouped launches for the tactic pick(it) of every GEMM.  The GEMMs
        are independent and all their inputs come from the cast before the
        first group, so every group after the first is marked as following
        an independent GEMM launch: its CTAs start as SMs free up instead of
        waiting for the previous group to finish."""
        by = {}
        for it in inst:
            t = pick(it)
            a = it["a_sp"] if t == "sparse" else it["a_dn"]
            by.setdefault((t, sp24.m_class(it["M"])), []).append(a)
        return [sp24.GemmGroup(v, after_independent=i > 0) for i, (_, v) in enumerate(sorted(by.items()))]

    groups = {"sparse": make_groups(lambda it: "sparse"), "dense": make_groups(lambda it: "dense")}

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
    kinds = ("sparse", "dense", "selected", "ungrouped", "gemm_only")
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

    ms_dense = time_graph(graphs["dense"], K_steps, W_warm)
    ms_sel = time_graph(graphs["selected"], K_steps, W_warm)
    ms_gemm = time_graph(graphs["gemm_only"], K_steps, W_warm)
    ms_ungrouped = time_graph(graphs["ungrouped"], K_steps, W_warm)

    # end to end through the public API: pinned host X in, host Y out, eager calls
    X_host = torch.empty(x_elems, dtype=torch.bfloat16, pin_memory=True)
    X_host.copy_(X_all.cpu())
    Y_host = torch.empty(y_elems, dtype=torch.bfloat16, pin_memory=True)
    e2e_steps = max(3, min(K_steps, 50))
    with torch.cuda.stream(stream):
        for _ in range(2):
            X_all.copy_(X_host, non_blocking=True)
            step("sparse")
            Y_host.copy_(Y_all, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            X_all.copy_(X_host, non_blocking=True)
            step("sparse")
            Y_host.copy_(Y_all, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)

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
        "config": {
            "workload": WORKLOAD,
            "gemms_per_step": len(gemms),
            "M": sorted(set(M for M, _, _ in gemms)),
            "NK": [list(s) for s in shapes],
            "parallelism": "replicas" if world > 1 else "single-gpu",
            "l2": L2_NOTE,
            "timing": "CUDA graph of one step replayed K times; CUDA events on the replay stream",
            "step": ("one grouped per-token e4m3 cast of the 16 activation matrices, then the 16 "
                     "GEMMs as %d grouped launches (one per token-count class: M in {1,8}, 32, 128)"
                     % len(groups["sparse"])),
        },
        "tflops": round(world * step_flops / t_step / 1e12, 3),
        "speedup_vs_dense": round(ms_dense / ms_sparse, 4),
        "ms_per_step_dense": round(ms_dense / K_steps, 5),
        "ms_per_step_selected": round(ms_sel / K_steps, 5),
        "ms_per_step_ungrouped": round(ms_ungrouped / K_steps, 5),
        "tactics": man["metrics"],
        "roofline": {
            "kernel": "k_gemm sparse e4m3 (tcgen05.mma.sp), grouped launch",
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
            "how": "eager public-API calls (one sp24_quantize_e4m3_rows_grouped + %d "
                   "sp24_gemm_grouped) with one pinned H2D copy of X and one D2H copy of Y per step"
                   % len(groups["sparse"]),
        },
        "gpu_launches": launches["sparse"] * K_steps,
    }
    if rank == 0:
        out["cpu_baseline"] = cpu_baseline(args.cpu_rows)
    return out


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def oracle_gemm_sample(M, N, K, rows, seed):
    """Time the oracle's per-call path for one decode GEMM on `rows` weight
    rows: per-token E4M3 quantization of X, dequantization, fp64 sparse GEMM.
    Weight preparation (prune + quantize, offline) is untimed.  Returns the
    time scaled to the full N rows."""
    from oracle import oracle as orc
    from semi_structured_sparse_02_b200 import inputs
    R = min(rows, N)
    Wb = inputs.normal_bf16((R, K), 0.02, seed=seed)
    vq, canon, wsc, _ = orc.prune_compress_e4m3(Wb)
    wv = orc.e4m3_decode(vq) * wsc.astype(np.float64)[:, None]
    Xb = inputs.normal_bf16((M, K), 1.0, seed=seed + 1)
    t0 = time.perf_counter()
    q, s = orc.quantize_rows_e4m3(Xb)
    Xh = orc.e4m3_decode(q) * s.astype(np.float64)[:, None]
    orc.gemm_sparse_f64(Xh, wv, canon)
    dt = time.perf_counter() - t0
    return dt * N / R


def cpu_baseline(rows):
    gemms = gemm_list()
    t = 0.0
    b = 0
    for i, (M, N, K) in enumerate(gemms):
        t += oracle_gemm_sample(M, N, K, rows, seed=7000 + i)
        b += gemm_bytes(M, N, K) + quant_bytes(M, K)
    return {"value": round(b / t / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "all 16 decode GEMMs, %d weight rows each (time scaled by N/%d), "
                      "single-threaded C oracle, fp64" % (rows, rows)}


def run_reference(args, world):
    gemms = gemm_list()
    rows = 64
    for i in range(args.warmup):
        M, N, K = gemms[i % len(gemms)]
        oracle_gemm_sample(M, N, K, rows, seed=9000 + i)
    t = 0.0
    b = 0
    for i in range(args.steps):
        M, N, K = gemms[i % len(gemms)]
        t += oracle_gemm_sample(M, N, K, rows, seed=9100 + i)
        b += gemm_bytes(M, N, K) + quant_bytes(M, K)
    value = b / t / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded numpy normal draws rounded to bf16)",
        "config": {"workload": WORKLOAD, "gemms_per_step": 1,
                   "note": "the reference arm is the CPU oracle; one step = one of the 16 decode "
                           "GEMMs in turn, on %d weight rows, time scaled to N rows" % rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "one decode GEMM per step on %d weight rows" % rows},
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    t, _ = _time_calls(lambda: grp(), args.steps, args.warmup, flush)
    byts = sum(gemm_bytes(a.M, a.N, a.K) for a in argl)
    print(json.dumps({"case": args.case, "gemms": len(argl), "us_median": round(t, 3),
                      "GBps": round(byts / t / 1e3, 1), "bytes": byts,
                      "workspace_bytes": grp.ws_bytes}), flush=True)


def run_case(args):
    """One GEMM shape, eager calls, CUDA-event timing (for profiler captures)."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, sp24
    if args.case.startswith("group:"):
        run_group_case(args)
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2: evicts W between calls
    t, _ = _time_calls(lambda: sp24.gemm(a), args.steps, args.warmup, flush)
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
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        pk = json.load(open(path))
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def _flush_l2(buf):
    """Evicts L2 by reading a buffer twice its size.  A read leaves clean lines
    behind; a memset would leave ~126 MB of dirty lines whose write-back
    lands inside the next timed call."""
    buf.max()


def _time_calls(fn, reps, warmup, flush):
    """Median and min device time (us) of fn(), each call after an L2 flush.

    All reps are enqueued before one synchronize, so the host runs ahead of
    the device and no host-side launch latency lands between the events."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    # the device waits (~0.1 ms per rep) while the host enqueues the reps, so
    # no host launch latency lands between a call's events even when one
    # call plus its flush takes less device time than the host takes to issue it
    torch.cuda._sleep(200_000 * reps)
    ev = []
    for _ in range(reps):
        _flush_l2(flush)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    ts = [e0.elapsed_time(e1) * 1e3 for e0, e1 in ev]
    return float(np.median(ts)), float(np.min(ts))


def _bf16_dev(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def _roofline(flops, byts, t_us, tflops_peak, hbm):
    t_roof = max(flops / (tflops_peak * 1e12), byts / (hbm * 1e9)) * 1e6
    bound = "tensor" if flops / (tflops_peak * 1e12) >= byts / (hbm * 1e9) else "hbm"
    return dict(bound=bound, t_roofline_us=round(t_roof, 3), frac=round(t_roof / t_us, 4))


class _Linear:
    """One linear layer's device operands in every form the suite times."""

    def __init__(self, W_bits, M, e4, dev, x_seed, mask=None):
        import torch

        from semi_structured_sparse_02_b200 import inputs, sp24
        N, K = W_bits.shape
        self.M, self.N, self.K, self.e4 = M, N, K, e4
        W = _bf16_dev(W_bits, dev)
        X = _bf16_dev(inputs.normal_bf16((M, K), 1.0, seed=x_seed), dev)
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

    def sparse_bytes(self):
        eb = 1 if self.e4 else 2
        M, N, K = self.M, self.N, self.K
        return N * K * eb // 2 + N * K // 8 + (4 * N if self.e4 else 0) + M * K * eb + \
            (4 * M if self.e4 else 0) + 2 * M * N

    def dense_bytes(self):
        eb = 1 if self.e4 else 2
        M, N, K = self.M, self.N, self.K
        return N * K * eb + (4 * N if self.e4 else 0) + M * K * eb + (4 * M if self.e4 else 0) + 2 * M * N


def run_config(args):
    """Times one of the non-headline workloads and prints one JSON line."""
    import torch

    from semi_structured_sparse_02_b200 import inputs, manifest, sp24
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sp24.lib()
    hbm, bf16_tf, src = _peaks()
    # dense-equivalent flops; sparse peaks are twice the dense ones, e4m3 twice bf16
    peak = {("sparse", False): 2 * bf16_tf, ("dense", False): bf16_tf,
            ("sparse", True): 4 * bf16_tf, ("dense", True): 2 * bf16_tf}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps, warm = max(5, min(args.steps, 30)), max(3, args.warmup)
    rows = []
    out = {"config": args.config, "unit_note": "us = median device time per call (CUDA events), "
           "L2 flushed before every call; TFLOPS = 2*M*N*K / t (dense-equivalent)",
           "peaks": {"hbm_gbs": hbm, "bf16_dense_tflops": bf16_tf, "source": src,
                     "sparse": "2x dense (2:4), e4m3 2x bf16 (nominal ratios)"}}

    def gemm_row(L, label, extra=None):
        t_sp, t_sp_min = _time_calls(lambda: sp24.gemm(L.sp), reps, warm, flush)
        t_dn, t_dn_min = _time_calls(lambda: sp24.gemm(L.dn), reps, warm, flush)
        F = 2.0 * L.M * L.N * L.K
        r = dict(gemm=label, M=L.M, N=L.N, K=L.K, dtype="e4m3" if L.e4 else "bf16",
                 us_sparse=round(t_sp, 2), us_dense=round(t_dn, 2),
                 tflops_sparse=round(F / t_sp / 1e6, 1), tflops_dense=round(F / t_dn / 1e6, 1),
                 gbs_sparse=round(L.sparse_bytes() / t_sp / 1e3, 1),
                 speedup_vs_dense=round(t_dn / t_sp, 3),
                 roofline_sparse=_roofline(F, L.sparse_bytes(), t_sp, peak[("sparse", L.e4)], hbm),
                 roofline_dense=_roofline(F, L.dense_bytes(), t_dn, peak[("dense", L.e4)], hbm))
        if extra:
            r.update(extra)
        rows.append(r)
        print(json.dumps(r), file=sys.stderr, flush=True)

    if args.config == "tiny":
        X, W = inputs.tiny(0)
        L = _Linear(W, 16, False, dev, 0)
        L.x.copy_(_bf16_dev(X, dev))
        gemm_row(L, "tiny")
    elif args.config == "prefill":
        for i, (N, K) in enumerate(inputs.PREFILL_NK):
            W = inputs.weights_with_outliers(N, K, seed=3 + i)
            for e4 in (False, True):
                for M in inputs.PREFILL_M:
                    L = _Linear(W, M, e4, dev, x_seed=3000 + M + i)
                    gemm_row(L, "prefill")
                    del L
                    torch.cuda.empty_cache()
    elif args.config == "hybrid":
        records = {}
        for e4 in (True,):
            for gi, (name, N, K) in enumerate(inputs.HYBRID_NK):
                W = inputs.normal_bf16((N, K), 0.02, seed=5 + gi)
                mask = inputs.hybrid_mask(N, K, seed=gi)
                for M in inputs.HYBRID_M:
                    L = _Linear(W, M, e4, dev, x_seed=5000 + M + gi, mask=mask)
                    rec = sp24.select_tactic(L.sp, L.dn, warmup=3, iters=15)
                    records["%s_M%d" % (name, M)] = rec
                    gemm_row(L, name, dict(selected=rec["selected"], dense_tiles=0.25))
                    del L
                    torch.cuda.empty_cache()
        out["tactics"] = manifest.build_manifest(records, revision="synthetic-seeded")["metrics"]
    elif args.config == "activation":
        M, K, N = inputs.ACT_SHAPE["M"], inputs.ACT_SHAPE["K"], inputs.ACT_SHAPE["N"]
        X = _bf16_dev(inputs.student_t_bf16((M, K), 3.0, seed=4), dev)
        W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=4), dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(sp24.activations_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
        t_f, t_f_min = _time_calls(lambda: sp24.prune_compress_activations_fused(X, W, Y, workspace=ws),
                                   reps, warm, flush)
        dn = sp24.gemm_args(X, W, Y, K, sp24.DENSE)
        t_d, t_d_min = _time_calls(lambda: sp24.gemm(dn), reps, warm, flush)
        F = 2.0 * M * N * K
        byts = 2 * M * K + 1.125 * M * K + 1.125 * M * K + 2 * N * K + 2 * M * N
        rows.append(dict(gemm="activation", M=M, N=N, K=K, dtype="bf16",
                         us_fused=round(t_f, 2), us_dense=round(t_d, 2),
                         tflops_fused=round(F / t_f / 1e6, 1), tflops_dense=round(F / t_d / 1e6, 1),
                         speedup_vs_dense=round(t_d / t_f, 3),
                         roofline_fused=_roofline(F, byts, t_f, peak[("sparse", False)], hbm),
                         roofline_dense=_roofline(F, 2 * M * K + 2 * N * K + 2 * M * N, t_d,
                                                  peak[("dense", False)], hbm),
                         note="fused = prune+compress of X every call, then the sparse GEMM with X as "
                              "the sparse operand; dense = the in-build dense GEMM on unpruned X"))
        # the same at the FP8 floor: X pruned and cast to e4m3 per token every call, W e4m3 per channel
        Wq = torch.empty(N, K, dtype=torch.uint8, device=dev)
        wsc = torch.empty(N, dtype=torch.float32, device=dev)
        sp24.quantize_e4m3_rows(W, Wq, wsc)
        ws8 = torch.empty(sp24.activations_e4m3_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
        t_f8, _ = _time_calls(lambda: sp24.prune_compress_activations_fused_e4m3(X, Wq, wsc, Y, workspace=ws8),
                              reps, warm, flush)
        Xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
        xsc = torch.empty(M, dtype=torch.float32, device=dev)
        dn8 = sp24.gemm_args(Xq, Wq, Y, K, sp24.DENSE, x_scales=xsc, w_scales=wsc)

        def dense8():
            sp24.quantize_e4m3_rows(X, Xq, xsc)
            sp24.gemm(dn8)
        t_d8, _ = _time_calls(dense8, reps, warm, flush)
        t_d8g, _ = _time_calls(lambda: sp24.gemm(dn8), reps, warm, flush)
        byts8 = 2 * M * K + (0.625 * M * K + 4 * M) * 2 + N * K + 4 * N + 2 * M * N
        rows.append(dict(gemm="activation_e4m3", M=M, N=N, K=K, dtype="e4m3",
                         us_fused=round(t_f8, 2), us_dense=round(t_d8, 2), us_dense_gemm_only=round(t_d8g, 2),
                         tflops_fused=round(F / t_f8 / 1e6, 1), tflops_dense=round(F / t_d8 / 1e6, 1),
                         speedup_vs_dense=round(t_d8 / t_f8, 3),
                         roofline_fused=_roofline(F, byts8, t_f8, peak[("sparse", True)], hbm),
                         roofline_dense=_roofline(F, 3 * M * K + N * K + 2 * M * N, t_d8, peak[("dense", True)], hbm),
                         note="fused = prune + per-token e4m3 cast of X every call (row amax, prune/cast, "
                              "scale passes), then the e4m3 sparse GEMM with X as the sparse operand; dense = "
                              "per-token e4m3 cast of unpruned X plus the in-build dense e4m3 GEMM"))
    elif args.config == "prune":
        shapes = [("decode", N, K, True) for N, K in inputs.DECODE_NK] + \
                 [("prefill", N, K, False) for N, K in inputs.PREFILL_NK] + \
                 [("hybrid", N, K, True) for _, N, K in inputs.HYBRID_NK]
        for name, N, K, e4 in shapes:
            W = _bf16_dev(inputs.normal_bf16((N, K), 0.02, seed=N + K), dev)
            vals = torch.empty(N, K // 2, dtype=torch.uint8 if e4 else torch.bfloat16, device=dev)
            meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device=dev)
            sc = torch.empty(N, dtype=torch.float32, device=dev) if e4 else None
            t, t_min = _time_calls(lambda: sp24.prune_compress(W, sp24.E4M3 if e4 else sp24.BF16,
                                                               vals, meta, row_scales=sc),
                                   reps, warm, flush)
            # algorithmic: read bf16 W once, write values + metadata (+ scales)
            byts = 2 * N * K + N * K * (1 if e4 else 2) // 2 + N * K // 8 + (4 * N if e4 else 0)
            rows.append(dict(weights=name, N=N, K=K, out="e4m3" if e4 else "bf16", us=round(t, 2),
                             gbs=round(byts / t / 1e3, 1), frac_hbm=round(byts / t / 1e3 / hbm, 4)))
            print(json.dumps(rows[-1]), file=sys.stderr, flush=True)
            # the 2:4 energy-loss diagnostic on the same weights: reads 2 B per element
            share = torch.empty(N, dtype=torch.float64, device=dev)
            sums = torch.empty(2, dtype=torch.float64, device=dev)
            te, _ = _time_calls(lambda: sp24.energy_loss(W, share, sums), reps, warm, flush)
            eb_ = 2 * N * K + 8 * N
            rows.append(dict(energy_loss=name, N=N, K=K, us=round(te, 2), gbs=round(eb_ / te / 1e3, 1),
                             frac_hbm=round(eb_ / te / 1e3 / hbm, 4),
                             e24=round(float(sums[0] / sums[1]), 5)))
            del share, sums
            del W, vals, meta, sc
    out["rows"] = rows
    print(json.dumps(out), flush=True)



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
