"""Tactic audit manifest: one record per GEMM ("layer") saying whether the
sparse call was eligible, which tactic the timing-based selector picked and
why, plus the summary counts and the sparse GPU-time coverage.

"Production 2:4 Structured Sparsity for LLMs" (oh-bug.com), section
"Sparse Tactic Audit: Layer-by-Layer Kernel Execution Auditing": every build
produces a layer-level manifest; Sparse GPU-Time Coverage is the time of the
selected sparse kernels over the total GPU time, and is more informative
than layer counts.  Section "Dense Fallback and Hybrid Sparsity Design":
every fallback decision is logged with its reason.

The records come from sp24_select_tactic (the C library times both tactics
on the device); this module only aggregates them.
"""
from __future__ import annotations

import json
from typing import Dict, Iterable


def build_manifest(records: Dict[str, dict], pattern: str = "2:4", revision: str = "") -> dict:
    """records: layer name -> sp24.select_tactic() result dict."""
    layers = {}
    t_sparse_selected = 0.0
    t_total = 0.0
    n_eligible = n_sparse = 0
    for name, r in records.items():
        entry = {"eligible": bool(r["eligible"]), "selected": r["selected"]}
        if r["selected"] == "dense" and r.get("reason"):
            entry["reason"] = r["reason"]
        entry["t_sparse_us"] = round(float(r["t_sparse_us"]), 3) if r["eligible"] else None
        entry["t_dense_us"] = round(float(r["t_dense_us"]), 3)
        layers[name] = entry
        n_eligible += int(bool(r["eligible"]))
        if r["selected"] == "sparse":
            n_sparse += 1
            t = float(r["t_sparse_us"])
            t_sparse_selected += t
        else:
            t = float(r["t_dense_us"])
        t_total += t
    n = len(records)
    metrics = {
        "candidate_layers": n,
        "eligible_layers": n_eligible,
        "sparse_selected_layers": n_sparse,
        "dense_fallback_layers": n - n_sparse,
        "sparse_selection_ratio": round(n_sparse / n_eligible, 4) if n_eligible else 0.0,
        "sparse_gpu_time_coverage": round(t_sparse_selected / t_total, 4) if t_total > 0 else 0.0,
    }
    return {"model_revision": revision, "sparsity_pattern": pattern, "metrics": metrics,
            "layers": layers}


def coverage(selected_times: Iterable) -> float:
    """Sparse GPU-time coverage of (tactic, time) pairs of the kernels that ran."""
    tot = sp = 0.0
    for tactic, t in selected_times:
        tot += t
        if tactic == "sparse":
            sp += t
    return sp / tot if tot > 0 else 0.0


def dumps(manifest: dict) -> str:
    return json.dumps(manifest, indent=2, sort_keys=False)
