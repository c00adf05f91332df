"""Manifest aggregation (host logic), pinned to the page's example manifest
and to the oracle's statement of the tactic rule and coverage."""
import json
import os

from oracle import oracle as orc
from semi_structured_sparse_02_b200 import manifest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "manifest_example.json")


def _rec(eligible, t_sparse, t_dense):
    sel, _, _ = orc.select_tactic([t_sparse], [t_dense]) if eligible else ("dense", 0, 0)
    reason = "" if sel == "sparse" else ("Alignment failure" if not eligible
                                         else "Dense kernel %.2fx faster" % (t_sparse / t_dense))
    return dict(eligible=eligible, selected=sel, reason=reason, t_sparse_us=t_sparse,
                t_dense_us=t_dense)


def test_counts_and_ratio_reproduce_the_page_example():
    g = json.load(open(GOLDEN))
    recs = {}
    # 71 layers where sparse wins, 25 where dense wins, all 96 eligible
    for i in range(71):
        recs["l%d" % i] = _rec(True, 1.0, 2.0)
    for i in range(71, 96):
        recs["l%d" % i] = _rec(True, 2.3, 2.0)
    m = manifest.build_manifest(recs)["metrics"]
    for k in ("candidate_layers", "eligible_layers", "sparse_selected_layers",
              "dense_fallback_layers", "sparse_selection_ratio"):
        assert m[k] == g[k], k
    assert manifest.build_manifest(recs)["layers"]["l80"]["reason"] == "Dense kernel 1.15x faster"


def test_coverage_matches_oracle_definition():
    recs = {"a": _rec(True, 3.0, 5.0), "b": _rec(True, 4.0, 2.0), "c": _rec(False, 0.0, 1.0)}
    m = manifest.build_manifest(recs)
    ran = [("sparse", 3.0), ("dense", 2.0), ("dense", 1.0)]
    assert abs(m["metrics"]["sparse_gpu_time_coverage"] - round(orc.sparse_gpu_time_coverage(ran), 4)) < 1e-12
    assert m["layers"]["c"] == {"eligible": False, "selected": "dense", "reason": "Alignment failure",
                                "t_sparse_us": None, "t_dense_us": 1.0}
    assert abs(manifest.coverage(ran) - 0.5) < 1e-12
    g = json.load(open(GOLDEN))
    assert abs(manifest.coverage([("sparse", 0.684), ("dense", 0.316)]) - g["sparse_gpu_time_coverage"]) < 1e-12
