"""The allocation-free GEMM entry point (sp24_gemm_noalloc), for callers that
cannot allocate device memory: it must give the same results as sp24_gemm
with a caller-provided workspace, call after call, taking its scratch from
the fixed array inside the library.  This file is collected last."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from semi_structured_sparse_02_b200 import inputs, sp24
from tests.gpu_helpers import OracleSparseW, check_tolerance, dev, dev_bf16, oracle_x, workspace_for

pytestmark = pytest.mark.gpu


def _args(M, N, K, seed):
    X, W = inputs.linear_pair(M, N, K, seed=seed)
    xq, xs, X_hat = oracle_x(X, True)
    ref = OracleSparseW(W, e4m3=True)
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    a = sp24.gemm_args(dev(xq), dev(ref.values), Y, K, sp24.SPARSE, W_meta=dev(ref.image),
                       x_scales=dev(xs), w_scales=dev(ref.scales))
    y_ref, a_ref = orc.gemm_f64(X_hat, ref.W_hat)
    return a, Y, y_ref, a_ref


@pytest.mark.parametrize("M,N,K", [(8, 1024, 4096), (32, 2560, 5120), (1, 5120, 5120)])
def test_noalloc_matches_existing_entry_point_on_two_calls(M, N, K):
    a, Y, y_ref, a_ref = _args(M, N, K, seed=M + N)
    ws = workspace_for(a)
    assert ws is not None  # the shape uses scratch (stream-K)
    assert sp24.gemm_workspace_bytes(a) <= sp24.gemm_noalloc_max_scratch_bytes()
    sp24.set_workspace(a, ws)
    sp24.gemm(a)
    torch.cuda.synchronize()
    y_existing = Y.cpu().numpy().astype(np.float64)
    check_tolerance(y_existing, y_ref, a_ref, "existing entry point")
    for call in range(2):
        Y.fill_(float("nan"))
        sp24.gemm_noalloc(a)
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        y = Y.cpu().numpy().astype(np.float64)
        check_tolerance(y, y_ref, a_ref, "noalloc call %d" % call)
        check_tolerance(y, y_existing, a_ref, "noalloc call %d vs existing" % call)


def _sampled_ref(X, W, ms, ns, e4):
    """Oracle values at (ms[i], ns[i]) only (full-size shapes)."""
    ref = OracleSparseW(W[ns], e4m3=e4)
    _, _, X_hat = oracle_x(X[ms], e4)
    return orc.gemm_f64_sampled(X_hat, ref.W_hat, np.arange(ms.size), np.arange(ns.size))


def test_noalloc_runs_whole_tiles_where_stream_k_scratch_would_not_fit():
    # M=128, N=5120, K=25600 (a decode-workload shape): its stream-K schedule
    # needs more scratch than the fixed array, so the allocation-free call runs
    # whole tiles per CTA; the results must still match sp24_gemm's (which
    # runs stream-K with a caller workspace) on two calls in a row
    M, N, K = 128, 5120, 25600
    X, W = inputs.linear_pair(M, N, K, seed=77)
    Wd = torch.from_numpy(W.view(np.int16).copy()).view(torch.bfloat16).cuda()
    vals = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    wsc = torch.empty(N, dtype=torch.float32, device="cuda")
    sp24.prune_compress(Wd, sp24.E4M3, vals, meta, row_scales=wsc)
    xq, xs, _ = oracle_x(X, True)
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    a = sp24.gemm_args(dev(xq), vals, Y, K, sp24.SPARSE, W_meta=meta, x_scales=dev(xs), w_scales=wsc)
    assert sp24.gemm_workspace_bytes(a) > sp24.gemm_noalloc_max_scratch_bytes()
    sp24.set_workspace(a, workspace_for(a))
    sp24.gemm(a)
    torch.cuda.synchronize()
    g = np.random.default_rng(5)
    ms = np.concatenate([g.integers(0, M, size=200), [0, M - 1]])
    ns = np.concatenate([g.integers(0, N, size=200), [0, N - 1]])
    y_ref, a_ref = _sampled_ref(X, W, ms, ns, True)
    y_existing = Y.cpu().numpy().astype(np.float64)[ms, ns]
    check_tolerance(y_existing, y_ref, a_ref, "existing entry point")
    for call in range(2):
        Y.fill_(float("nan"))
        assert sp24.lib().sp24_gemm_noalloc(ctypes.byref(a), None) == sp24.SP24_OK
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        y = Y.cpu().numpy().astype(np.float64)
        assert np.isfinite(y).all()
        check_tolerance(y[ms, ns], y_ref, a_ref, "noalloc call %d" % call)
        check_tolerance(y[ms, ns], y_existing, a_ref, "noalloc call %d vs existing" % call)


@pytest.mark.parametrize("e4", [False, True])
def test_noalloc_on_cta_pair_shapes(e4):
    # M, N >= 256 run on the CTA-pair kernel, which takes no scratch
    M, N, K = 256, 256, 4096
    X, W = inputs.linear_pair(M, N, K, seed=11)
    xq, xs, X_hat = oracle_x(X, e4)
    ref = OracleSparseW(W, e4m3=e4)
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    a = sp24.gemm_args(dev(xq) if e4 else dev_bf16(X), dev(ref.values) if e4 else dev_bf16(ref.values), Y, K,
                       sp24.SPARSE,
                       W_meta=dev(ref.image), x_scales=dev(xs) if e4 else None,
                       w_scales=dev(ref.scales) if e4 else None)
    y_ref, a_ref = orc.gemm_f64(X_hat, ref.W_hat)
    sp24.gemm(a)
    torch.cuda.synchronize()
    y_existing = Y.cpu().numpy().astype(np.float64)
    check_tolerance(y_existing, y_ref, a_ref, "existing entry point")
    for call in range(2):
        Y.fill_(float("nan"))
        sp24.gemm_noalloc(a)
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        y = Y.cpu().numpy().astype(np.float64)
        check_tolerance(y, y_ref, a_ref, "noalloc call %d" % call)
        check_tolerance(y, y_existing, a_ref, "noalloc call %d vs existing" % call)
