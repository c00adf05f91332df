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
from tests.gpu_helpers import OracleSparseW, check_tolerance, dev, oracle_x, workspace_for

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


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # M=128, N=20480, K=25600 plans a stream-K schedule whose accumulators
    # (160 tiles x 64 KB) exceed the fixed scratch; the call must refuse
    M, N, K = 128, 20480, 25600
    X = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    W = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.meta_bytes(N, K), dtype=torch.uint8, device="cuda")
    xs = torch.ones(M, dtype=torch.float32, device="cuda")
    ws_ = torch.ones(N, dtype=torch.float32, device="cuda")
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = sp24.gemm_args(X, W, Y, K, sp24.SPARSE, W_meta=meta, x_scales=xs, w_scales=ws_)
    assert sp24.gemm_workspace_bytes(a) > sp24.gemm_noalloc_max_scratch_bytes()
    st = sp24.lib().sp24_gemm_noalloc(ctypes.byref(a), None)
    assert st == sp24.SP24_ERR_WORKSPACE
