"""Pairwise 4:8 sparse NVFP4 and dense NVFP4 on the GPU, through the C ABI,
against the oracle: the prune / cast kernels bit for bit (values, metadata
image, scale image, tensor scale), the block-scaled GEMMs within the
tolerance |y - y_ref| <= 2e-3 * sum_k |x_k w_k| + 1e-6 of the oracle's fp64
product of the dequantized operands.  The GEMM inputs come from the oracle,
not from the device cast, so the GEMM checks do not lean on the cast kernels."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from semi_structured_sparse_02_b200 import inputs, sp24
from tests.gpu_helpers import check_tolerance, dev, dev_bf16, f32_bits, u8, workspace_for

pytestmark = pytest.mark.gpu


def _f32_bits(x: float) -> int:
    return int(np.array([x], np.float32).view(np.uint32)[0])


def _device_48(W):
    rows, K = W.shape
    vals = torch.empty(rows, K // 4, dtype=torch.uint8, device="cuda")
    meta = torch.empty(sp24.nvfp4_48_meta_bytes(rows, K), dtype=torch.uint8, device="cuda")
    sc = torch.empty(sp24.nvfp4_scales_bytes(rows, K, 32), dtype=torch.uint8, device="cuda")
    ts = torch.empty(1, dtype=torch.float32, device="cuda")
    sp24.prune_compress_nvfp4_48(dev_bf16(W), vals, meta, sc, ts)
    torch.cuda.synchronize()
    return vals, meta, sc, ts


def _oracle_48(W):
    rows, K = W.shape
    v, m, s, st = orc.nvfp4_48_compress(W)
    return v, orc.nvfp4_48_meta_image(m, rows, K), orc.nvfp4_scale_image(s, rows), st, (v, m, s)


def _ties_and_zeros(rows, K, seed):
    """bf16 rows with exact pair-energy ties, zero groups and zero rows."""
    g = np.random.default_rng(seed)
    W = inputs.normal_bf16((rows, K), 0.02, seed=seed)
    W[0, :] = 0                                   # a zero row: every block scale 0
    W[1, :8] = np.array([0x3F80, 0, 0, 0x3F80, 0x3F80, 0, 0, 0x3F80], np.uint16)  # four equal pairs
    W[2, 8:16] = np.array([0xBF80, 0x3F80, 0x3F80, 0xBF80, 0, 0, 0, 0], np.uint16)  # signs, two ties
    W[3, 16:32] = 0                               # zero groups
    W[4, :] = g.integers(0, 3, size=K).astype(np.uint16) << 14 & 0x4000  # tiny set of values, many ties
    return W


@pytest.mark.parametrize("rows,K", [(1, 256), (128, 256), (200, 512), (256, 5120), (37, 1280)])
def test_nvfp4_48_prune_compress_bit_exact(rows, K):
    W = inputs.normal_bf16((rows, K), 0.02, seed=rows + K)
    if rows >= 8:
        W = _ties_and_zeros(rows, K, seed=rows)
    vals, meta, sc, ts = _device_48(W)
    ov, om, osc, ost, _ = _oracle_48(W)
    assert np.array_equal(u8(vals), ov), "values"
    assert np.array_equal(u8(meta), om), "metadata image"
    assert np.array_equal(u8(sc), osc), "scale image"
    assert int(f32_bits(ts)[0]) == _f32_bits(ost), "tensor scale"


@pytest.mark.parametrize("rows,K,block", [(1, 64, 16), (16, 512, 16), (130, 1024, 32), (8, 5120, 32),
                                          (300, 768, 16)])
def test_nvfp4_quantize_bit_exact(rows, K, block):
    X = inputs.student_t_bf16((rows, K), 3.0, seed=rows * K + block)
    if rows > 1:
        X[1, :] = 0
    codes = torch.empty(rows, K // 2, dtype=torch.uint8, device="cuda")
    sc = torch.empty(sp24.nvfp4_scales_bytes(rows, K, block), dtype=torch.uint8, device="cuda")
    ts = torch.empty(1, dtype=torch.float32, device="cuda")
    sp24.quantize_nvfp4(dev_bf16(X), block, codes, sc, ts)
    torch.cuda.synchronize()
    oc, osc, ost = orc.nvfp4_quantize(X, block=block)
    assert np.array_equal(u8(codes), oc), "codes"
    assert np.array_equal(u8(sc), orc.nvfp4_scale_image(osc, rows)), "scale image"
    assert int(f32_bits(ts)[0]) == _f32_bits(ost), "tensor scale"


def _gemm_case(M, N, K, tactic, out_f32=True, seed=0, flags=0, use_ws=True):
    X, W = inputs.linear_pair(M, N, K, seed=seed + M + N + K, outliers=True)
    block = 32 if tactic == sp24.SPARSE else 16
    xc, xs, xst = orc.nvfp4_quantize(X, block=block)
    X_hat = orc.nvfp4_dequant(xc, xs, xst, M, K, block=block)
    if tactic == sp24.SPARSE:
        wv, wm, wsc, wst = orc.nvfp4_48_compress(W)
        W_hat = orc.nvfp4_48_dequant(wv, wm, wsc, wst, N, K)
        Wd, Wm = dev(wv), dev(orc.nvfp4_48_meta_image(wm, N, K))
    else:
        wv, wsc, wst = orc.nvfp4_quantize(W, block=16)
        W_hat = orc.nvfp4_dequant(wv, wsc, wst, N, K, block=16)
        Wd, Wm = dev(wv), None
    Y = torch.empty(M, N, dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    a = sp24.nvfp4_gemm_args(dev(xc), dev(orc.nvfp4_scale_image(xs, M)), torch.tensor([xst], device="cuda"),
                             Wd, dev(orc.nvfp4_scale_image(wsc, N)), torch.tensor([wst], device="cuda"),
                             Y, K, tactic, W_meta=Wm, flags=flags)
    if use_ws:
        n = sp24.gemm_nvfp4_workspace_bytes(a)
        if n:
            ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
            a.workspace, a.workspace_bytes = ws.data_ptr(), n
            a._keep.append(ws)
    y_ref, a_ref = orc.gemm_f64(X_hat, W_hat)
    return a, Y, y_ref, a_ref


NV_SHAPES = [
    (1, 256, 512),      # decode-like, one stage
    (16, 512, 1024),    # two stages
    (40, 384, 768),     # a half last stage (sparse: K % 512 == 256)
    (128, 256, 256),    # one half stage only
    (200, 256, 2048),   # two token tiles of 128 rows, ragged
    (8, 1024, 5120),    # stream-K over many stages
]


@pytest.mark.parametrize("M,N,K", NV_SHAPES)
@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_gemm_nvfp4_parity(M, N, K, tactic):
    for out_f32 in (True, False):
        a, Y, y_ref, a_ref = _gemm_case(M, N, K, tactic, out_f32)
        sp24.gemm_nvfp4(a)
        torch.cuda.synchronize()
        assert sp24.last_device_error() == sp24.SP24_OK
        check_tolerance(Y.float().cpu().numpy().astype(np.float64), y_ref, a_ref,
                        "nvfp4 M%d N%d K%d tactic %d f32=%s" % (M, N, K, tactic, out_f32))


# NVFP4 groups: token-count classes, shapes and stage counts mixed in one launch
NV_GROUPS = {
    "decode": [(1, 256, 512), (8, 1024, 5120), (16, 512, 1024), (40, 384, 768)],
    "to128": [(1, 512, 1024), (128, 256, 2048), (33, 384, 512), (200, 256, 1024), (8, 768, 2560)],
}


@pytest.mark.parametrize("group", sorted(NV_GROUPS))
@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_gemm_nvfp4_grouped_parity(group, tactic):
    """One sp24_gemm_nvfp4_grouped launch over problems of different M, N and
    K (each with its own token-tile width; one output type per group, as the
    call requires), with the group's workspace and without one (whole tiles),
    twice each; every output against the oracle."""
    out_f32 = group == "decode"  # one output type per group: fp32 here, bf16 for the other
    cases = [_gemm_case(M, N, K, tactic, out_f32=out_f32, seed=17 * i, use_ws=False)
             for i, (M, N, K) in enumerate(NV_GROUPS[group])]
    for use_ws in (True, False):
        grp = sp24.Nvfp4GemmGroup([c[0] for c in cases])  # allocates the workspace the schedule needs
        if not use_ws:
            grp.workspace, grp.ws_bytes = None, 0  # whole tiles per CTA
        for _ in range(2):
            for (_, Y, _, _) in cases:
                Y.fill_(float("nan"))
            grp()
            torch.cuda.synchronize()
            assert sp24.last_device_error() == sp24.SP24_OK
            for i, (_, Y, y_ref, a_ref) in enumerate(cases):
                check_tolerance(Y.float().cpu().numpy().astype(np.float64), y_ref, a_ref,
                                "nvfp4 group %s problem %d tactic %d ws=%s" % (group, i, tactic, use_ws))


@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_gemm_nvfp4_whole_tiles_and_static_weights(tactic):
    # without a workspace the stream-K shape runs whole tiles; with
    # W_STATIC the weights stream before the upstream kernel finishes
    for use_ws, flags in ((False, 0), (True, sp24.GEMM_W_STATIC)):
        a, Y, y_ref, a_ref = _gemm_case(8, 1024, 5120, tactic, seed=3, flags=flags, use_ws=use_ws)
        for _ in range(2):
            Y.fill_(float("nan"))
            sp24.gemm_nvfp4(a)
            torch.cuda.synchronize()
            check_tolerance(Y.cpu().numpy().astype(np.float64), y_ref, a_ref, "nvfp4 ws=%s" % use_ws)


def test_nvfp4_device_cast_then_gemm_full_size_sampled():
    """The decode shape end to end on the device: W pruned and cast by the
    device kernel, X cast per call, the sparse 4:8 GEMM; sampled outputs
    against the oracle on the same bf16 inputs."""
    M, N, K = 8, 5120, 5120
    X, W = inputs.linear_pair(M, N, K, seed=55)
    vals, meta, wsc, wts = _device_48(W)
    xc = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    xs = torch.empty(sp24.nvfp4_scales_bytes(M, K, 32), dtype=torch.uint8, device="cuda")
    xts = torch.empty(1, dtype=torch.float32, device="cuda")
    sp24.quantize_nvfp4(dev_bf16(X), 32, xc, xs, xts)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    a = sp24.nvfp4_gemm_args(xc, xs, xts, vals, wsc, wts, Y, K, sp24.SPARSE, W_meta=meta)
    ws = workspace_for_nv(a)
    sp24.gemm_nvfp4(a)
    torch.cuda.synchronize()
    g = np.random.default_rng(8)
    ns = g.choice(N, size=64, replace=False)
    ms = g.integers(0, M, size=64)
    wv, wm, wsc_o, wst = orc.nvfp4_48_compress(W)  # tensor scale over all of W
    W_hat = orc.nvfp4_48_dequant(wv[ns], wm[ns], wsc_o[ns], wst, ns.size, K)
    xc_o, xs_o, xst = orc.nvfp4_quantize(X, block=32)
    X_hat = orc.nvfp4_dequant(xc_o, xs_o, xst, M, K, block=32)
    y_ref, a_ref = orc.gemm_f64_sampled(X_hat, W_hat, ms, np.arange(ns.size))
    y_gpu = Y.float().cpu().numpy().astype(np.float64)[ms, ns]
    check_tolerance(y_gpu, y_ref, a_ref, "nvfp4 decode sampled")
    del ws


@pytest.mark.parametrize("tactic", [sp24.SPARSE, sp24.DENSE])
def test_nvfp4_prefill_full_size_sampled(tactic):
    """The prefill shape 8192 x 4096 x 4096 end to end on the device (W pruned
    and cast, or cast, by the device kernels; X cast per call; the block-scaled
    GEMM on 128-row tiles); sampled outputs against the oracle's fp64 product of
    the dequantized operands, with the tensor scales over all of W and X."""
    M, N, K = 8192, 4096, 4096
    X, W = inputs.linear_pair(M, N, K, seed=77)
    blk = 32 if tactic == sp24.SPARSE else 16
    if tactic == sp24.SPARSE:
        vals, meta, wsc, wts = _device_48(W)
    else:
        vals = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
        wsc = torch.empty(sp24.nvfp4_scales_bytes(N, K, 16), dtype=torch.uint8, device="cuda")
        wts = torch.empty(1, dtype=torch.float32, device="cuda")
        sp24.quantize_nvfp4(dev_bf16(W), 16, vals, wsc, wts)
        meta = None
    xc = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    xs = torch.empty(sp24.nvfp4_scales_bytes(M, K, blk), dtype=torch.uint8, device="cuda")
    xts = torch.empty(1, dtype=torch.float32, device="cuda")
    sp24.quantize_nvfp4(dev_bf16(X), blk, xc, xs, xts)
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    a = sp24.nvfp4_gemm_args(xc, xs, xts, vals, wsc, wts, Y, K, tactic, W_meta=meta)
    ws = workspace_for_nv(a)
    sp24.gemm_nvfp4(a)
    torch.cuda.synchronize()
    assert sp24.last_device_error() == sp24.SP24_OK
    g = np.random.default_rng(9)
    ns = g.choice(N, size=48, replace=False)
    ms = g.choice(M, size=48, replace=False)
    if tactic == sp24.SPARSE:
        wv, wm, wsc_o, wst = orc.nvfp4_48_compress(W)  # tensor scale over all of W
        W_hat = orc.nvfp4_48_dequant(wv[ns], wm[ns], wsc_o[ns], wst, ns.size, K)
    else:
        wv, wsc_o, wst = orc.nvfp4_quantize(W, block=16)
        W_hat = orc.nvfp4_dequant(wv[ns], wsc_o[ns], wst, ns.size, K, block=16)
    xc_o, xs_o, xst = orc.nvfp4_quantize(X, block=blk)
    X_hat = orc.nvfp4_dequant(xc_o[ms], xs_o[ms], xst, ms.size, K, block=blk)
    y_ref, a_ref = orc.gemm_f64_sampled(X_hat, W_hat, np.arange(ms.size), np.arange(ns.size))
    y_gpu = Y.cpu().numpy().astype(np.float64)[ms, ns]
    check_tolerance(y_gpu, y_ref, a_ref, "nvfp4 prefill sampled tactic %d" % tactic)
    del ws


def workspace_for_nv(a):
    n = sp24.gemm_nvfp4_workspace_bytes(a)
    if n == 0:
        return None
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    a.workspace, a.workspace_bytes = ws.data_ptr(), n
    a._keep.append(ws)
    return ws
