"""The C ABI on a machine without a GPU: the library loads, exports every
function include/sp24.h declares, computes sizes, and rejects bad arguments
with the documented status codes before any CUDA launch."""
import ctypes

import pytest
import torch

from semi_structured_sparse_02_b200 import build as sp24_build
from semi_structured_sparse_02_b200 import sp24

sp24_build.build()
L = sp24.lib()

FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: validation fails first
NO_GPU = not torch.cuda.is_available()


def test_exports_every_declared_function():
    names = sp24.header_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(L, n), n


def test_sizes():
    assert sp24.values_bytes(256, 256, sp24.BF16) == 65536
    assert sp24.values_bytes(256, 256, sp24.E4M3) == 32768
    assert sp24.meta_bytes(256, 256) == 8192          # 256*256/8: one bit per element
    assert sp24.meta_bytes(40, 256) == 4096           # rows padded to a 128-row block
    assert sp24.values_bytes(256, 256, sp24.BF16) + sp24.meta_bytes(256, 256) == 73728


def test_status_strings():
    for s in range(10):
        assert isinstance(sp24.status_string(s), str) and sp24.status_string(s)
    assert sp24.status_string(sp24.SP24_ERR_NOT_2_4).startswith("operand not eligible")


def prune(src=FAKE, rows=256, K=256, ld=256, dt=sp24.BF16, vals=FAKE, meta=FAKE, sc=None, mask=None,
          dense=None):
    return L.sp24_prune_compress(src, rows, K, ld, dt, vals, meta, sc, mask, dense, None)


def test_prune_compress_validation():
    assert prune(src=None) == sp24.SP24_ERR_NULL
    assert prune(meta=None) == sp24.SP24_ERR_NULL
    assert prune(dt=sp24.E4M3) == sp24.SP24_ERR_NULL          # scales required
    assert prune(dt=sp24.F32) == sp24.SP24_ERR_DTYPE
    assert prune(mask=FAKE) == sp24.SP24_ERR_NULL             # dense tiles required
    assert prune(rows=0) == sp24.SP24_ERR_INVALID_ARG
    assert prune(K=192, ld=192) == sp24.SP24_ERR_NOT_2_4
    assert prune(ld=100) == sp24.SP24_ERR_INVALID_ARG
    assert prune(ld=260) == sp24.SP24_ERR_ALIGNMENT
    assert prune(src=FAKE + 8) == sp24.SP24_ERR_ALIGNMENT


@pytest.mark.skipif(not NO_GPU, reason="only meaningful without a device")
def test_valid_arguments_without_device_report_unsupported_device():
    assert prune() == sp24.SP24_ERR_UNSUPPORTED_DEVICE
    assert L.sp24_last_device_error() == sp24.SP24_ERR_UNSUPPORTED_DEVICE


def gemm_args(**kw):
    a = sp24.GemmArgs()
    a.M, a.N, a.K = kw.get("M", 16), kw.get("N", 256), kw.get("K", 256)
    a.in_dtype = kw.get("in_dtype", sp24.BF16)
    a.out_dtype = kw.get("out_dtype", sp24.BF16)
    a.tactic = kw.get("tactic", sp24.SPARSE)
    a.X, a.ldx = kw.get("X", FAKE), kw.get("ldx", a.K)
    a.W, a.ldw = kw.get("W", FAKE), kw.get("ldw", a.K // 2 if a.tactic == sp24.SPARSE else a.K)
    a.W_meta = kw.get("W_meta", FAKE)
    a.x_scales = kw.get("x_scales", None)
    a.w_scales = kw.get("w_scales", None)
    a.tile_dense_mask = kw.get("mask", None)
    a.W_dense_tiles = kw.get("dense", None)
    a.Y, a.ldy = kw.get("Y", FAKE), kw.get("ldy", a.N)
    return a


def g(**kw):
    return L.sp24_gemm(ctypes.byref(gemm_args(**kw)), None)


def test_gemm_validation():
    assert L.sp24_gemm(None, None) == sp24.SP24_ERR_NULL
    assert g(M=0) == sp24.SP24_ERR_INVALID_ARG
    assert g(in_dtype=sp24.F32) == sp24.SP24_ERR_DTYPE
    assert g(out_dtype=sp24.E4M3) == sp24.SP24_ERR_DTYPE
    assert g(X=None) == sp24.SP24_ERR_NULL
    assert g(W_meta=None) == sp24.SP24_ERR_NULL
    assert g(N=200, ldy=200) == sp24.SP24_ERR_NOT_2_4           # sparse needs N % 128
    assert g(K=320, ldx=320, ldw=160) == sp24.SP24_ERR_NOT_2_4  # sparse needs K % 128
    assert g(in_dtype=sp24.E4M3) == sp24.SP24_ERR_NULL          # scales required
    assert g(mask=FAKE, dense=FAKE) == sp24.SP24_ERR_DTYPE      # hybrid is e4m3 only
    assert g(ldx=100) == sp24.SP24_ERR_INVALID_ARG
    assert g(ldx=260) == sp24.SP24_ERR_ALIGNMENT
    assert g(X=FAKE + 4) == sp24.SP24_ERR_ALIGNMENT
    assert g(tactic=sp24.DENSE, K=200, ldx=200, ldw=200) == sp24.SP24_ERR_ALIGNMENT
    assert g(tactic=7) == sp24.SP24_ERR_INVALID_ARG
    assert L.sp24_gemm_workspace_bytes(ctypes.byref(gemm_args(M=0))) == 0


def test_grouped_quantize_validation():
    f = L.sp24_quantize_e4m3_rows_grouped
    assert f(None, 1, None) == sp24.SP24_ERR_NULL
    items = (sp24.QuantItem * 2)()
    items[0] = sp24.QuantItem(FAKE, 4, 256, 256, FAKE, FAKE)
    items[1] = sp24.QuantItem(FAKE, 4, 256, 256, None, FAKE)
    assert f(items, 0, None) == sp24.SP24_ERR_INVALID_ARG
    assert f(items, 33, None) == sp24.SP24_ERR_INVALID_ARG
    assert f(items, 2, None) == sp24.SP24_ERR_NULL
    items[1] = sp24.QuantItem(FAKE, 4, 250, 256, FAKE, FAKE)
    assert f(items, 2, None) == sp24.SP24_ERR_ALIGNMENT
    items[1] = sp24.QuantItem(FAKE, 0, 256, 256, FAKE, FAKE)
    assert f(items, 2, None) == sp24.SP24_ERR_INVALID_ARG


def test_activation_and_selector_validation():
    f = L.sp24_prune_compress_activations_fused
    assert f(None, 16, 256, 256, FAKE, 256, 256, FAKE, 256, sp24.BF16, None, None, None, 0, None) \
        == sp24.SP24_ERR_NULL
    assert f(FAKE, 16, 192, 192, FAKE, 256, 192, FAKE, 256, sp24.BF16, None, None, None, 0, None) \
        == sp24.SP24_ERR_NOT_2_4
    assert f(FAKE, 16, 256, 256, FAKE, 256, 256, FAKE, 256, sp24.BF16, None, None, None, 0, None) \
        == sp24.SP24_ERR_WORKSPACE
    assert f(FAKE, 16, 256, 256, FAKE, 256, 256, FAKE, 256, sp24.BF16, FAKE, None, None, 0, None) \
        == sp24.SP24_ERR_NULL
    rec = sp24.TacticRecord()
    assert L.sp24_select_tactic(None, None, 1, 1, ctypes.byref(rec), None) == sp24.SP24_ERR_NULL
    d = gemm_args(tactic=sp24.DENSE)
    assert L.sp24_select_tactic(None, ctypes.byref(d), 1, 0, ctypes.byref(rec), None) \
        == sp24.SP24_ERR_INVALID_ARG
    # values [16 x 128] bf16 (4096 B, 256-aligned) + one row block x 2 chunks of image
    assert sp24.activations_workspace_bytes(16, 256) == 4096 + 2 * 2048


def test_grouped_gemm_validation():
    f = L.sp24_gemm_grouped
    assert f(None, 1, None, 0, None) == sp24.SP24_ERR_NULL
    arr = (sp24.GemmArgs * 17)(*[gemm_args() for _ in range(17)])
    assert f(arr, 0, None, 0, None) == sp24.SP24_ERR_INVALID_ARG
    assert f(arr, 17, None, 0, None) == sp24.SP24_ERR_INVALID_ARG   # at most 16 problems
    arr[1] = gemm_args(in_dtype=sp24.E4M3, x_scales=FAKE, w_scales=FAKE)
    assert f(arr, 2, None, 0, None) == sp24.SP24_ERR_INVALID_ARG    # mixed input dtypes
    arr[1] = gemm_args(out_dtype=sp24.F32)
    assert f(arr, 2, None, 0, None) == sp24.SP24_ERR_INVALID_ARG    # mixed output dtypes
    arr[1] = gemm_args(tactic=sp24.DENSE)
    assert f(arr, 2, None, 0, None) == sp24.SP24_ERR_INVALID_ARG    # mixed tactics
    if NO_GPU:  # token classes may differ within a group: validation passes (no device here)
        arr[1] = gemm_args(M=17)
        assert f(arr, 2, None, 0, None) == sp24.SP24_ERR_UNSUPPORTED_DEVICE
    arr[1] = gemm_args(M=9, N=512, K=1024)
    assert f(arr, 2, FAKE + 8, 1024, None) == sp24.SP24_ERR_ALIGNMENT
    arr[1] = gemm_args(X=None)
    assert f(arr, 2, None, 0, None) == sp24.SP24_ERR_NULL           # each problem validated
    e4 = dict(in_dtype=sp24.E4M3, x_scales=FAKE, w_scales=FAKE)
    arr[0] = gemm_args(mask=FAKE, dense=FAKE, **e4)
    arr[1] = gemm_args(**e4)
    assert f(arr, 2, None, 0, None) == sp24.SP24_ERR_INVALID_ARG    # hybrid and plain weights in one group
    assert L.sp24_gemm_grouped_workspace_bytes(arr, 2) == 0


@pytest.mark.skipif(not NO_GPU, reason="only meaningful without a device")
def test_grouped_gemm_without_device():
    arr = (sp24.GemmArgs * 2)(gemm_args(), gemm_args(M=3, N=512, K=512))
    assert L.sp24_gemm_grouped(arr, 2, None, 0, None) == sp24.SP24_ERR_UNSUPPORTED_DEVICE


def test_activation_e4m3_validation():
    f = L.sp24_prune_compress_activations_fused_e4m3
    ok = dict(X=FAKE, M=16, K=256, ldx=256, W=FAKE, ws=FAKE, N=256, ldw=256, Y=FAKE, ldy=256, out=sp24.BF16,
              xv=FAKE, xm=FAKE, xs=FAKE, work=None, wbytes=0)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["X"], a["M"], a["K"], a["ldx"], a["W"], a["ws"], a["N"], a["ldw"], a["Y"], a["ldy"], a["out"],
                 a["xv"], a["xm"], a["xs"], a["work"], a["wbytes"], None)
    assert call(ws=None) == sp24.SP24_ERR_NULL                  # weight scales required
    assert call(xs=None) == sp24.SP24_ERR_NULL                  # all three outputs or none
    assert call(xv=None, xm=None, xs=None) == sp24.SP24_ERR_WORKSPACE
    assert call(K=192, ldx=192, ldw=192) == sp24.SP24_ERR_NOT_2_4
    assert call(ldw=264) == sp24.SP24_ERR_ALIGNMENT             # e4m3 rows: 16-byte multiple
    assert call(out=sp24.E4M3) == sp24.SP24_ERR_DTYPE
    # values [16 x 128] e4m3 (2048 B) + image (one row block x 2 chunks) + 16 scales
    assert sp24.activations_e4m3_workspace_bytes(16, 256) == 2048 + 2 * 2048 + 16 * 4


def test_energy_loss_validation():
    f = L.sp24_energy_loss
    assert f(None, 4, 64, 64, FAKE, None, None) == sp24.SP24_ERR_NULL
    assert f(FAKE, 4, 64, 64, None, None, None) == sp24.SP24_ERR_NULL      # one output at least
    assert f(FAKE, 0, 64, 64, FAKE, None, None) == sp24.SP24_ERR_INVALID_ARG
    assert f(FAKE, 4, 60, 60, FAKE, None, None) == sp24.SP24_ERR_NOT_2_4
    assert f(FAKE, 4, 64, 68, FAKE, None, None) == sp24.SP24_ERR_ALIGNMENT
    assert f(FAKE + 8, 4, 64, 64, FAKE, None, None) == sp24.SP24_ERR_ALIGNMENT


def test_binding_constants_match_the_header():
    """The Python binding's enum and flag values are the header's."""
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sp24.h")).read()
    defines = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define\s+SP24_(GEMM_\w+)\s+(\d+)u", hdr)}
    assert defines == {"GEMM_W_STATIC": sp24.GEMM_W_STATIC, "GEMM_SINGLE_CTA": sp24.GEMM_SINGLE_CTA,
                       "GEMM_CTA_PAIR": sp24.GEMM_CTA_PAIR, "GEMM_AFTER_INDEPENDENT": sp24.GEMM_AFTER_INDEPENDENT}
    # flag bits are distinct
    vals = list(defines.values())
    assert all(v & (v - 1) == 0 for v in vals) and len(set(vals)) == len(vals)


def test_nvfp4_sizes():
    assert sp24.nvfp4_48_values_bytes(256, 512) == 256 * 128          # 2 bits of value per position
    assert sp24.nvfp4_48_meta_bytes(256, 512) == 2 * 2 * 2048         # 4 bits per 8 positions
    assert sp24.nvfp4_48_meta_bytes(40, 256) == 2048                  # rows padded to 128
    assert sp24.nvfp4_codes_bytes(10, 512) == 2560
    assert sp24.nvfp4_scales_bytes(200, 512, 32) == 256 * 16
    assert sp24.nvfp4_scales_bytes(200, 512, 16) == 256 * 32
    assert sp24.nvfp4_scales_bytes(200, 512, 8) == 0
    # 4:8 NVFP4 stores 2 + 0.5 bits per position of values and metadata
    # plus 8 bits per 32 positions of scales: 2.75 bits against dense NVFP4's 4.5
    rows, K = 1024, 4096
    sparse = sp24.nvfp4_48_values_bytes(rows, K) + sp24.nvfp4_48_meta_bytes(rows, K) + \
        sp24.nvfp4_scales_bytes(rows, K, 32)
    dense = sp24.nvfp4_codes_bytes(rows, K) + sp24.nvfp4_scales_bytes(rows, K, 16)
    assert sparse * 8 == rows * K * 2.75 and dense * 8 == rows * K * 4.5


def nvargs(**kw):
    a = sp24.Nvfp4GemmArgs()
    a.M, a.N, a.K = kw.get("M", 16), kw.get("N", 256), kw.get("K", 512)
    a.tactic = kw.get("tactic", sp24.SPARSE)
    a.out_dtype = kw.get("out_dtype", sp24.BF16)
    for f in ("X", "x_scales", "x_tensor_scale", "W", "W_meta", "w_scales", "w_tensor_scale", "Y"):
        setattr(a, f, kw.get(f, FAKE))
    a.ldy = kw.get("ldy", a.N)
    return a


def nvgemm(**kw):
    return L.sp24_gemm_nvfp4(ctypes.byref(nvargs(**kw)), None)


def test_nvfp4_grouped_validation():
    G = L.sp24_gemm_nvfp4_grouped
    arr = lambda *xs: (sp24.Nvfp4GemmArgs * len(xs))(*xs)
    assert G(None, 1, None, 0, None) == sp24.SP24_ERR_NULL
    one = arr(nvargs())
    assert G(one, 0, None, 0, None) == sp24.SP24_ERR_INVALID_ARG
    assert G(arr(*[nvargs() for _ in range(17)]), 17, None, 0, None) == sp24.SP24_ERR_INVALID_ARG
    assert G(arr(nvargs(), nvargs(tactic=sp24.DENSE)), 2, None, 0, None) == sp24.SP24_ERR_INVALID_ARG
    assert G(arr(nvargs(), nvargs(out_dtype=sp24.F32)), 2, None, 0, None) == sp24.SP24_ERR_DTYPE
    assert G(arr(nvargs(), nvargs(K=384)), 2, None, 0, None) == sp24.SP24_ERR_NOT_2_4  # each problem's own checks
    assert G(one, 1, FAKE + 4, 1024, None) == sp24.SP24_ERR_ALIGNMENT
    assert L.sp24_gemm_nvfp4_grouped_workspace_bytes(arr(nvargs(), nvargs(tactic=sp24.DENSE)), 2) == 0
    if NO_GPU:
        assert G(arr(nvargs(M=1), nvargs(M=128, N=512, K=1024)), 2, None, 0, None) == sp24.SP24_ERR_UNSUPPORTED_DEVICE


def test_nvfp4_validation():
    assert L.sp24_gemm_nvfp4(None, None) == sp24.SP24_ERR_NULL
    assert nvgemm(M=0) == sp24.SP24_ERR_INVALID_ARG
    assert nvgemm(tactic=5) == sp24.SP24_ERR_INVALID_ARG
    assert nvgemm(out_dtype=sp24.E4M3) == sp24.SP24_ERR_DTYPE
    assert nvgemm(W_meta=None) == sp24.SP24_ERR_NULL
    assert nvgemm(tactic=sp24.DENSE, W_meta=None) != sp24.SP24_ERR_NULL  # dense needs no metadata
    assert nvgemm(x_tensor_scale=None) == sp24.SP24_ERR_NULL
    assert nvgemm(K=384) == sp24.SP24_ERR_NOT_2_4
    assert nvgemm(tactic=sp24.DENSE, K=384) == sp24.SP24_ERR_ALIGNMENT
    assert nvgemm(X=FAKE + 8) == sp24.SP24_ERR_ALIGNMENT
    assert nvgemm(ldy=100) == sp24.SP24_ERR_INVALID_ARG
    P = L.sp24_prune_compress_nvfp4_48
    assert P(None, 128, 512, 512, FAKE, FAKE, FAKE, FAKE, None) == sp24.SP24_ERR_NULL
    assert P(FAKE, 128, 384, 384, FAKE, FAKE, FAKE, FAKE, None) == sp24.SP24_ERR_NOT_2_4
    assert P(FAKE, 0, 512, 512, FAKE, FAKE, FAKE, FAKE, None) == sp24.SP24_ERR_INVALID_ARG
    assert P(FAKE, 128, 512, 516, FAKE, FAKE, FAKE, FAKE, None) == sp24.SP24_ERR_ALIGNMENT
    Q = L.sp24_quantize_nvfp4
    assert Q(FAKE, 16, 512, 512, 8, FAKE, FAKE, FAKE, None) == sp24.SP24_ERR_INVALID_ARG
    assert Q(FAKE, 16, 96, 96, 16, FAKE, FAKE, FAKE, None) == sp24.SP24_ERR_ALIGNMENT
    assert Q(FAKE, 16, 512, 512, 32, FAKE, FAKE, FAKE + 2, None) == sp24.SP24_ERR_ALIGNMENT
    if NO_GPU:
        assert nvgemm() == sp24.SP24_ERR_UNSUPPORTED_DEVICE
        assert P(FAKE, 128, 512, 512, FAKE, FAKE, FAKE, FAKE, None) == sp24.SP24_ERR_UNSUPPORTED_DEVICE


def test_prune_in_gemm_validation():
    F = L.sp24_prune_activations_in_gemm
    ok = dict(X=FAKE, M=512, K=1024, ldx=1024, W=FAKE, N=512, ldw=1024, Y=FAKE, ldy=512, dt=sp24.BF16, xv=None,
              xm=None)

    def call(**kw):
        a = dict(ok, **kw)
        return F(a["X"], a["M"], a["K"], a["ldx"], a["W"], a["N"], a["ldw"], a["Y"], a["ldy"], a["dt"], a["xv"],
                 a["xm"], None)
    assert call(X=None) == sp24.SP24_ERR_NULL
    assert call(xv=FAKE) == sp24.SP24_ERR_NULL           # values and metadata together
    assert call(dt=sp24.E4M3) == sp24.SP24_ERR_DTYPE
    assert call(M=128) == sp24.SP24_ERR_INVALID_ARG       # the CTA-pair kernel: M, N >= 256
    assert call(N=200, ldy=200) == sp24.SP24_ERR_INVALID_ARG
    assert call(K=1000, ldx=1000, ldw=1000) == sp24.SP24_ERR_NOT_2_4
    assert call(ldx=1028) == sp24.SP24_ERR_ALIGNMENT
    assert call(Y=FAKE + 2) == sp24.SP24_ERR_ALIGNMENT
    if NO_GPU:
        assert call() == sp24.SP24_ERR_UNSUPPORTED_DEVICE
