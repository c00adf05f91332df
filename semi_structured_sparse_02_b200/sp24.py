"""ctypes binding of libsp24.so (the C ABI in include/sp24.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Tensors are torch tensors on the current CUDA device (torch is used
for device memory and streams); their data pointers and the current stream
are passed through unchanged.  If the library has not been built this module
raises on first use -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsp24.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "sp24.h")

SP24_OK = 0
SP24_ERR_INVALID_ARG = 1
SP24_ERR_NULL = 2
SP24_ERR_DTYPE = 3
SP24_ERR_ALIGNMENT = 4
SP24_ERR_NOT_2_4 = 5
SP24_ERR_UNSUPPORTED_DEVICE = 6
SP24_ERR_CUDA = 7
SP24_ERR_DEVICE_TIMEOUT = 8
SP24_ERR_WORKSPACE = 9

BF16, E4M3, F32 = 0, 1, 2
SPARSE, DENSE = 0, 1
GEMM_W_STATIC = 1
GEMM_SINGLE_CTA = 2
GEMM_CTA_PAIR = 4
GEMM_AFTER_INDEPENDENT = 8


class Sp24Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_string(status), status))


class GemmArgs(ctypes.Structure):
    _fields_ = [
        ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int), ("tactic", ctypes.c_int),
        ("X", ctypes.c_void_p), ("ldx", ctypes.c_int64),
        ("W", ctypes.c_void_p), ("ldw", ctypes.c_int64),
        ("W_meta", ctypes.c_void_p),
        ("x_scales", ctypes.c_void_p), ("w_scales", ctypes.c_void_p),
        ("tile_dense_mask", ctypes.c_void_p), ("W_dense_tiles", ctypes.c_void_p),
        ("Y", ctypes.c_void_p), ("ldy", ctypes.c_int64),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("flags", ctypes.c_uint32),
    ]


class Nvfp4GemmArgs(ctypes.Structure):
    _fields_ = [
        ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
        ("tactic", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("X", ctypes.c_void_p), ("x_scales", ctypes.c_void_p), ("x_tensor_scale", ctypes.c_void_p),
        ("W", ctypes.c_void_p), ("W_meta", ctypes.c_void_p), ("w_scales", ctypes.c_void_p),
        ("w_tensor_scale", ctypes.c_void_p),
        ("Y", ctypes.c_void_p), ("ldy", ctypes.c_int64),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("flags", ctypes.c_uint32),
    ]


class QuantItem(ctypes.Structure):
    _fields_ = [
        ("src", ctypes.c_void_p), ("rows", ctypes.c_int64), ("K", ctypes.c_int64),
        ("ld", ctypes.c_int64), ("q", ctypes.c_void_p), ("scales", ctypes.c_void_p),
    ]


class TacticRecord(ctypes.Structure):
    _fields_ = [
        ("t_sparse_us", ctypes.c_double), ("t_dense_us", ctypes.c_double),
        ("t_sparse_min_us", ctypes.c_double), ("t_dense_min_us", ctypes.c_double),
        ("iters", ctypes.c_int32), ("eligible", ctypes.c_int32),
        ("selected", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("reason", ctypes.c_char * 64),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libsp24.so; raises if it is missing (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libsp24.so not found at %s: build it with "
                           "`python semi_structured_sparse_02_b200/build.py` "
                           "(the CUDA path is the only implementation)" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sigs = {
        "sp24_values_bytes": (ctypes.c_size_t, [I64, I64, I]),
        "sp24_meta_bytes": (ctypes.c_size_t, [I64, I64]),
        "sp24_prune_compress": (I, [P, I64, I64, I64, I, P, P, P, P, P, P]),
        "sp24_decompress": (I, [P, P, I64, I64, I, P, P]),
        "sp24_quantize_e4m3_rows": (I, [P, I64, I64, I64, P, P, P]),
        "sp24_quantize_e4m3_rows_grouped": (I, [ctypes.POINTER(QuantItem), I, P]),
        "sp24_gemm_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(GemmArgs)]),
        "sp24_gemm": (I, [ctypes.POINTER(GemmArgs), P]),
        "sp24_gemm_noalloc": (I, [ctypes.POINTER(GemmArgs), P]),
        "sp24_gemm_noalloc_max_scratch_bytes": (ctypes.c_size_t, []),
        "sp24_gemm_grouped": (I, [ctypes.POINTER(GemmArgs), I, P, ctypes.c_size_t, P]),
        "sp24_gemm_grouped_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(GemmArgs), I]),
        "sp24_gemm_workspace_state_bytes": (ctypes.c_size_t, [ctypes.POINTER(GemmArgs)]),
        "sp24_gemm_grouped_workspace_state_bytes": (ctypes.c_size_t, [ctypes.POINTER(GemmArgs), I]),
        "sp24_activations_workspace_bytes": (ctypes.c_size_t, [I64, I64]),
        "sp24_prune_compress_activations_fused": (I, [P, I64, I64, I64, P, I64, I64, P, I64, I,
                                                      P, P, P, ctypes.c_size_t, P]),
        "sp24_activations_e4m3_workspace_bytes": (ctypes.c_size_t, [I64, I64]),
        "sp24_energy_loss": (I, [P, I64, I64, I64, P, P, P]),
        "sp24_prune_compress_activations_fused_e4m3": (I, [P, I64, I64, I64, P, P, I64, I64, P, I64, I,
                                                           P, P, P, P, ctypes.c_size_t, P]),
        "sp24_select_tactic": (I, [ctypes.POINTER(GemmArgs), ctypes.POINTER(GemmArgs), I, I,
                                   ctypes.POINTER(TacticRecord), P]),
        "sp24_nvfp4_48_values_bytes": (ctypes.c_size_t, [I64, I64]),
        "sp24_nvfp4_48_meta_bytes": (ctypes.c_size_t, [I64, I64]),
        "sp24_nvfp4_codes_bytes": (ctypes.c_size_t, [I64, I64]),
        "sp24_nvfp4_scales_bytes": (ctypes.c_size_t, [I64, I64, I]),
        "sp24_prune_compress_nvfp4_48": (I, [P, I64, I64, I64, P, P, P, P, P]),
        "sp24_quantize_nvfp4": (I, [P, I64, I64, I64, I, P, P, P, P]),
        "sp24_gemm_nvfp4_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Nvfp4GemmArgs)]),
        "sp24_gemm_nvfp4": (I, [ctypes.POINTER(Nvfp4GemmArgs), P]),
        "sp24_gemm_nvfp4_grouped": (I, [ctypes.POINTER(Nvfp4GemmArgs), I, P, ctypes.c_size_t, P]),
        "sp24_gemm_nvfp4_grouped_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Nvfp4GemmArgs), I]),
        "sp24_prune_activations_in_gemm": (I, [P, I64, I64, I64, P, I64, I64, P, I64, I, P, P, P]),
        "sp24_status_string": (ctypes.c_char_p, [I]),
        "sp24_last_device_error": (I, []),
        "sp24_clear_device_error": (I, []),
        "sp24_set_wait_timeout_ns": (None, [ctypes.c_uint64]),
        "sp24_selftest_bounded_wait": (I, [ctypes.c_uint64, P]),
        "sp24_launch_count": (ctypes.c_uint64, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def header_functions() -> list:
    """Names of the functions include/sp24.h declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sp24_[a-z0-9_]+)\s*\(", src)))


def status_string(status: int) -> str:
    try:
        return lib().sp24_status_string(status).decode()
    except Exception:  # pragma: no cover
        return "status %d" % status


def _check(status: int, what: str):
    if status != SP24_OK:
        raise Sp24Error(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t in (torch.float8_e4m3fn, torch.uint8):
        return E4M3
    if t == torch.float32:
        return F32
    raise ValueError("unsupported dtype %s" % t)


# ---------------------------------------------------------------------------
# sizes
# ---------------------------------------------------------------------------

def values_bytes(rows: int, K: int, dtype: int) -> int:
    return lib().sp24_values_bytes(rows, K, dtype)


def meta_bytes(rows: int, K: int) -> int:
    return lib().sp24_meta_bytes(rows, K)


# ---------------------------------------------------------------------------
# prune / compress / decompress / quantize
# ---------------------------------------------------------------------------

def prune_compress(src: torch.Tensor, out_dtype: int, values: torch.Tensor, meta: torch.Tensor,
                   row_scales: Optional[torch.Tensor] = None,
                   tile_mask: Optional[torch.Tensor] = None,
                   dense_tiles: Optional[torch.Tensor] = None, stream=None):
    rows, K = src.shape
    _check(lib().sp24_prune_compress(_ptr(src), rows, K, src.stride(0), out_dtype, _ptr(values),
                                     _ptr(meta), _ptr(row_scales), _ptr(tile_mask), _ptr(dense_tiles),
                                     _stream(stream)), "sp24_prune_compress")


def decompress(values: torch.Tensor, meta: torch.Tensor, rows: int, K: int, dtype: int,
               dst: torch.Tensor, stream=None):
    _check(lib().sp24_decompress(_ptr(values), _ptr(meta), rows, K, dtype, _ptr(dst), _stream(stream)),
           "sp24_decompress")


def quantize_e4m3_rows(src: torch.Tensor, q: torch.Tensor, scales: torch.Tensor, stream=None):
    rows, K = src.shape
    _check(lib().sp24_quantize_e4m3_rows(_ptr(src), rows, K, src.stride(0), _ptr(q), _ptr(scales),
                                         _stream(stream)), "sp24_quantize_e4m3_rows")


class QuantGroup:
    """A prepared grouped per-token quantization (the item array and the
    tensors it points at are kept alive with it)."""

    def __init__(self, pairs):
        # pairs: list of (src bf16 [rows x K], q e4m3 [rows x K], scales fp32 [rows])
        self.items = (QuantItem * len(pairs))()
        self._keep = []
        for i, (src, q, sc) in enumerate(pairs):
            rows, K = src.shape
            self.items[i] = QuantItem(src.data_ptr(), rows, K, src.stride(0), q.data_ptr(),
                                      sc.data_ptr())
            self._keep += [src, q, sc]

    def __call__(self, stream=None):
        _check(lib().sp24_quantize_e4m3_rows_grouped(self.items, len(self.items), _stream(stream)),
               "sp24_quantize_e4m3_rows_grouped")


# ---------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------

def gemm_args(X: torch.Tensor, W: torch.Tensor, Y: torch.Tensor, K: int, tactic: int,
              W_meta: Optional[torch.Tensor] = None, x_scales: Optional[torch.Tensor] = None,
              w_scales: Optional[torch.Tensor] = None, tile_mask: Optional[torch.Tensor] = None,
              W_dense_tiles: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, flags: int = 0) -> GemmArgs:
    """Y [M x N] = X [M x K] * W^T; W is [N x K] (dense) or values [N x K/2]."""
    a = GemmArgs()
    a.M, a.N, a.K = X.shape[0], Y.shape[1], K
    a.in_dtype = dtype_code(X.dtype)
    a.out_dtype = dtype_code(Y.dtype)
    a.tactic = tactic
    a.X, a.ldx = X.data_ptr(), X.stride(0)
    a.W, a.ldw = W.data_ptr(), W.stride(0)
    a.W_meta = W_meta.data_ptr() if W_meta is not None else None
    a.x_scales = x_scales.data_ptr() if x_scales is not None else None
    a.w_scales = w_scales.data_ptr() if w_scales is not None else None
    a.tile_dense_mask = tile_mask.data_ptr() if tile_mask is not None else None
    a.W_dense_tiles = W_dense_tiles.data_ptr() if W_dense_tiles is not None else None
    a.Y, a.ldy = Y.data_ptr(), Y.stride(0)
    a.flags = flags
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    # the argument block holds raw pointers: keep the tensors alive with it
    a._keep = [X, W, Y, W_meta, x_scales, w_scales, tile_mask, W_dense_tiles, workspace]
    return a


def set_workspace(args: GemmArgs, workspace: Optional[torch.Tensor]):
    """Attach a workspace tensor (kept alive with the argument block)."""
    if workspace is None:
        args.workspace, args.workspace_bytes = None, 0
        return
    args.workspace = workspace.data_ptr()
    args.workspace_bytes = workspace.numel() * workspace.element_size()
    keep = getattr(args, "_keep", [])
    keep.append(workspace)
    args._keep = keep


def gemm_workspace_bytes(args: GemmArgs) -> int:
    return lib().sp24_gemm_workspace_bytes(ctypes.byref(args))


def gemm_workspace_state_bytes(args: GemmArgs) -> int:
    return lib().sp24_gemm_workspace_state_bytes(ctypes.byref(args))


def gemm(args: GemmArgs, stream=None):
    _check(lib().sp24_gemm(ctypes.byref(args), _stream(stream)), "sp24_gemm")


def gemm_noalloc(args: GemmArgs, stream=None):
    """sp24_gemm without any device allocation: stream-K scratch comes from a
    fixed array in the library (args.workspace is ignored)."""
    _check(lib().sp24_gemm_noalloc(ctypes.byref(args), _stream(stream)), "sp24_gemm_noalloc")


class GemmGroup:
    """Up to 16 independent GEMMs run by one sp24_gemm_grouped launch.

    The argument array is built once; `workspace` (zero-filled, reusable
    across calls on one stream) is allocated here when the group's schedule
    needs one.  The GemmArgs objects (and the tensors they keep alive) are
    held for the group's lifetime."""

    def __init__(self, args_list, workspace: Optional[torch.Tensor] = None,
                 allocate_workspace: bool = True, after_independent: bool = False):
        self.args_list = list(args_list)
        n = len(self.args_list)
        self.arr = (GemmArgs * n)(*self.args_list)
        if after_independent:
            # the launch before this one in the stream is an independent GEMM
            # group (GEMM_AFTER_INDEPENDENT); set on this group's copies only
            for i in range(n):
                self.arr[i].flags |= GEMM_AFTER_INDEPENDENT
        self.n = n
        need = lib().sp24_gemm_grouped_workspace_bytes(self.arr, n)
        if workspace is None and need > 0 and allocate_workspace:
            workspace = torch.zeros(need, dtype=torch.uint8, device=torch.cuda.current_device())
        self.workspace = workspace
        self.ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()

    def workspace_bytes(self) -> int:
        return lib().sp24_gemm_grouped_workspace_bytes(self.arr, self.n)

    def workspace_state_bytes(self) -> int:
        return lib().sp24_gemm_grouped_workspace_state_bytes(self.arr, self.n)

    def __call__(self, stream=None):
        _check(lib().sp24_gemm_grouped(self.arr, self.n, _ptr(self.workspace), self.ws_bytes,
                                       _stream(stream)), "sp24_gemm_grouped")


def m_class(M: int) -> int:
    """The token-count class of a GEMM (1-16, 17-32, 33-64, >64): the token
    tile width it runs with.  A grouped launch may mix classes; it is built
    for the widest."""
    return 16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128


def gemm_grouped(args_list, workspace: Optional[torch.Tensor] = None, stream=None) -> GemmGroup:
    """Runs the GEMMs of args_list in one grouped launch; returns the group
    so that it can be called again."""
    g = GemmGroup(args_list, workspace)
    g(stream)
    return g


def gemm_noalloc_max_scratch_bytes() -> int:
    return lib().sp24_gemm_noalloc_max_scratch_bytes()


def activations_workspace_bytes(M: int, K: int) -> int:
    return lib().sp24_activations_workspace_bytes(M, K)


def prune_compress_activations_fused(X: torch.Tensor, W: torch.Tensor, Y: torch.Tensor,
                                     x_values: Optional[torch.Tensor] = None,
                                     x_meta: Optional[torch.Tensor] = None,
                                     workspace: Optional[torch.Tensor] = None, stream=None):
    M, K = X.shape
    N = W.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sp24_prune_compress_activations_fused(
        _ptr(X), M, K, X.stride(0), _ptr(W), N, W.stride(0), _ptr(Y), Y.stride(0),
        dtype_code(Y.dtype), _ptr(x_values), _ptr(x_meta), _ptr(workspace), ws_bytes,
        _stream(stream)), "sp24_prune_compress_activations_fused")


def prune_activations_in_gemm(X: torch.Tensor, W: torch.Tensor, Y: torch.Tensor,
                              x_values: Optional[torch.Tensor] = None, x_meta: Optional[torch.Tensor] = None,
                              stream=None):
    """Y = prune(X) * W^T with the prune done inside the GEMM kernel (X, W
    bf16; x_values / x_meta optionally receive the compressed X)."""
    M, K = X.shape
    N = W.shape[0]
    _check(lib().sp24_prune_activations_in_gemm(
        _ptr(X), M, K, X.stride(0), _ptr(W), N, W.stride(0), _ptr(Y), Y.stride(0), dtype_code(Y.dtype),
        _ptr(x_values), _ptr(x_meta), _stream(stream)), "sp24_prune_activations_in_gemm")


def energy_loss(src: torch.Tensor, row_share: Optional[torch.Tensor] = None,
                sums: Optional[torch.Tensor] = None, stream=None):
    """2:4 energy loss of a bf16 matrix: per-row share (fp64 [rows]) and/or the
    tensor's dropped and total energy (fp64 [2])."""
    rows, K = src.shape
    _check(lib().sp24_energy_loss(_ptr(src), rows, K, src.stride(0), _ptr(row_share), _ptr(sums),
                                  _stream(stream)), "sp24_energy_loss")


def activations_e4m3_workspace_bytes(M: int, K: int) -> int:
    return lib().sp24_activations_e4m3_workspace_bytes(M, K)


def prune_compress_activations_fused_e4m3(X: torch.Tensor, Wq: torch.Tensor, w_scales: torch.Tensor,
                                          Y: torch.Tensor, x_values: Optional[torch.Tensor] = None,
                                          x_meta: Optional[torch.Tensor] = None,
                                          x_scales: Optional[torch.Tensor] = None,
                                          workspace: Optional[torch.Tensor] = None, stream=None):
    """X bf16 [M x K] pruned 2:4 and cast to e4m3 per token each call, then
    Y = X_sparse * Wq^T with Wq e4m3 [N x K] (per-channel scales)."""
    M, K = X.shape
    N = Wq.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sp24_prune_compress_activations_fused_e4m3(
        _ptr(X), M, K, X.stride(0), _ptr(Wq), _ptr(w_scales), N, Wq.stride(0), _ptr(Y), Y.stride(0),
        dtype_code(Y.dtype), _ptr(x_values), _ptr(x_meta), _ptr(x_scales), _ptr(workspace), ws_bytes,
        _stream(stream)), "sp24_prune_compress_activations_fused_e4m3")


def select_tactic(sparse_args: Optional[GemmArgs], dense_args: GemmArgs, warmup: int = 3,
                  iters: int = 10, stream=None) -> dict:
    rec = TacticRecord()
    sp = ctypes.byref(sparse_args) if sparse_args is not None else None
    _check(lib().sp24_select_tactic(sp, ctypes.byref(dense_args), warmup, iters, ctypes.byref(rec),
                                    _stream(stream)), "sp24_select_tactic")
    return dict(t_sparse_us=rec.t_sparse_us, t_dense_us=rec.t_dense_us,
                t_sparse_min_us=rec.t_sparse_min_us, t_dense_min_us=rec.t_dense_min_us,
                iters=rec.iters, eligible=bool(rec.eligible),
                selected="sparse" if rec.selected == SPARSE else "dense",
                reason=rec.reason.decode())


# ---------------------------------------------------------------------------
# pairwise 4:8 sparse NVFP4 and dense NVFP4
# ---------------------------------------------------------------------------

def nvfp4_48_values_bytes(rows: int, K: int) -> int:
    return lib().sp24_nvfp4_48_values_bytes(rows, K)


def nvfp4_48_meta_bytes(rows: int, K: int) -> int:
    return lib().sp24_nvfp4_48_meta_bytes(rows, K)


def nvfp4_codes_bytes(rows: int, K: int) -> int:
    return lib().sp24_nvfp4_codes_bytes(rows, K)


def nvfp4_scales_bytes(rows: int, K: int, block: int) -> int:
    return lib().sp24_nvfp4_scales_bytes(rows, K, block)


def prune_compress_nvfp4_48(src: torch.Tensor, values: torch.Tensor, meta: torch.Tensor, scales: torch.Tensor,
                            tensor_scale: torch.Tensor, stream=None):
    """Pairwise 4:8 prune + NVFP4 cast of a bf16 matrix: values [rows, K/4],
    metadata image, scale image (per 32 positions), tensor scale (fp32 [1])."""
    rows, K = src.shape
    _check(lib().sp24_prune_compress_nvfp4_48(_ptr(src), rows, K, src.stride(0), _ptr(values), _ptr(meta),
                                              _ptr(scales), _ptr(tensor_scale), _stream(stream)),
           "sp24_prune_compress_nvfp4_48")


def quantize_nvfp4(src: torch.Tensor, block: int, codes: torch.Tensor, scales: torch.Tensor,
                   tensor_scale: torch.Tensor, stream=None):
    """Dense NVFP4 cast of a bf16 matrix, one scale per `block` (16 or 32)."""
    rows, K = src.shape
    _check(lib().sp24_quantize_nvfp4(_ptr(src), rows, K, src.stride(0), block, _ptr(codes), _ptr(scales),
                                     _ptr(tensor_scale), _stream(stream)), "sp24_quantize_nvfp4")


def nvfp4_gemm_args(X: torch.Tensor, x_scales: torch.Tensor, x_ts: torch.Tensor, W: torch.Tensor,
                    w_scales: torch.Tensor, w_ts: torch.Tensor, Y: torch.Tensor, K: int, tactic: int,
                    W_meta: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    flags: int = 0) -> Nvfp4GemmArgs:
    """Y [M x N] = X * W^T with NVFP4 operands: X codes [M, K/2] (+ scale
    image, tensor scale); W sparse values [N, K/4] + metadata image, or dense
    codes [N, K/2] (+ scale image, tensor scale)."""
    a = Nvfp4GemmArgs()
    a.M, a.N, a.K = X.shape[0], Y.shape[1], K
    a.tactic = tactic
    a.out_dtype = dtype_code(Y.dtype)
    a.X, a.x_scales, a.x_tensor_scale = X.data_ptr(), x_scales.data_ptr(), x_ts.data_ptr()
    a.W, a.w_scales, a.w_tensor_scale = W.data_ptr(), w_scales.data_ptr(), w_ts.data_ptr()
    a.W_meta = W_meta.data_ptr() if W_meta is not None else None
    a.Y, a.ldy = Y.data_ptr(), Y.stride(0)
    a.flags = flags
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a._keep = [X, x_scales, x_ts, W, w_scales, w_ts, W_meta, Y, workspace]
    return a


def gemm_nvfp4_workspace_bytes(args: Nvfp4GemmArgs) -> int:
    return lib().sp24_gemm_nvfp4_workspace_bytes(ctypes.byref(args))


def gemm_nvfp4(args: Nvfp4GemmArgs, stream=None):
    _check(lib().sp24_gemm_nvfp4(ctypes.byref(args), _stream(stream)), "sp24_gemm_nvfp4")


class Nvfp4GemmGroup:
    """Up to 16 independent NVFP4 GEMMs (one tactic, one output type) run by
    one sp24_gemm_nvfp4_grouped launch; `workspace` (zero-filled, reusable
    across calls on one stream) is allocated here when the schedule needs
    one.  The argument objects are held for the group's lifetime."""

    def __init__(self, args_list, workspace: Optional[torch.Tensor] = None):
        self.args_list = list(args_list)
        self.n = len(self.args_list)
        self.arr = (Nvfp4GemmArgs * self.n)(*self.args_list)
        need = lib().sp24_gemm_nvfp4_grouped_workspace_bytes(self.arr, self.n)
        if workspace is None and need > 0:
            workspace = torch.zeros(need, dtype=torch.uint8, device=torch.cuda.current_device())
        self.workspace = workspace
        self.ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()

    def workspace_bytes(self) -> int:
        return lib().sp24_gemm_nvfp4_grouped_workspace_bytes(self.arr, self.n)

    def __call__(self, stream=None):
        _check(lib().sp24_gemm_nvfp4_grouped(self.arr, self.n, _ptr(self.workspace), self.ws_bytes,
                                             _stream(stream)), "sp24_gemm_nvfp4_grouped")


# ---------------------------------------------------------------------------
# status
# ---------------------------------------------------------------------------

def last_device_error() -> int:
    return lib().sp24_last_device_error()


def clear_device_error() -> int:
    return lib().sp24_clear_device_error()


def set_wait_timeout_ns(ns: int):
    lib().sp24_set_wait_timeout_ns(ns)


def selftest_bounded_wait(timeout_ns: int, stream=None) -> int:
    return lib().sp24_selftest_bounded_wait(timeout_ns, _stream(stream))


def launch_count() -> int:
    return lib().sp24_launch_count()
