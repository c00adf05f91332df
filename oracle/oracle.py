"""Python face of the CPU oracle (sp24_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It never
imports the CUDA package and the CUDA package never imports it.

Every function here is a thin numpy/ctypes wrapper around the C oracle, plus
the few definitions that are plain arithmetic on numbers (dequantization,
the tactic rule and the coverage ratio), each citing the page it restates.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sp24_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with plain gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        sig = {
            "orc_prune_group": (ctypes.c_int, [P, P, P]),
            "orc_prune_compress_bf16": (None, [P, I64, I64, I64, P, P, P]),
            "orc_prune_compress_bf16_hybrid": (None, [P, I64, I64, I64, P, P, P, P]),
            "orc_prune_compress_e4m3": (None, [P, I64, I64, I64, P, P, P, P, P]),
            "orc_decompress": (None, [P, P, I64, I64, ctypes.c_int, P]),
            "orc_e4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e4m3_encode": (ctypes.c_uint8, [ctypes.c_double]),
            "orc_e4m3_encode_array": (None, [P, I64, P]),
            "orc_e4m3_row_scale": (None, [ctypes.c_float, P, P]),
            "orc_quantize_rows_e4m3": (None, [P, I64, I64, I64, P, P]),
            "orc_meta_image": (None, [P, I64, I64, ctypes.c_int, P, P]),
            "orc_gemm_f64": (None, [P, P, I64, I64, I64, P, P]),
            "orc_gemm_f64_sampled": (None, [P, P, I64, P, P, I64, P, P]),
            "orc_gemm_sparse_f64": (None, [P, I64, I64, P, P, I64, P]),
            "orc_bf16_to_double": (ctypes.c_double, [ctypes.c_uint16]),
            "orc_energy_loss": (None, [P, I64, I64, I64, P, P]),
            "orc_e2m1_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e2m1_encode": (ctypes.c_uint8, [ctypes.c_double]),
            "orc_prune_pairs8": (ctypes.c_int, [P, P, P]),
            "orc_prune_pairs_bf16": (None, [P, I64, I64, I64, P]),
            "orc_nvfp4_tensor_scale": (ctypes.c_float, [ctypes.c_float]),
            "orc_nvfp4_block_code": (ctypes.c_uint8, [ctypes.c_float, ctypes.c_float]),
            "orc_nvfp4_code": (ctypes.c_uint8, [ctypes.c_float, ctypes.c_uint8, ctypes.c_float]),
            "orc_nvfp4_48_compress": (None, [P, I64, I64, I64, P, P, P, P]),
            "orc_nvfp4_48_dequant": (None, [P, P, P, ctypes.c_float, I64, I64, P]),
            "orc_nvfp4_quantize_blocks": (None, [P, I64, I64, I64, ctypes.c_int, P, P, P]),
            "orc_nvfp4_dequant_blocks": (None, [P, P, ctypes.c_float, I64, I64, ctypes.c_int, P]),
            "orc_energy_loss_48": (None, [P, I64, I64, I64, P, P]),
            "orc_nvfp4_48_meta_image": (None, [P, I64, I64, P]),
            "orc_nvfp4_scale_image": (None, [P, I64, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------------------
# exact number conversions
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (bf16 = top 16 bits of an fp32)."""
    u = bits.astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


_E4M3_TABLE = None


def e4m3_table() -> np.ndarray:
    """Value of each of the 256 E4M3 codes, from the oracle's own decoder."""
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        L = lib()
        _E4M3_TABLE = np.array([L.orc_e4m3_decode(i) for i in range(256)], dtype=np.float64)
    return _E4M3_TABLE


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return e4m3_table()[codes.astype(np.int64)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even, saturating E4M3 encoding of fp32 values."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32).astype(np.float64))
    q = np.empty(x.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_p(x), x.size, _p(q))
    return q


def e4m3_row_scale(amax: float):
    s = ctypes.c_float()
    i = ctypes.c_float()
    lib().orc_e4m3_row_scale(ctypes.c_float(amax), ctypes.byref(s), ctypes.byref(i))
    return s.value, i.value


# ---------------------------------------------------------------------------
# prune / compress / decompress
# ---------------------------------------------------------------------------

def prune_group(v_bits: Sequence[int]):
    """(nibble, i0, i1) for one group of four bf16 bit patterns."""
    a = np.ascontiguousarray(np.asarray(v_bits, dtype=np.uint16))
    i0 = ctypes.c_int()
    i1 = ctypes.c_int()
    nib = lib().orc_prune_group(_p(a), ctypes.byref(i0), ctypes.byref(i1))
    return nib, i0.value, i1.value


def prune_compress_bf16(W_bits: np.ndarray):
    """Return (pruned [rows,K], values [rows,K/2], meta_canon [rows,K/8])."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    assert K % 4 == 0
    pruned = np.empty((rows, K), np.uint16)
    values = np.empty((rows, K // 2), np.uint16)
    meta = np.empty((rows, K // 8), np.uint8)
    lib().orc_prune_compress_bf16(_p(W), rows, K, K, _p(pruned), _p(values), _p(meta))
    return pruned, values, meta


def prune_compress_bf16_hybrid(W_bits: np.ndarray, mask: np.ndarray):
    """Hybrid bf16: (values, meta_canon, dense_out); dense_out is the hybrid
    matrix in dense form (dense tiles unpruned, sparse tiles pruned)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    values = np.empty((rows, K // 2), np.uint16)
    meta = np.empty((rows, K // 8), np.uint8)
    dense = np.zeros((rows, K), np.uint16)
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    lib().orc_prune_compress_bf16_hybrid(_p(W), rows, K, K, _p(m), _p(values), _p(meta), _p(dense))
    return values, meta, dense


def prune_compress_e4m3(W_bits: np.ndarray, mask: Optional[np.ndarray] = None):
    """Return (values_q [rows,K/2], meta_canon, scales [rows] f32, dense_q [rows,K]).
    With a mask, dense_q is the hybrid matrix in dense form (dense tiles
    quantized unpruned, sparse tiles their kept codes and zero bytes); without
    one it stays zero."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    values = np.empty((rows, K // 2), np.uint8)
    meta = np.empty((rows, K // 8), np.uint8)
    scales = np.empty((rows,), np.float32)
    dense = np.zeros((rows, K), np.uint8)
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    lib().orc_prune_compress_e4m3(_p(W), rows, K, K, _p(m), _p(values), _p(meta),
                                  _p(scales), _p(dense))
    return values, meta, scales, dense


def energy_loss(W_bits: np.ndarray):
    """2:4 energy loss [P4 sections 1 and 5]: (per-row dropped energy, per-row
    total energy, per-row share, tensor share).  A row (or tensor) with no
    energy has share 0 (reading)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    dropped = np.empty(rows, np.float64)
    total = np.empty(rows, np.float64)
    lib().orc_energy_loss(_p(W), rows, K, K, _p(dropped), _p(total))
    share = np.where(total > 0, dropped / np.where(total > 0, total, 1.0), 0.0)
    t = total.sum()
    return dropped, total, share, (dropped.sum() / t if t > 0 else 0.0)


def decompress(values: np.ndarray, meta_canon: np.ndarray, rows: int, K: int) -> np.ndarray:
    values = np.ascontiguousarray(values)
    eb = values.dtype.itemsize
    out = np.empty((rows, K), values.dtype)
    lib().orc_decompress(_p(values), _p(np.ascontiguousarray(meta_canon)), rows, K, eb, _p(out))
    return out


def meta_image(meta_canon: np.ndarray, rows: int, K: int, is_8bit: bool,
               mask: Optional[np.ndarray] = None) -> np.ndarray:
    RB = (rows + 127) // 128
    img = np.empty((RB * (K // 128) * 2048,), np.uint8)
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    lib().orc_meta_image(_p(np.ascontiguousarray(meta_canon)), rows, K, int(is_8bit), _p(m), _p(img))
    return img


def quantize_rows_e4m3(X_bits: np.ndarray):
    """Per-row (per-token) E4M3: (q [rows,K], scales [rows])."""
    X = np.ascontiguousarray(X_bits, dtype=np.uint16)
    rows, K = X.shape
    q = np.empty((rows, K), np.uint8)
    s = np.empty((rows,), np.float32)
    lib().orc_quantize_rows_e4m3(_p(X), rows, K, K, _p(q), _p(s))
    return q, s


# ---------------------------------------------------------------------------
# GEMM (fp64)
# ---------------------------------------------------------------------------

def gemm_f64(X: np.ndarray, W: np.ndarray):
    """Y = X W^T and A = |X| |W|^T elementwise-product sums, both fp64."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = X.shape
    N = W.shape[0]
    Y = np.empty((M, N), np.float64)
    A = np.empty((M, N), np.float64)
    lib().orc_gemm_f64(_p(X), _p(W), M, N, K, _p(Y), _p(A))
    return Y, A


def gemm_f64_sampled(X: np.ndarray, W: np.ndarray, ms: np.ndarray, ns: np.ndarray):
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    Y = np.empty(ms.shape, np.float64)
    A = np.empty(ms.shape, np.float64)
    lib().orc_gemm_f64_sampled(_p(X), _p(W), X.shape[1], _p(ms), _p(ns), ms.size, _p(Y), _p(A))
    return Y, A


def gemm_sparse_f64(X: np.ndarray, wvals: np.ndarray, meta_canon: np.ndarray):
    X = np.ascontiguousarray(X, dtype=np.float64)
    wv = np.ascontiguousarray(wvals, dtype=np.float64)
    M, K = X.shape
    N = wv.shape[0]
    Y = np.empty((M, N), np.float64)
    lib().orc_gemm_sparse_f64(_p(X), M, K, _p(wv), _p(np.ascontiguousarray(meta_canon)), N, _p(Y))
    return Y


def within_tolerance(y_gpu: np.ndarray, y_ref: np.ndarray, a_ref: np.ndarray,
                     rel: float = 2e-3, abs_: float = 1e-6) -> np.ndarray:
    """Per-element pass mask of |y_gpu - y| <= rel * sum_k |x_k w_k| + abs."""
    return np.abs(y_gpu.astype(np.float64) - y_ref) <= rel * a_ref + abs_


# ---------------------------------------------------------------------------
# tactic rule and coverage  [P1 "Sparse Tactic Audit": latency is the sole
# criterion; Sparse GPU-Time Coverage = time of selected sparse kernels over
# total GPU time]
# ---------------------------------------------------------------------------

def select_tactic(t_sparse_samples, t_dense_samples):
    """'sparse' iff median sparse time < median dense time (a tie -> dense)."""
    ts = float(np.median(np.asarray(t_sparse_samples, dtype=np.float64)))
    td = float(np.median(np.asarray(t_dense_samples, dtype=np.float64)))
    return ("sparse" if ts < td else "dense"), ts, td


def sparse_gpu_time_coverage(selected_times):
    """selected_times: iterable of (tactic, time) for the kernels that ran."""
    tot = sum(t for _, t in selected_times)
    sp = sum(t for tac, t in selected_times if tac == "sparse")
    return sp / tot if tot > 0 else 0.0


# ---------------------------------------------------------------------------
# pairwise 4:8 sparsity with NVFP4 values  [P4 section 2 "Quantization";
# section 6.2 "What pairwise 4:8 costs on Blackwell"]
# ---------------------------------------------------------------------------

def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """Values of E2M1 codes (low 4 bits: sign, two exponent bits, mantissa)."""
    table = np.array([lib().orc_e2m1_decode(c) for c in range(16)], np.float64)
    return table[np.asarray(codes, dtype=np.uint8) & 0xF]


def e2m1_encode(x) -> np.ndarray:
    """Round to nearest E2M1 (ties to the even code, saturating to 6)."""
    xs = np.asarray(x, dtype=np.float64)
    return np.array([lib().orc_e2m1_encode(float(v)) for v in xs.ravel()], np.uint8).reshape(xs.shape)


def prune_pairs8(v_bits: Sequence[int]):
    """(nibble, p0, p1) for one group of eight bf16 bit patterns."""
    a = np.ascontiguousarray(np.asarray(v_bits, dtype=np.uint16))
    p0 = ctypes.c_int()
    p1 = ctypes.c_int()
    nib = lib().orc_prune_pairs8(_p(a), ctypes.byref(p0), ctypes.byref(p1))
    return nib, p0.value, p1.value


def prune_pairs_bf16(W_bits: np.ndarray) -> np.ndarray:
    """The pairwise 4:8 pruned matrix (bf16 bits, dropped positions +0)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    out = np.empty((rows, K), np.uint16)
    lib().orc_prune_pairs_bf16(_p(W), rows, K, K, _p(out))
    return out


def nvfp4_tensor_scale(amax: float) -> float:
    return float(lib().orc_nvfp4_tensor_scale(ctypes.c_float(amax)))


def nvfp4_block_code(amax_b: float, s_t: float) -> int:
    return int(lib().orc_nvfp4_block_code(ctypes.c_float(amax_b), ctypes.c_float(s_t)))


def nvfp4_code(v: float, b: int, s_t: float) -> int:
    return int(lib().orc_nvfp4_code(ctypes.c_float(v), ctypes.c_uint8(b), ctypes.c_float(s_t)))


def nvfp4_48_compress(W_bits: np.ndarray):
    """Sparse pairwise 4:8 NVFP4 operand: (values [rows, K/4] packed codes,
    meta [rows, K/16] canonical nibbles, block scales [rows, K/32] E4M3
    codes, tensor scale)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    assert K % 32 == 0
    values = np.empty((rows, K // 4), np.uint8)
    meta = np.empty((rows, K // 16), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    st = ctypes.c_float()
    lib().orc_nvfp4_48_compress(_p(W), rows, K, K, _p(values), _p(meta), _p(scales), ctypes.byref(st))
    return values, meta, scales, float(st.value)


def nvfp4_48_dequant(values, meta, scales, tensor_scale: float, rows: int, K: int) -> np.ndarray:
    out = np.empty((rows, K), np.float64)
    lib().orc_nvfp4_48_dequant(_p(np.ascontiguousarray(values)), _p(np.ascontiguousarray(meta)),
                               _p(np.ascontiguousarray(scales)), ctypes.c_float(tensor_scale), rows, K, _p(out))
    return out


def nvfp4_quantize(W_bits: np.ndarray, block: int = 16):
    """Dense NVFP4: (codes [rows, K/2] packed, block scales [rows, K/block],
    tensor scale).  block 16 is dense NVFP4; block 32 is the dense operand of
    the sparse block-scaled GEMM (one scale per 32 positions of K)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    assert K % block == 0
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // block), np.uint8)
    st = ctypes.c_float()
    lib().orc_nvfp4_quantize_blocks(_p(W), rows, K, K, block, _p(codes), _p(scales), ctypes.byref(st))
    return codes, scales, float(st.value)


def nvfp4_dequant(codes, scales, tensor_scale: float, rows: int, K: int, block: int = 16) -> np.ndarray:
    out = np.empty((rows, K), np.float64)
    lib().orc_nvfp4_dequant_blocks(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                                   ctypes.c_float(tensor_scale), rows, K, block, _p(out))
    return out


def nvfp4_48_meta_image(meta: np.ndarray, rows: int, K: int) -> np.ndarray:
    """The 4:8 metadata image the block-scaled GEMM copies to tensor memory
    (layout spec): 2048-byte chunks of 128 rows x 256 positions of K."""
    assert K % 256 == 0
    out = np.empty(((rows + 127) // 128) * (K // 256) * 2048, np.uint8)
    lib().orc_nvfp4_48_meta_image(_p(np.ascontiguousarray(meta, dtype=np.uint8)), rows, K, _p(out))
    return out


def nvfp4_scale_image(scales: np.ndarray, rows: int) -> np.ndarray:
    """The block-scale image (layout spec): 512-byte chunks of 128 rows x 4
    consecutive scale blocks."""
    sc = np.ascontiguousarray(scales, dtype=np.uint8)
    nblk = sc.shape[1]
    assert nblk % 4 == 0
    out = np.empty(((rows + 127) // 128) * 128 * nblk, np.uint8)
    lib().orc_nvfp4_scale_image(_p(sc), rows, nblk, _p(out))
    return out


def energy_loss_48(W_bits: np.ndarray):
    """Pairwise 4:8 energy loss: (per-row dropped, per-row total, per-row
    share, tensor share), as energy_loss for 2:4."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    rows, K = W.shape
    dropped = np.empty(rows, np.float64)
    total = np.empty(rows, np.float64)
    lib().orc_energy_loss_48(_p(W), rows, K, K, _p(dropped), _p(total))
    share = np.where(total > 0, dropped / np.where(total > 0, total, 1.0), 0.0)
    tensor = float(dropped.sum() / total.sum()) if total.sum() > 0 else 0.0
    return dropped, total, share, tensor
