"""Shared helpers for the GPU parity tests: moving seeded inputs to the
device and computing the oracle's expected values from the same inputs.
No expected value is ever computed from a CUDA output."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as orc
from semi_structured_sparse_02_b200 import sp24


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).copy()).cuda()


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.uint8).cpu().numpy()


def f32_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy().view(np.uint32)


class OracleSparseW:
    """The oracle's compressed form of W and its dequantized dense value."""

    def __init__(self, W_bits: np.ndarray, e4m3: bool, mask: np.ndarray | None = None):
        N, K = W_bits.shape
        self.N, self.K, self.e4m3 = N, K, e4m3
        if e4m3:
            vq, canon, s, dq = orc.prune_compress_e4m3(W_bits, mask)
            self.values, self.canon, self.scales, self.dense = vq, canon, s, dq
            self.image = orc.meta_image(canon, N, K, True, mask)
            w = orc.e4m3_decode(orc.decompress(vq, canon, N, K))
            if mask is not None:
                dm = np.kron(mask, np.ones((128, 128), np.uint8))[:N, :K].astype(bool)
                w = np.where(dm, orc.e4m3_decode(dq), w)
            self.W_hat = w * s.astype(np.float64)[:, None]
        else:
            if mask is not None:
                vals, canon, dense = orc.prune_compress_bf16_hybrid(W_bits, mask)
                self.values, self.canon, self.dense = vals, canon, dense
                pruned = orc.decompress(vals, canon, N, K)
                dm = np.kron(mask, np.ones((128, 128), np.uint8))[:N, :K].astype(bool)
                self.W_hat = np.where(dm, orc.bf16_bits_to_f64(dense), orc.bf16_bits_to_f64(pruned))
            else:
                pruned, vals, canon = orc.prune_compress_bf16(W_bits)
                self.values, self.canon, self.dense = vals, canon, None
                self.W_hat = orc.bf16_bits_to_f64(pruned)
            self.scales = None
            self.image = orc.meta_image(canon, N, K, False, mask)


def oracle_x(X_bits: np.ndarray, e4m3: bool):
    """(device-ready operand, scales, dequantized fp64 X) from the oracle."""
    if e4m3:
        q, s = orc.quantize_rows_e4m3(X_bits)
        return q, s, orc.e4m3_decode(q) * s.astype(np.float64)[:, None]
    return X_bits, None, orc.bf16_bits_to_f64(X_bits)


def bf16_half_ulp(y: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |y| (the largest error of rounding a value of
    that binade to bf16: 8 significant bits, so 2^-8 relative at the bottom
    of a binade)."""
    m = np.abs(np.asarray(y, dtype=np.float64))
    e = np.floor(np.log2(np.where(m > 0, m, 1.0)))
    return np.where(m > 0, np.exp2(e - 8), 0.0)


def check_tolerance(y_gpu: np.ndarray, y: np.ndarray, a: np.ndarray, what: str = ""):
    """|y_gpu - y| <= 2e-3 * a + 1e-6 (the GEMM's bound on its fp32 result),
    plus, when the output was stored as bf16, the rounding of that cast:
    half a bf16 spacing of the stored value.  A bf16 output is recognized by
    every value's fp32 image having zero low 16 bits."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    f32 = y_gpu.astype(np.float32)
    if y_gpu.size and np.all((f32.view(np.uint32) & 0xFFFF) == 0):
        ok = np.abs(y_gpu - y) <= 2e-3 * a + 1e-6 + bf16_half_ulp(y_gpu)
    else:
        ok = orc.within_tolerance(y_gpu, y, a)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        det = ["(%s) gpu=%r ref=%r a=%r" % (tuple(i), float(y_gpu[tuple(i)]), float(y[tuple(i)]),
                                           float(a[tuple(i)])) for i in idx]
        raise AssertionError("%s: %d/%d outside 2e-3*a+1e-6: %s" % (what, (~ok).sum(), ok.size,
                                                                   "; ".join(det)))


def workspace_for(args: sp24.GemmArgs) -> torch.Tensor | None:
    n = sp24.gemm_workspace_bytes(args)
    if n == 0:
        return None
    return torch.zeros(n, dtype=torch.uint8, device="cuda")
