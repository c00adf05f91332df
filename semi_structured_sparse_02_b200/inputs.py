"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method: it only draws random numbers
with numpy's ``default_rng(seed)``, rounds fp32 draws to bf16 bit patterns,
and names the workload shapes.  Both the CUDA path and the CPU oracle take
their inputs from here.

Workloads (the shapes of the pages' LLM linear layers; there is no dataset):
  tiny      X[16 x 256] ~ N(0,1), W[256 x 256] ~ N(0, 0.02^2)
  decode    (N,K) in {(5120,5120),(25600,5120),(5120,25600),(10240,5120)},
            M in {1,8,32,128}; W ~ N(0,0.02^2), X ~ N(0,1)
  prefill   M in {2048,8192,16384} x (N,K) in {(4096,4096),(12288,4096),
            (4096,12288),(6144,4096)}; W ~ N(0,0.02^2) with 0.1% of the
            elements (seeded permutation) multiplied by 20; X ~ N(0,1)
  act       X[8192 x 4096] Student-t nu=3, W[12288 x 4096] ~ N(0,0.02^2)
  hybrid    one 8B-shape block: QKV (6144,4096), O (4096,4096), gate/up
            (24576,4096), down (4096,12288); M in {1,16,256,4096}; 25% of
            the 128 x 128 tiles dense, chosen by seeded permutation
"""
from __future__ import annotations

import numpy as np
import torch

DECODE_NK = [(5120, 5120), (25600, 5120), (5120, 25600), (10240, 5120)]
DECODE_M = [1, 8, 32, 128]
PREFILL_M = [2048, 8192, 16384]
PREFILL_NK = [(4096, 4096), (12288, 4096), (4096, 12288), (6144, 4096)]
ACT_SHAPE = dict(M=8192, K=4096, N=12288)
HYBRID_NK = [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 24576, 4096),
             ("down", 4096, 12288)]
HYBRID_M = [1, 16, 256, 4096]
HYBRID_TILE = 128
HYBRID_DENSE_FRACTION = 0.25


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 draws to bf16 (round-to-nearest-even) and return the bits."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def normal_bf16(shape, std: float, seed: int) -> np.ndarray:
    return to_bf16_bits(rng(seed).normal(0.0, std, size=shape).astype(np.float32))


def weights_with_outliers(N: int, K: int, seed: int, std: float = 0.02,
                          frac: float = 0.001, mult: float = 20.0) -> np.ndarray:
    """W ~ N(0, std^2); a seeded permutation picks round(frac*N*K) elements x mult."""
    g = rng(seed)
    w = g.normal(0.0, std, size=(N, K)).astype(np.float32)
    n_out = int(round(frac * N * K))
    idx = g.permutation(N * K)[:n_out]
    w.reshape(-1)[idx] *= np.float32(mult)
    return to_bf16_bits(w)


def student_t_bf16(shape, nu: float, seed: int) -> np.ndarray:
    return to_bf16_bits(rng(seed).standard_t(nu, size=shape).astype(np.float32))


def hybrid_mask(rows: int, K: int, seed: int,
                fraction: float = HYBRID_DENSE_FRACTION) -> np.ndarray:
    """One byte per 128 x 128 tile (row-block major); exactly round(f*T) ones."""
    RB = (rows + HYBRID_TILE - 1) // HYBRID_TILE
    KT = K // HYBRID_TILE
    T = RB * KT
    mask = np.zeros(T, np.uint8)
    mask[rng(seed).permutation(T)[:int(round(fraction * T))]] = 1
    return mask.reshape(RB, KT)


def tiny(seed: int = 0):
    """X[16 x 256] ~ N(0,1), W[256 x 256] ~ N(0, 0.02^2) as bf16 bits."""
    g = rng(seed)
    X = to_bf16_bits(g.normal(0.0, 1.0, size=(16, 256)).astype(np.float32))
    W = to_bf16_bits(g.normal(0.0, 0.02, size=(256, 256)).astype(np.float32))
    return X, W


def linear_pair(M: int, N: int, K: int, seed: int, outliers: bool = False):
    """(X bits [M x K] ~ N(0,1), W bits [N x K] ~ N(0,0.02^2)) for one GEMM."""
    if outliers:
        W = weights_with_outliers(N, K, seed)
    else:
        W = normal_bf16((N, K), 0.02, seed)
    X = normal_bf16((M, K), 1.0, seed + 1_000_003)
    return X, W
