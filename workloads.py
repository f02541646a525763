"""Seeded synthetic inputs for the fused NVFP4 + binary-sign low-rank GEMM.

This module only draws random numbers and rounds the activation to BF16 (the
input type).  It holds none of the method's arithmetic: no NVFP4 quantisation,
no sign packing, no GEMM.  Both the CPU oracle tests and the GPU path take their
inputs from here, so the two sides always see the same operands.

Workloads (BiLoCo README, section "Kernel": decode batches of up to 32 rows;
FluxBin Table 12 uses the same 5120x5120 and 5120x13824 weight sizes):

    tiny      M=1,  N=256,   K=256,   r=16,  seed 0, no outlier channels, alpha_i = 0.05*0.9^i
    decode    M=1,  N=5120,  K=5120,  r=512, seed 1
    mlp_up    M=16, N=13824, K=5120,  r=512, seed 2
    mlp_down  M=32, N=5120,  K=13824, r=512, seed 3
    sweep     N=K=5120, M in {1,8,32,64,128}, r in {0,32,128,512,1024}, seed 4

Recipe (draw order is fixed: x, outlier channels, R, U, V):
    x      float32 N(0,1) of shape [M,K]; 1% of the K channels (rng.choice without
           replacement, round(0.01*K) of them) multiplied by 20; then rounded to
           BF16 with round-to-nearest-even.
    R      float32 N(0, 0.02^2) of shape [N,K] (the NVFP4 residual before quantisation).
    U, V   Rademacher +-1, shapes [N,r] and [K,r] (int8).
    alpha  alpha_i = 0.05 * decay^i in float32 (decay 0.995, or 0.9 for tiny).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = ["Workload", "CONFIGS", "SWEEP_MS", "SWEEP_RS", "sweep_config", "make_inputs",
           "decompose_inputs", "f32_to_bf16_bits", "bf16_bits_to_f32"]


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    r: int
    seed: int
    outliers: bool = True
    alpha_decay: float = 0.995


CONFIGS = {
    "tiny": Workload("tiny", 1, 256, 256, 16, 0, outliers=False, alpha_decay=0.9),
    "decode": Workload("decode", 1, 5120, 5120, 512, 1),
    "mlp_up": Workload("mlp_up", 16, 13824, 5120, 512, 2),
    "mlp_down": Workload("mlp_down", 32, 5120, 13824, 512, 3),
}

SWEEP_MS = (1, 8, 32, 64, 128)
SWEEP_RS = (0, 32, 128, 512, 1024)


def sweep_config(M: int, r: int) -> Workload:
    return Workload(f"sweep_M{M}_r{r}", M, 5120, 5120, r, 4)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to BF16 (nearest, ties to even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_inputs(w: Workload, *, with_R: bool = True) -> dict:
    """Draw one workload's operands.

    Returns a dict with
      x_bf16  uint16 [M,K]   BF16 bit patterns of the activation
      x       float32 [M,K]  the same values widened to float32 (exact)
      R       float32 [N,K]  residual before NVFP4 quantisation (omitted if with_R=False,
                             which still consumes the same random draws)
      U       int8 [N,r], V int8 [K,r]   +-1 sign factors
      alpha   float32 [r]
    """
    rng = np.random.default_rng(w.seed)
    x = rng.standard_normal((w.M, w.K), dtype=np.float32)
    if w.outliers:
        n_out = int(round(0.01 * w.K))
        ch = rng.choice(w.K, n_out, replace=False)
        x[:, ch] *= np.float32(20.0)
    x_bits = f32_to_bf16_bits(x)
    R = rng.standard_normal((w.N, w.K), dtype=np.float32) * np.float32(0.02)
    U = (2 * rng.integers(0, 2, size=(w.N, w.r), dtype=np.int8) - 1).astype(np.int8)
    V = (2 * rng.integers(0, 2, size=(w.K, w.r), dtype=np.int8) - 1).astype(np.int8)
    alpha = (0.05 * np.power(w.alpha_decay, np.arange(w.r, dtype=np.float64))).astype(np.float32)
    out = dict(x_bf16=x_bits, x=bf16_bits_to_f32(x_bits), U=U, V=V, alpha=alpha)
    if with_R:
        out["R"] = R
    return out


def decompose_inputs(N: int, K: int, r: int, seed: int, planted: int = 0) -> dict:
    """A weight to decompose and the start signs of the decomposition's terms.

    W      float32 [N, K]: N(0, 0.02^2), plus `planted` binary rank-one terms
           0.03 * 0.9^j * u_j v_j^T with Rademacher u_j, v_j (a structured part for
           the peeling to find); drawn in this order: noise, planted signs.
    v0     int8 [r, K]: Rademacher start signs, one row per term (the random
           draws the method makes, handed to both sides).
    """
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    for j in range(planted):
        u = (2 * rng.integers(0, 2, size=N) - 1).astype(np.float32)
        v = (2 * rng.integers(0, 2, size=K) - 1).astype(np.float32)
        W += np.float32(0.03 * 0.9 ** j) * np.outer(u, v).astype(np.float32)
    v0 = (2 * rng.integers(0, 2, size=(r, K), dtype=np.int8) - 1).astype(np.int8)
    return dict(W=W.astype(np.float32), v0=v0)
