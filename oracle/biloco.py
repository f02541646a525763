"""Fused NVFP4 GEMM with a binary-sign low-rank correction: plain FP64 definition.

TEST INFRASTRUCTURE ONLY (part of the CPU oracle).  Only the tests, the smoke
check and the benchmark's CPU-baseline leg may import it.

What is computed (BiLoCo README, sections "Decomposition" and "Kernel"):

    W ~= U diag(alpha) V^T + R,   U in {+-1}^{N x r},  V in {+-1}^{K x r},  R in NVFP4
    y  = FP4(x) FP4(R)^T + sum_i alpha_i (x . v_i) u_i

with y[m, n] for activation row m and weight row n.  The FP4 product is the
exact product of the dequantised operands, and the tensor scale g of R
multiplies it:

    y[m, n] = g * sum_k deq(xq)[m, k] * deq(Rq)[n, k]
              + sum_i alpha_i * (sum_k V[k, i] * x[m, k]) * U[n, i]

Readings where the pages are silent:
  * The correction uses the BF16 activation x, not FP4(x): the formula writes
    (x . v_i) with the unquantised x, and the kernel call passes the BF16 x next
    to the NVFP4 one.
  * alpha stays FP32 (the page's example casts it to BF16; the library does not).
  * Sign bits: bit 1 means -1, bit 0 means +1 (sign(0) = +1), least significant
    bit first within little-endian 32-bit words.  V is packed rank-major
    (Vbits[i][k/32], the layout of pack_signs(V.T) in the README's example) and
    U row-major over the rank (Ubits[n][i/32]).
  * Output is y[M, N] without the README's padding to 128 rows.

Everything here is FP64 except the NVFP4 rounding decisions, which follow the
FP32 rules of `oracle.nvfp4`.
"""

from __future__ import annotations

import numpy as np

from . import nvfp4


def pack_signs(S: np.ndarray) -> np.ndarray:
    """+-1 matrix [rows, cols] -> uint32 [rows, ceil(cols/32)], bit j of word w is
    set when S[row, 32 w + j] is negative.  Unused tail bits are zero."""
    S = np.asarray(S)
    rows, cols = S.shape
    words = (cols + 31) // 32
    out = np.zeros((rows, words), dtype=np.uint32)
    neg = S < 0
    for c in range(cols):
        out[:, c // 32] |= (neg[:, c].astype(np.uint32) << np.uint32(c % 32))
    return out


def unpack_signs(bits: np.ndarray, cols: int) -> np.ndarray:
    """Inverse of pack_signs: uint32 [rows, words] -> int8 +-1 [rows, cols]."""
    bits = np.asarray(bits, dtype=np.uint32)
    rows = bits.shape[0]
    out = np.empty((rows, cols), dtype=np.int8)
    for c in range(cols):
        b = (bits[:, c // 32] >> np.uint32(c % 32)) & np.uint32(1)
        out[:, c] = np.where(b == 1, -1, 1)
    return out


def gemm_part(xq, xs, wq, ws, g) -> np.ndarray:
    """g * FP4(x) FP4(R)^T in FP64 from codes and scales: [M, N]."""
    Xd = nvfp4.dequant(xq, xs)                 # [M, K]
    Wd = nvfp4.dequant(wq, ws)                 # [N, K]
    return float(g) * (Xd @ Wd.T)


def z_vector(x, V, alpha) -> np.ndarray:
    """z[m, i] = alpha_i * sum_k V[k, i] x[m, k] in FP64: [M, r]."""
    x64 = np.asarray(x, dtype=np.float64)
    V64 = np.asarray(V, dtype=np.float64)
    return (x64 @ V64) * np.asarray(alpha, dtype=np.float64)[None, :]


def correction_part(x, U, V, alpha) -> np.ndarray:
    """sum_i alpha_i (x . v_i) u_i in FP64: [M, N]."""
    z = z_vector(x, V, alpha)
    return z @ np.asarray(U, dtype=np.float64).T


def biloco_reference(x, R, U, V, alpha) -> dict:
    """Quantise the operands the way the library must, then y in FP64.

    x: float32 [M, K] (BF16 values); R: float32 [N, K]; U: [N, r]; V: [K, r];
    alpha: float32 [r].  Returns the bit-exact artefacts and the FP64 y with its
    two parts.
    """
    xq, xs = nvfp4.quant_act(x)
    wq, ws, g = nvfp4.quant_weight(R)
    gemm = gemm_part(xq, xs, wq, ws, g)
    r = np.asarray(alpha).shape[0]
    if r:
        corr = correction_part(x, U, V, alpha)
    else:
        corr = np.zeros_like(gemm)
    return dict(xq=xq, xs=xs, wq=wq, ws=ws, g=g,
                Ubits=pack_signs(U) if r else np.zeros((R.shape[0], 0), np.uint32),
                Vbits=pack_signs(np.asarray(V).T) if r else np.zeros((0, R.shape[1] // 32), np.uint32),
                gemm=gemm, corr=corr, y=gemm + corr)
