"""NVFP4 codec written out from its definition: E2M1 elements, E4M3 block scales.

TEST INFRASTRUCTURE ONLY.  This is part of the CPU oracle: a plain, slow,
obviously-correct restatement used to check the GPU library.  Only the test
suite, the smoke check and the benchmark's CPU-baseline leg may import it; the
library never does.

Source passages
  BiLoCo README (github jindavid/BiLoCo), section "Decomposition": the residual
    R is quantised to NVFP4 after the decomposition.
  BiLoCo README, section "Kernel": FP4(x) FP4(R)^T, with the activation passed as
    NVFP4 codes plus block scales (A_pad, A_sf) and the weight as codes, block
    scales and a global scale (W_fp4, W_sf, w_global_scale).
  North-star statement of the format: E2M1 codes on the grid
    {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}, one E4M3 scale per 16 elements
    along K, an FP32 tensor scale for the weight.

Readings where the pages are silent (each one is listed in the design notes):
  * Block scale: s = E4M3_RNE_satfinite(t) with t = amax_b / 6 for activations and
    t = amax_b / (6 g) for the weight; the product 6*g and the quotient are FP32,
    each rounded to nearest.
  * Weight tensor scale g = amax(|R|) / 2688 in FP32 (2688 = 6 * 448), g = 1 when R == 0.
    Activations have no tensor scale (the kernel call passes none).
  * Element code: q = v / S in FP32 (correctly rounded), S = scale for activations
    and S = fp32(scale * g) for the weight; q is rounded to the E2M1 magnitude
    grid to nearest with ties to the even code (mantissa bit 0), |q| > 6
    saturates to 6.  If S == 0 every code of the block is 0.
  * Signed zero: a zero magnitude is always stored as code 0 (never 0x8).
  * Packing: element 2j of a row sits in the low nibble of byte j.

Every step that decides a code (division, rounding) is carried out in FP32, as
the pages' FP4 hardware path would; the decode of codes and scales is exact.
"""

from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# E2M1 element format: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
# ---------------------------------------------------------------------------


def e2m1_value(code: int) -> float:
    """Value of one 4-bit E2M1 code, from the bit fields."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        mag = 0.5 * m                       # subnormal: 0 or 0.5
    else:
        mag = 2.0 ** (e - 1) * (1.0 + 0.5 * m)
    return -mag if s else mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)

# Positive magnitudes in code order 0..7: 0, .5, 1, 1.5, 2, 3, 4, 6; the
# rounding boundaries lie halfway between neighbours.
_E2M1_MAGS = E2M1_TABLE[:8]
_E2M1_MIDPOINTS = (_E2M1_MAGS[:-1] + _E2M1_MAGS[1:]) / 2.0   # .25 .75 1.25 1.75 2.5 3.5 5


def e2m1_encode(q: np.ndarray) -> np.ndarray:
    """Round FP32 values to E2M1 codes: nearest, ties to even code, saturating at 6."""
    a = np.abs(np.asarray(q, dtype=np.float32)).astype(np.float64)
    mag = np.zeros(a.shape, dtype=np.uint8)
    for j, t in enumerate(_E2M1_MIDPOINTS):
        upper = j + 1                                   # code just above this midpoint
        passed = (a > t) | ((a == t) & (upper % 2 == 0))
        mag += passed.astype(np.uint8)
    neg = (np.asarray(q, dtype=np.float32) < 0) & (mag != 0)
    return (mag | (neg.astype(np.uint8) << 3)).astype(np.uint8)


# ---------------------------------------------------------------------------
# E4M3 (the "fn" variant: no infinities, 0x7F/0xFF are NaN, max finite 448).
# ---------------------------------------------------------------------------


def e4m3_value(byte: int) -> float:
    s = (byte >> 7) & 1
    e = (byte >> 3) & 15
    m = byte & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        mag = (m / 8.0) * 2.0 ** -6
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E4M3_TABLE = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)
_E4M3_POS = E4M3_TABLE[:127]          # bytes 0..126: 0 .. 448, strictly increasing
E4M3_MAX = 448.0


def e4m3_encode_nonneg(t: np.ndarray) -> np.ndarray:
    """Round non-negative FP32 values to E4M3: nearest, ties to even, clamp to 448."""
    t = np.asarray(t, dtype=np.float32).astype(np.float64)
    if np.any(t < 0) or np.any(np.isnan(t)):
        raise ValueError("block scales are non-negative and finite")
    # Neighbours on the grid: value[lo] <= t < value[lo + 1] (both exact in float64).
    lo = np.clip(np.searchsorted(_E4M3_POS, t, side="right") - 1, 0, 125)
    hi = lo + 1
    d_lo = t - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - t
    tie = d_lo == d_hi
    # Nearer neighbour; on a tie the even byte (its mantissa LSB is the byte LSB).
    pick_hi = (d_hi < d_lo) | (tie & (lo % 2 == 1))
    out = np.where(pick_hi, hi, lo)
    out = np.where(t >= E4M3_MAX, 126, out)                 # satfinite: clamp to 448
    return out.astype(np.uint8)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(b, dtype=np.uint8)]


# ---------------------------------------------------------------------------
# Nibble packing.
# ---------------------------------------------------------------------------


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., K] 4-bit codes -> [..., K/2] bytes, element 2j in the low nibble of byte j."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


# ---------------------------------------------------------------------------
# Block quantisers.
# ---------------------------------------------------------------------------

BLOCK = 16


def _quantise_blocks(v: np.ndarray, t: np.ndarray, g: np.float32 | None):
    """v: float32 [..., nb, 16]; t: float32 [..., nb] the pre-rounding scale."""
    s = e4m3_encode_nonneg(t)
    S = e4m3_decode(s).astype(np.float32)
    if g is not None:
        S = (S * np.float32(g)).astype(np.float32)           # fp32 product, nearest
    codes = np.zeros(v.shape, dtype=np.uint8)
    nz = S != 0
    if np.any(nz):
        with np.errstate(divide="ignore", invalid="ignore"):
            q = (v / S[..., None]).astype(np.float32)        # fp32 quotient, nearest
        codes = np.where(nz[..., None], e2m1_encode(q), np.uint8(0)).astype(np.uint8)
    return codes, s


def quant_act(x: np.ndarray):
    """NVFP4 activation quantiser, no tensor scale.

    x: float32 [M, K] (BF16 values), K a multiple of 16.
    Returns codes uint8 [M, K/2] (packed) and scales uint8 [M, K/16] (E4M3 bytes).
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    blocks = x.reshape(M, K // BLOCK, BLOCK)
    amax = np.abs(blocks).max(axis=2).astype(np.float32)
    t = (amax / np.float32(6.0)).astype(np.float32)
    codes, s = _quantise_blocks(blocks, t, None)
    return pack_nibbles(codes.reshape(M, K)), s.astype(np.uint8)


def weight_global_scale(R: np.ndarray) -> np.float32:
    amax = np.float32(np.abs(np.asarray(R, dtype=np.float32)).max()) if R.size else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(6.0 * 448.0))


def quant_weight(R: np.ndarray):
    """NVFP4 weight quantiser with an FP32 tensor scale.

    R: float32 [N, K].  Returns codes uint8 [N, K/2], scales uint8 [N, K/16] (row-major),
    and the tensor scale g (float32).
    """
    R = np.asarray(R, dtype=np.float32)
    N, K = R.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = weight_global_scale(R)
    blocks = R.reshape(N, K // BLOCK, BLOCK)
    amax = np.abs(blocks).max(axis=2).astype(np.float32)
    d = np.float32(np.float32(6.0) * g)
    t = (amax / d).astype(np.float32)
    codes, s = _quantise_blocks(blocks, t, g)
    return pack_nibbles(codes.reshape(N, K)), s.astype(np.uint8), g


def dequant(codes_packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact float64 value of NVFP4 codes times their E4M3 block scales (no tensor scale)."""
    c = unpack_nibbles(codes_packed)
    rows, K = c.shape
    vals = E2M1_TABLE[c]
    sc = np.repeat(e4m3_decode(scales), BLOCK, axis=1)
    assert sc.shape == (rows, K)
    return vals * sc
