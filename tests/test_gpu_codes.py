"""Bit-exact check of the activation codes and scales that biloco_gemm quantises
inside the call, on every path that does so (through the C-ABI).

biloco_gemm never returns its quantised activation, so the test makes y reveal
it.  Row n of the weight has a single non-zero, 21 * 2^-5 (exact in FP32), at
column k(n) = n mod K, with N >= K so that every column is hit.  The library's
packer (itself bit-exact against the oracle) then gives g = 2^-12, block scale
448 and code 6 for that element, zero codes elsewhere, so

    y[m, n] = BF16( g * 6 * 448 * deq(x)[m, k(n)] ) = BF16( 0.65625 * deq(x)[m, k(n)] )

where deq(x) is the product of the E2M1 code and the E4M3 scale.  The product
with a single non-zero term is exact in FP32 on every path (11 significant bits
at most), so y must equal the oracle's deq(x) pushed through the same exact
product and one BF16 rounding, element for element.  Distinct codes or scales
give distinct y here (neighbouring E2M1 values differ by at least 4/3 and
E4M3 steps by at least 1/16, far above BF16 rounding), so a wrong code, scale,
swizzle lane or scale slot changes y.

With r > 0 and alpha = 0 the correction is exactly zero, so the same check runs
the whole correction path (grid arrivals, tensor-core V pieces, U side) and the
FP4 part must still come out bit-exact.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4 as on
from gpu_common import to_dev_bf16
from test_gpu_pack import _adversarial_x
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

HOT = 0.65625          # 21 * 2^-5: g = HOT / 2688 = 2^-12 exactly, block scale 448, code 6


@pytest.fixture(scope="module")
def nb():
    import nvfp4_binary_rank_b200 as nb
    nb.load()
    return nb


def _one_hot_weight(nb, N, K):
    assert N >= K
    R = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    n = torch.arange(N, device="cuda")
    sign = torch.where((n * 7919) % 3 == 0, -1.0, 1.0)
    R[n, n % K] = HOT * sign
    W, sf, g = nb.pack_weight(R)
    del R
    assert g.item() == 2.0 ** -12
    return W, sf, g, sign.cpu().numpy()


def _expected_y(x_f32, N, K, sign):
    xq, xs = on.quant_act(x_f32)
    deq = on.dequant(xq, xs)                               # exact, float64
    cols = np.arange(N) % K
    val = HOT * deq[:, cols] * sign[None, :]               # exact in float64 and float32
    return bf16_bits_to_f32(f32_to_bf16_bits(val.astype(np.float32)))


# (M, N, K): the decode-batch classes 1, 2, 4 (each CTA quantises its own chunks)
# and 8 to 128 (one activation image shared by the grid; from 32 rows streamed with
# the weight stages), the general kernel quantising per unit (M <= 8 with more than
# 16 units per CTA) and the activation pre-pass (M > 8 with more units per CTA than
# the decode classes take), at full K and with a ragged last chunk.
SHAPES = [
    (1, 5120, 5120), (1, 5248, 5184), (2, 5120, 5120), (3, 5120, 5120), (4, 5248, 5184),
    (5, 5120, 5120), (8, 5120, 5120), (11, 5248, 5184), (16, 5120, 5120),
    (1, 13824, 13824), (4, 13824, 13824), (8, 13824, 13824),
    (12, 13824, 13824), (17, 5248, 5184), (32, 5120, 5120), (33, 5120, 5120), (64, 5120, 5120),
    (100, 5248, 5184), (128, 5248, 5184), (128, 13824, 13824),
]


@pytest.mark.parametrize("r", [0, 512])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_in_gemm_activation_codes_bit_exact(nb, M, N, K, r):
    bits, xf = _adversarial_x(M, K, seed=M * 131 + K)
    x = to_dev_bf16(bits)
    W, sf, g, sign = _one_hot_weight(nb, N, K)
    if r:
        rng = np.random.default_rng(M + r)
        U = torch.from_numpy((2 * rng.integers(0, 2, (N, r)) - 1).astype(np.float32)).cuda()
        Vt = torch.from_numpy((2 * rng.integers(0, 2, (r, K)) - 1).astype(np.float32)).cuda()
        Ub, Vb = nb.pack_signs(U), nb.pack_signs(Vt)
        alpha = torch.zeros((r,), dtype=torch.float32, device="cuda")
    else:
        Ub = Vb = alpha = None
    y = nb.gemm(x, W, sf, g, Ub, Vb, alpha)
    st = nb.last_error()
    assert st == 0, nb.status_string(st)
    got = y.float().cpu().numpy()
    want = _expected_y(xf, N, K, sign)
    bad = np.argwhere(got != want)
    assert bad.size == 0, (f"{len(bad)} elements differ, first (m, n) = {tuple(bad[0])}: "
                           f"{got[tuple(bad[0])]} vs {want[tuple(bad[0])]}")
