"""Bit-exact parity of the activation quantiser, weight packer and sign packer
against the CPU oracle (through the C-ABI)."""

import numpy as np
import pytest
import torch

import workloads
from oracle import biloco as ob
from oracle import nvfp4 as on
from gpu_common import device_problem, to_dev_bf16, untile_weight_sf

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nb():
    import nvfp4_binary_rank_b200 as nb
    nb.load()
    return nb


def _adversarial_x(M, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    grid = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    # blocks whose amax is 6 hold exact E2M1 midpoints (ties), some blocks are zero,
    # some tiny (subnormal E4M3 scales), some huge (scale saturates at 448)
    for m in range(M):
        for b in range(K // 16):
            kind = (m * 7 + b) % 6
            blk = slice(16 * b, 16 * b + 16)
            if kind == 0:
                x[m, blk] = np.resize(np.concatenate([grid, -grid]), 16)
            elif kind == 1:
                x[m, blk] = 0.0
            elif kind == 2:
                x[m, blk] *= np.float32(1e-4)
            elif kind == 3:
                x[m, blk] *= np.float32(3e3)
    from workloads import f32_to_bf16_bits, bf16_bits_to_f32
    bits = f32_to_bf16_bits(x)
    return bits, bf16_bits_to_f32(bits)


@pytest.mark.parametrize("M,K,seed", [(1, 256, 0), (3, 320, 1), (32, 5120, 2), (128, 1024, 3)])
def test_quant_act_bit_exact(nb, M, K, seed):
    bits, xf = _adversarial_x(M, K, seed)
    codes, sf = nb.quant_act(to_dev_bf16(bits))
    rq, rs = on.quant_act(xf)
    np.testing.assert_array_equal(sf.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rq)


def test_quant_act_bit_exact_decode_workload(nb):
    d = workloads.make_inputs(workloads.CONFIGS["mlp_down"], with_R=False)
    codes, sf = nb.quant_act(to_dev_bf16(d["x_bf16"]))
    rq, rs = on.quant_act(d["x"])
    np.testing.assert_array_equal(sf.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rq)


@pytest.mark.parametrize("N,K,seed", [(128, 64, 0), (256, 320, 1), (384, 1024, 2)])
def test_pack_weight_bit_exact(nb, N, K, seed):
    rng = np.random.default_rng(seed)
    R = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    R[0, :16] = 0.0                                   # a zero block
    R[1, :16] *= np.float32(1e-3)                     # a tiny block
    W, sf, g = nb.pack_weight(torch.from_numpy(R).cuda())
    rq, rs, rg = on.quant_weight(R)
    assert g.item() == float(rg)
    np.testing.assert_array_equal(W.cpu().numpy(), rq)
    sfn = sf.cpu().numpy()
    np.testing.assert_array_equal(untile_weight_sf(sfn, N, K), rs)
    # the padding of the last 256-element chunk is zero
    used = np.zeros(sfn.size, bool)
    KC = (K + 255) // 256
    n = np.arange(N)[:, None]; b = np.arange(K // 16)[None, :]
    used[((((n // 128) * KC + b // 16) * 4 + (b % 16) // 4) * 512 + (n % 32) * 16
          + ((n % 128) // 32) * 4 + (b % 4)).reshape(-1)] = True
    assert not sfn[~used].any()


def test_pack_weight_zero_matrix(nb):
    W, sf, g = nb.pack_weight(torch.zeros((128, 256), device="cuda"))
    assert g.item() == 1.0 and not W.any().item() and not sf.any().item()


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_pack_weight_workloads_bit_exact(nb, name):
    w = workloads.CONFIGS[name]
    d = workloads.make_inputs(w)
    W, sf, g = nb.pack_weight(torch.from_numpy(d["R"]).cuda())
    rq, rs, rg = on.quant_weight(d["R"])
    assert g.item() == float(rg)
    np.testing.assert_array_equal(W.cpu().numpy(), rq)
    np.testing.assert_array_equal(untile_weight_sf(sf.cpu().numpy(), w.N, w.K), rs)


@pytest.mark.parametrize("rows,cols", [(1, 1), (7, 40), (512, 5120), (5120, 512), (3, 1024)])
def test_pack_signs_bit_exact(nb, rows, cols):
    rng = np.random.default_rng(rows * 31 + cols)
    S = (2 * rng.integers(0, 2, (rows, cols)) - 1).astype(np.float32)
    S[0, 0] = 0.0                                     # sign(0) = +1
    bits = nb.pack_signs(torch.from_numpy(S).cuda())
    want = ob.pack_signs(S).view(np.int32)
    np.testing.assert_array_equal(bits.cpu().numpy(), want)
