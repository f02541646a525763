"""Shared helpers of the GPU parity tests: device operands from the seeded
workloads, the documented weight-scale tile layout read back to row-major, and
the y tolerance (relative L2 <= 5e-3 and max |err| <= 2e-2 * rms(y_ref))."""

from __future__ import annotations

import functools

import numpy as np
import torch

import workloads
from oracle import biloco as ob

REL_L2 = 5e-3
MAX_ABS_RMS = 2e-2


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).cuda()


def untile_weight_sf(sf: np.ndarray, N: int, K: int) -> np.ndarray:
    """Tile-layout weight scales (include/biloco.h, biloco_pack_weight) -> [N][K/16]."""
    KC = (K + 255) // 256
    n = np.arange(N)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((((n // 128) * KC + b // 16) * 4 + (b % 16) // 4) * 512
           + (n % 32) * 16 + ((n % 128) // 32) * 4 + (b % 4))
    return sf.reshape(-1)[off]


def device_problem(w: workloads.Workload, d: dict | None = None):
    """Pack one workload on the GPU through the library; returns the operands."""
    import nvfp4_binary_rank_b200 as nb
    if d is None:
        d = workloads.make_inputs(w)
    x = to_dev_bf16(d["x_bf16"])
    R = torch.from_numpy(d["R"]).cuda()
    W, sf, g = nb.pack_weight(R)
    if w.r:
        U = torch.from_numpy(d["U"].astype(np.float32)).cuda()
        Vt = torch.from_numpy(np.ascontiguousarray(d["V"].T).astype(np.float32)).cuda()
        Ub = nb.pack_signs(U)
        Vb = nb.pack_signs(Vt)
        alpha = torch.from_numpy(d["alpha"]).cuda()
    else:
        Ub = Vb = alpha = None
    torch.cuda.synchronize()
    return dict(x=x, W=W, sf=sf, g=g, Ub=Ub, Vb=Vb, alpha=alpha, inputs=d)


@functools.lru_cache(maxsize=16)
def oracle_for(w: workloads.Workload):
    d = workloads.make_inputs(w)
    return d, ob.biloco_reference(d["x"], d["R"], d["U"], d["V"], d["alpha"])


def y_errors(y: np.ndarray, ref: np.ndarray):
    y = y.astype(np.float64)
    err = y - ref
    rms = float(np.sqrt(np.mean(ref ** 2)))
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    return rel, float(np.abs(err).max()), rms


def assert_y_close(y: np.ndarray, ref: np.ndarray, what: str = "y"):
    rel, mx, rms = y_errors(y, ref)
    assert rel <= REL_L2, f"{what}: relative L2 error {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_RMS * rms, f"{what}: max |err| {mx:.3e} > {MAX_ABS_RMS} * rms {rms:.3e}"


def y_to_numpy(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy()
