"""Fused NVFP4 GEMM with a binary-sign low-rank correction for one B200 (sm_100a).

    y = FP4(x) FP4(R)^T + sum_i alpha_i (x . v_i) u_i

The compute is the C-ABI library libbiloco.so (include/biloco.h); this package
is its thin ctypes binding.  Build the library with
`python -m nvfp4_binary_rank_b200.build`.
"""

from ._lib import (  # noqa: F401
    BilocoError, CORR_AUTO, CORR_LUT, CORR_SIGNS, LAUNCH_COOPERATIVE, LAUNCH_PDL, MODE_AUTO, MODE_LOCAL_Z, MODE_SHARED_Z, MAX_M, MAX_R,
    decompose, gemm, gemm_kernel_count, gemm_noalloc, get_launch, selftest_drop_arrivals, selftest_wait_timeout,
    resolve_correction, set_correction, set_launch,
    last_error, load, pack_signs, pack_weight, quant_act, resolve_mode, set_mode, shutdown,
    status_string, weight_sf_bytes,
)
