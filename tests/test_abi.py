"""The C-ABI library loads and exports every entry point include/biloco.h declares
(CPU only: no call here reaches the GPU)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "biloco.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(biloco_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from nvfp4_binary_rank_b200 import build, _lib
    build.build()
    return _lib.load()


def test_header_declares_the_four_hot_path_calls():
    names = _declared()
    for n in ("biloco_quant_act", "biloco_pack_signs", "biloco_pack_weight", "biloco_gemm"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_signatures_cover_the_header(lib):
    from nvfp4_binary_rank_b200 import _lib
    assert sorted(_lib.SIGNATURES) == _declared()


def test_status_strings(lib):
    from nvfp4_binary_rank_b200 import _lib
    assert _lib.status_string(0) == "ok"
    assert "timed out" in _lib.status_string(_lib.ERR_TIMEOUT)
    assert _lib.status_string(12345) == "unknown status"


def test_weight_sf_bytes(lib):
    from nvfp4_binary_rank_b200 import _lib
    assert _lib.weight_sf_bytes(5120, 5120) == 5120 * 5120 // 16
    assert _lib.weight_sf_bytes(128, 320) == 128 * 2 * 16     # K padded to whole 256-chunks


def test_host_validation_rejects_bad_arguments_without_a_gpu(lib):
    # argument and shape checks run before any CUDA call
    P = ctypes.c_void_p
    fake = P(0x10000)
    assert lib.biloco_gemm(None, fake, fake, fake, None, None, None, fake, 1, 128, 64, 0, None) == -1
    assert lib.biloco_gemm(fake, fake, fake, fake, None, None, None, fake, 0, 128, 64, 0, None) == -2
    assert lib.biloco_gemm(fake, fake, fake, fake, None, None, None, fake, 129, 128, 64, 0, None) == -2
    assert lib.biloco_gemm(fake, fake, fake, fake, None, None, None, fake, 1, 100, 64, 0, None) == -2
    assert lib.biloco_gemm(fake, fake, fake, fake, None, None, None, fake, 1, 128, 96, 0, None) == -2
    assert lib.biloco_gemm(fake, fake, fake, fake, None, None, None, fake, 1, 128, 64, 1025, None) == -1
    assert lib.biloco_gemm(fake, fake, fake, fake, fake, fake, fake, fake, 1, 128, 64, 1025, None) == -2
    assert lib.biloco_gemm(P(0x10008), fake, fake, fake, None, None, None, fake, 1, 128, 64, 0, None) == -3
    assert lib.biloco_pack_weight(fake, 100, 64, fake, fake, fake, None) == -2
    assert lib.biloco_quant_act(fake, 1, 24, fake, fake, None) == -2
    assert lib.biloco_pack_signs(None, 1, 1, fake, None) == -1
    assert lib.biloco_gemm_noalloc(None, fake, fake, fake, None, None, None, fake, 1, 128, 64, 0, None) == -1
    assert lib.biloco_gemm_noalloc(fake, fake, fake, fake, None, None, None, fake, 1, 100, 64, 0, None) == -2


def test_mode_setting(lib):
    from nvfp4_binary_rank_b200 import _lib
    assert lib.biloco_set_mode(7) == -1
    for m in (_lib.MODE_SHARED_Z, _lib.MODE_LOCAL_Z):
        assert lib.biloco_set_mode(m) == 0
        assert lib.biloco_resolve_mode(1, 5120, 5120, 512) == m
    assert lib.biloco_set_mode(_lib.MODE_AUTO) == 0
    assert lib.biloco_resolve_mode(1, 5120, 5120, 512) in (_lib.MODE_SHARED_Z, _lib.MODE_LOCAL_Z)


def test_kernel_count_follows_the_schedule(lib):
    from nvfp4_binary_rank_b200 import _lib
    # decode batches run one kernel (it quantises the activation itself)
    assert lib.biloco_gemm_kernel_count(1, 5120, 5120, 512) == 1
    assert lib.biloco_gemm_kernel_count(16, 13824, 5120, 512) == 1
    assert lib.biloco_gemm_kernel_count(32, 5120, 13824, 512) == 1
    assert lib.biloco_gemm_kernel_count(17, 5120, 5120, 1024) == 1
    assert lib.biloco_gemm_kernel_count(33, 5120, 13824, 512) == 1
    assert lib.biloco_gemm_kernel_count(128, 5120, 5120, 512) == 1
    # more than 64 units per CTA: quantiser + general GEMM
    assert lib.biloco_gemm_kernel_count(33, 65536, 65536, 512) == 2
    assert lib.biloco_gemm_kernel_count(128, 65536, 65536, 512) == 2
    # the local-z schedule runs the general kernel (in-kernel quantisation up to M = 8)
    assert lib.biloco_set_mode(_lib.MODE_LOCAL_Z) == 0
    try:
        assert lib.biloco_gemm_kernel_count(8, 5120, 5120, 512) == 1
        assert lib.biloco_gemm_kernel_count(16, 5120, 5120, 512) == 2
    finally:
        lib.biloco_set_mode(_lib.MODE_AUTO)
    assert lib.biloco_gemm_kernel_count(1, 100, 64, 0) == -2


def test_launch_form_and_selftest_controls(lib):
    from nvfp4_binary_rank_b200 import _lib
    assert lib.biloco_get_launch() == _lib.LAUNCH_PDL
    assert lib.biloco_set_launch(4) == -1
    assert lib.biloco_set_launch(-1) == -1
    for f in (0, 1, 2, 3):
        assert lib.biloco_set_launch(f) == 0
        assert lib.biloco_get_launch() == f
    assert lib.biloco_set_launch(_lib.LAUNCH_PDL) == 0
    assert lib.biloco_selftest_drop_arrivals(4) == -1
    assert lib.biloco_selftest_drop_arrivals(-1) == -1
    assert lib.biloco_status_string(-8).decode() == "grid cannot be resident on the GPU at once"


def test_correction_setting(lib):
    from nvfp4_binary_rank_b200 import _lib
    assert lib.biloco_set_correction(3) == -1
    for a in (_lib.CORR_SIGNS, _lib.CORR_LUT):
        assert lib.biloco_set_correction(a) == 0
        assert lib.biloco_resolve_correction(1, 5120, 5120, 512) == a
    assert lib.biloco_set_correction(_lib.CORR_AUTO) == 0
    assert lib.biloco_resolve_correction(1, 5120, 5120, 512) in (_lib.CORR_SIGNS, _lib.CORR_LUT)
