"""ctypes binding of libbiloco.so (include/biloco.h).

Argument marshalling only: every step runs in the library's CUDA kernels.  The
binding allocates outputs with PyTorch (device memory) and passes PyTorch's
current stream.  There is no CPU fallback: if the library is missing or the
device is not an sm_100 GPU the calls raise.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbiloco.so")

OK = 0
ERR_ARG, ERR_SHAPE, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT, ERR_NOMEM, ERR_DEVICE, ERR_RESIDENCY = range(-1, -9, -1)
LAUNCH_PDL, LAUNCH_COOPERATIVE = 1, 2
CORR_AUTO, CORR_SIGNS, CORR_LUT = 0, 1, 2
MODE_AUTO, MODE_SHARED_Z, MODE_LOCAL_Z = 0, 1, 2
MAX_M, MAX_R = 128, 1024

_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int

# name -> (restype, argtypes); must match include/biloco.h
SIGNATURES = {
    "biloco_quant_act": (_I, [_P, _I, _I, _P, _P, _P]),
    "biloco_pack_signs": (_I, [_P, _I, _I, _P, _P]),
    "biloco_pack_weight": (_I, [_P, _I, _I, _P, _P, _P, _P]),
    "biloco_weight_sf_bytes": (ctypes.c_size_t, [_I, _I]),
    "biloco_decompose_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I]),
    "biloco_decompose": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "biloco_gemm": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "biloco_gemm_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "biloco_set_mode": (_I, [_I]),
    "biloco_resolve_mode": (_I, [_I, _I, _I, _I]),
    "biloco_last_error": (_I, [_P]),
    "biloco_selftest_wait_timeout": (_I, [_P]),
    "biloco_selftest_drop_arrivals": (_I, [_I]),
    "biloco_set_launch": (_I, [_I]),
    "biloco_get_launch": (_I, []),
    "biloco_set_correction": (_I, [_I]),
    "biloco_resolve_correction": (_I, [_I, _I, _I, _I]),
    "biloco_status_string": (ctypes.c_char_p, [_I]),
    "biloco_gemm_kernel_count": (_I, [_I, _I, _I, _I]),
    "biloco_shutdown": (None, []),
}


class BilocoError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m nvfp4_binary_rank_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().biloco_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != OK:
        raise BilocoError(fn, status)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need_cuda(t: torch.Tensor, name: str, dtype):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def weight_sf_bytes(N: int, K: int) -> int:
    return int(load().biloco_weight_sf_bytes(N, K))


def quant_act(x: torch.Tensor, stream=None):
    """BF16 [M, K] -> (codes uint8 [M, K/2], scales uint8 [M, K/16])."""
    _need_cuda(x, "x", torch.bfloat16)
    M, K = x.shape
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    sf = torch.empty((M, K // 16), dtype=torch.uint8, device=x.device)
    _check("biloco_quant_act",
           load().biloco_quant_act(_ptr(x), M, K, _ptr(codes), _ptr(sf), _stream(stream)))
    return codes, sf


def pack_signs(S: torch.Tensor, stream=None) -> torch.Tensor:
    """float32 [rows, cols] -> int32 [rows, ceil(cols/32)] holding the uint32 sign words."""
    _need_cuda(S, "S", torch.float32)
    rows, cols = S.shape
    bits = torch.empty((rows, (cols + 31) // 32), dtype=torch.int32, device=S.device)
    _check("biloco_pack_signs",
           load().biloco_pack_signs(_ptr(S), rows, cols, _ptr(bits), _stream(stream)))
    return bits


def pack_weight(R: torch.Tensor, stream=None):
    """float32 [N, K] -> (W_fp4 uint8 [N, K/2], W_sf uint8 [tile layout], gscale float32 [1])."""
    _need_cuda(R, "R", torch.float32)
    N, K = R.shape
    W = torch.empty((N, K // 2), dtype=torch.uint8, device=R.device)
    sf = torch.empty((weight_sf_bytes(N, K),), dtype=torch.uint8, device=R.device)
    g = torch.empty((1,), dtype=torch.float32, device=R.device)
    _check("biloco_pack_weight",
           load().biloco_pack_weight(_ptr(R), N, K, _ptr(W), _ptr(sf), _ptr(g), _stream(stream)))
    return W, sf, g


def decompose(W: torch.Tensor, r: int, T: int, v0bits: torch.Tensor | None, stream=None):
    """float32 [N, K] -> (Ubits int32 [N, ceil(r/32)], Vbits int32 [r, ceil(K/32)],
    alpha float32 [r], R float32 [N, K]) with W ~= U diag(alpha) V^T + R.
    v0bits: int32 [r, ceil(K/32)], the packed start signs of each term."""
    _need_cuda(W, "W", torch.float32)
    N, K = W.shape
    RW, KW = (r + 31) // 32, (K + 31) // 32
    if r:
        _need_cuda(v0bits, "v0bits", torch.int32)
        if tuple(v0bits.shape) != (r, KW):
            raise ValueError("v0bits must be [r, ceil(K/32)]")
    Ub = torch.empty((N, max(RW, 1)), dtype=torch.int32, device=W.device)
    Vb = torch.empty((max(r, 1), KW), dtype=torch.int32, device=W.device)
    alpha = torch.empty((max(r, 1),), dtype=torch.float32, device=W.device)
    R = torch.empty_like(W)
    nbytes = int(load().biloco_decompose_workspace_bytes(N, K, r))
    if nbytes == 0:
        raise BilocoError("biloco_decompose_workspace_bytes", ERR_SHAPE)
    ws = torch.empty((nbytes,), dtype=torch.uint8, device=W.device)
    _check("biloco_decompose", load().biloco_decompose(
        _ptr(W), N, K, r, T, _ptr(v0bits if r else None), _ptr(Ub), _ptr(Vb), _ptr(alpha), _ptr(R),
        _ptr(ws), nbytes, _stream(stream)))
    return Ub[:, :RW], Vb[:r], alpha[:r], R


def _gemm_call(fn: str, x, W_fp4, W_sf, gscale, Ubits, Vbits, alpha, out, stream):
    _need_cuda(x, "x", torch.bfloat16)
    _need_cuda(W_fp4, "W_fp4", torch.uint8)
    _need_cuda(W_sf, "W_sf", torch.uint8)
    _need_cuda(gscale, "gscale", torch.float32)
    M, K = x.shape
    N = W_fp4.shape[0]
    if W_fp4.shape[1] * 2 != K:
        raise ValueError("W_fp4 must be [N, K/2]")
    r = 0 if alpha is None else int(alpha.shape[0])
    if r:
        _need_cuda(Ubits, "Ubits", torch.int32)
        _need_cuda(Vbits, "Vbits", torch.int32)
        _need_cuda(alpha, "alpha", torch.float32)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    else:
        _need_cuda(out, "out", torch.bfloat16)
    _check(fn, getattr(load(), fn)(
        _ptr(x), _ptr(W_fp4), _ptr(W_sf), _ptr(gscale), _ptr(Ubits if r else None),
        _ptr(Vbits if r else None), _ptr(alpha if r else None), _ptr(out), M, N, K, r,
        _stream(stream)))
    return out


def gemm(x: torch.Tensor, W_fp4: torch.Tensor, W_sf: torch.Tensor, gscale: torch.Tensor,
         Ubits: torch.Tensor | None, Vbits: torch.Tensor | None, alpha: torch.Tensor | None,
         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[M, N] (bfloat16) = FP4(x) FP4(R)^T * g + sum_i alpha_i (x . v_i) u_i."""
    return _gemm_call("biloco_gemm", x, W_fp4, W_sf, gscale, Ubits, Vbits, alpha, out, stream)


def gemm_noalloc(x: torch.Tensor, W_fp4: torch.Tensor, W_sf: torch.Tensor, gscale: torch.Tensor,
                 Ubits: torch.Tensor | None, Vbits: torch.Tensor | None,
                 alpha: torch.Tensor | None, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """gemm() whose library scratch is a fixed static device array: no device
    allocation inside the call (only `out`, when not given, is allocated here by
    PyTorch).  Overlapping calls race on that array; order them."""
    return _gemm_call("biloco_gemm_noalloc", x, W_fp4, W_sf, gscale, Ubits, Vbits, alpha, out,
                      stream)


def set_mode(mode: int):
    _check("biloco_set_mode", load().biloco_set_mode(int(mode)))


def resolve_mode(M: int, N: int, K: int, r: int) -> int:
    return int(load().biloco_resolve_mode(M, N, K, r))


def selftest_wait_timeout(stream=None):
    """Launch the bounded-wait self test (about 1 s on the GPU); biloco_last_error
    on the same stream then reports BILOCO_ERR_TIMEOUT."""
    _check("biloco_selftest_wait_timeout", load().biloco_selftest_wait_timeout(_stream(stream)))


def selftest_drop_arrivals(mask: int):
    """Make the next decode-kernel GEMM call leave out the grid arrivals in `mask`
    (1: z slices, 2: activation image); its bounded waits expire after about 1 s
    and biloco_last_error then reports BILOCO_ERR_TIMEOUT."""
    _check("biloco_selftest_drop_arrivals", load().biloco_selftest_drop_arrivals(int(mask)))


def set_launch(flags: int):
    """Launch form of the GEMM kernels: LAUNCH_PDL, LAUNCH_COOPERATIVE or both."""
    _check("biloco_set_launch", load().biloco_set_launch(int(flags)))


def set_correction(arith: int):
    """Correction arithmetic of the 1-2-row U side: CORR_AUTO, CORR_SIGNS or CORR_LUT."""
    _check("biloco_set_correction", load().biloco_set_correction(int(arith)))


def resolve_correction(M: int, N: int, K: int, r: int) -> int:
    return int(load().biloco_resolve_correction(M, N, K, r))


def get_launch() -> int:
    return int(load().biloco_get_launch())


def last_error(stream=None) -> int:
    return int(load().biloco_last_error(_stream(stream)))


def gemm_kernel_count(M: int, N: int, K: int, r: int) -> int:
    n = int(load().biloco_gemm_kernel_count(M, N, K, r))
    _check("biloco_gemm_kernel_count", min(n, 0))
    return n


def shutdown():
    if _lib is not None:
        _lib.biloco_shutdown()
