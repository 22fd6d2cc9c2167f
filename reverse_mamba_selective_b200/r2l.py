"""Thin ctypes binding of libr2l.so (include/r2l.h): argument marshalling only.

Every step of the computation runs in the CUDA kernels of libr2l.so.  PyTorch is
used for device memory and the current CUDA stream.  There is no CPU fallback:
if the library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libr2l.so")

R2L_OK, R2L_ERR_INVALID_ARG, R2L_ERR_UNSUPPORTED, R2L_ERR_CUDA, R2L_ERR_TIMEOUT = range(5)
R2L_F32, R2L_BF16 = 0, 1

_DTYPE_CODE = {torch.float32: R2L_F32, torch.bfloat16: R2L_BF16}
_CODE_DTYPE = {R2L_F32: torch.float32, R2L_BF16: torch.bfloat16}


class R2LError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if status == R2L_ERR_CUDA:
            msg += f" [{load().r2l_last_error().decode()}]"
        super().__init__(msg)


class ScanArgs(ctypes.Structure):
    """Mirror of r2l_scan_args."""

    _fields_ = [
        ("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("block_len", ctypes.c_int),
        ("d_inner", ctypes.c_int), ("d_state", ctypes.c_int), ("conv_width", ctypes.c_int),
        ("in_dtype", ctypes.c_int),
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("B", ctypes.c_void_p), ("C", ctypes.c_void_p),
        ("z", ctypes.c_void_p),
        ("A", ctypes.c_void_p), ("D", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
        ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load libr2l.so (built in-tree by reverse_mamba_selective_b200._build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libr2l.so not found at {LIB_PATH}; build it with "
                          "`python -m reverse_mamba_selective_b200._build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.r2l_scan_block.argtypes = [ctypes.POINTER(ScanArgs), vp, ci, vp]
    lib.r2l_scan_block.restype = ci
    lib.fwd_scan_from_state.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanArgs), vp, vp, vp, ci, vp]
    lib.fwd_scan_from_state.restype = ci
    lib.r2l_residual_apply.argtypes = [vp, vp, vp, cf, ci, ci, ci, ci, vp]
    lib.r2l_residual_apply.restype = ci
    lib.r2l_status_string.argtypes = [ci]
    lib.r2l_status_string.restype = ctypes.c_char_p
    lib.r2l_device_status.argtypes = [vp]
    lib.r2l_device_status.restype = ci
    lib.r2l_last_error.argtypes = []
    lib.r2l_last_error.restype = ctypes.c_char_p
    lib.r2l_abi_version.argtypes = []
    lib.r2l_abi_version.restype = ci
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().r2l_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check_dev(name: str, t: Optional[torch.Tensor], dtype=None, shape=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def make_scan_args(x, dt, B, C, z, A, D, dt_bias, conv_w=None, conv_b=None, block_len=None) -> ScanArgs:
    """Build an r2l_scan_args from device tensors (x, dt, z [b, L, d]; B, C [b, L, n])."""
    batch, seqlen, d_inner = x.shape
    d_state = B.shape[-1]
    io = x.dtype
    if io not in _DTYPE_CODE:
        raise TypeError(f"unsupported input dtype {io}")
    for name, t in (("x", x), ("dt", dt), ("z", z)):
        _check_dev(name, t, io, (batch, seqlen, d_inner))
    for name, t in (("B", B), ("C", C)):
        _check_dev(name, t, io, (batch, seqlen, d_state))
    _check_dev("A", A, torch.float32, (d_inner, d_state))
    _check_dev("D", D, torch.float32, (d_inner,))
    _check_dev("dt_bias", dt_bias, torch.float32, (d_inner,))
    conv_width = 0 if conv_w is None else conv_w.shape[-1]
    _check_dev("conv_w", conv_w, torch.float32, (d_inner, conv_width) if conv_w is not None else None)
    _check_dev("conv_b", conv_b, torch.float32, (d_inner,) if conv_b is not None else None)
    return ScanArgs(batch, seqlen, seqlen if block_len is None else int(block_len), d_inner, d_state, conv_width,
                    _DTYPE_CODE[io], _ptr(x), _ptr(dt), _ptr(B), _ptr(C), _ptr(z), _ptr(A), _ptr(D),
                    _ptr(dt_bias), _ptr(conv_w), _ptr(conv_b))


def _raise(st: int, where: str):
    if st != R2L_OK:
        raise R2LError(st, where)


def r2l_scan_block(x, dt, B, C, z, A, D, dt_bias, conv_w=None, conv_b=None, *, block_len: int,
                   y: Optional[torch.Tensor] = None, y_dtype: Optional[torch.dtype] = None,
                   stream=None) -> torch.Tensor:
    """Right-to-left selective scan over blocks of ``block_len`` tokens; returns y [b, L, d]."""
    lib = load()
    args = make_scan_args(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, block_len)
    y_dtype = y_dtype or (y.dtype if y is not None else x.dtype)
    if y is None:
        y = torch.empty(x.shape, dtype=y_dtype, device=x.device)
    _check_dev("y", y, y_dtype, x.shape)
    _raise(lib.r2l_scan_block(ctypes.byref(args), _ptr(y), _DTYPE_CODE[y_dtype], _stream(stream)),
           "r2l_scan_block")
    return y


def fwd_scan_from_state(x, z, fwd: Dict[str, torch.Tensor], rev: Optional[Dict[str, torch.Tensor]] = None, *,
                        h0: Optional[torch.Tensor] = None, h_last: Optional[torch.Tensor] = None,
                        want_h_last: bool = True, rev_block_len: Optional[int] = None,
                        y: Optional[torch.Tensor] = None, y_dtype: Optional[torch.dtype] = None,
                        stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Forward scan resumed from ``h0`` (+ optional fused block-confined reverse).

    ``fwd``/``rev`` hold dt, B, C, A, D, dt_bias (and optional conv_w, conv_b); x, z shared.
    Returns (y, h_last).
    """
    lib = load()
    fa = make_scan_args(x, fwd["dt"], fwd["B"], fwd["C"], z, fwd["A"], fwd["D"], fwd["dt_bias"],
                        fwd.get("conv_w"), fwd.get("conv_b"))
    ra = None
    if rev is not None:
        ra = make_scan_args(x, rev["dt"], rev["B"], rev["C"], z, rev["A"], rev["D"], rev["dt_bias"],
                            rev.get("conv_w"), rev.get("conv_b"),
                            rev_block_len if rev_block_len is not None else x.shape[1])
    batch, seqlen, d_inner = x.shape
    d_state = fwd["B"].shape[-1]
    _check_dev("h0", h0, torch.float32, (batch, d_inner, d_state))
    if h_last is None and want_h_last:
        h_last = torch.empty((batch, d_inner, d_state), dtype=torch.float32, device=x.device)
    _check_dev("h_last", h_last, torch.float32, (batch, d_inner, d_state))
    y_dtype = y_dtype or (y.dtype if y is not None else x.dtype)
    if y is None:
        y = torch.empty(x.shape, dtype=y_dtype, device=x.device)
    _check_dev("y", y, y_dtype, x.shape)
    st = lib.fwd_scan_from_state(ctypes.byref(fa), ctypes.byref(ra) if ra is not None else None,
                                 _ptr(h0), _ptr(h_last), _ptr(y), _DTYPE_CODE[y_dtype], _stream(stream))
    _raise(st, "fwd_scan_from_state")
    return y, h_last


def r2l_residual_apply(hidden: torch.Tensor, y: torch.Tensor, W_out: torch.Tensor, s: float,
                       stream=None) -> torch.Tensor:
    """hidden <- hidden + s * y @ W_out^T, in place; returns hidden."""
    lib = load()
    M, d_model = hidden.shape
    d_inner = y.shape[-1]
    _check_dev("hidden", hidden)
    _check_dev("y", y, hidden.dtype, (M, d_inner))
    _check_dev("W_out", W_out, hidden.dtype, (d_model, d_inner))
    if hidden.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported dtype {hidden.dtype}")
    st = lib.r2l_residual_apply(_ptr(hidden), _ptr(y), _ptr(W_out), float(s), M, d_model, d_inner,
                                _DTYPE_CODE[hidden.dtype], _stream(stream))
    _raise(st, "r2l_residual_apply")
    return hidden


def r2l_device_status(stream=None) -> int:
    """Synchronise and read/clear the library's device status word (R2L_OK or R2L_ERR_TIMEOUT)."""
    return int(load().r2l_device_status(_stream(stream)))


def r2l_abi_version() -> int:
    return int(load().r2l_abi_version())
