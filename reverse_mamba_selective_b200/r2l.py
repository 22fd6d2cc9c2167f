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
        ("conv_state", ctypes.c_void_p), ("conv_state_out", ctypes.c_void_p),
    ]


class SidecarWeights(ctypes.Structure):
    """Mirror of r2l_sidecar_weights."""

    _fields_ = [
        ("d_model", ctypes.c_int), ("d_inner", ctypes.c_int), ("d_state", ctypes.c_int),
        ("dt_rank", ctypes.c_int), ("conv_width", ctypes.c_int),
        ("W_in", ctypes.c_void_p), ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p),
        ("W_x", ctypes.c_void_p), ("W_dt", ctypes.c_void_p),
        ("A", ctypes.c_void_p), ("D", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
        ("W_out", ctypes.c_void_p),
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
    lib.r2l_decode_step.argtypes = [ctypes.POINTER(ScanArgs), vp, vp, vp, cf, ci, ci, vp]
    lib.r2l_decode_step.restype = ci
    lib.r2l_status_string.argtypes = [ci]
    lib.r2l_status_string.restype = ctypes.c_char_p
    lib.r2l_device_status.argtypes = [vp]
    lib.r2l_device_status.restype = ci
    lib.r2l_last_error.argtypes = []
    lib.r2l_last_error.restype = ctypes.c_char_p
    lib.r2l_wait_selftest.argtypes = [vp]
    lib.r2l_wait_selftest.restype = ci
    lib.r2l_abi_version.argtypes = []
    lib.r2l_abi_version.restype = ci
    sz = ctypes.c_size_t
    lib.r2l_in_proj.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, vp, vp, vp]
    lib.r2l_in_proj.restype = ci
    lib.r2l_x_proj_workspace_size.argtypes = [ci, ci, ci, ci]
    lib.r2l_x_proj_workspace_size.restype = sz
    lib.r2l_x_proj.argtypes = [vp, vp, ci, ci, ci, ci, vp, vp, vp, vp, sz, vp]
    lib.r2l_x_proj.restype = ci
    lib.r2l_x_proj_noalloc.argtypes = [vp, vp, ci, ci, ci, ci, vp, vp, vp, vp]
    lib.r2l_x_proj_noalloc.restype = ci
    lib.r2l_bidir_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs)]
    lib.r2l_bidir_scan_workspace_size.restype = ctypes.c_size_t
    lib.r2l_bidir_scan.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ScanArgs), vp, vp, vp, ci, vp,
                                   ctypes.c_size_t, vp]
    lib.r2l_bidir_scan.restype = ci
    lib.r2l_scan_block_bwd.argtypes = [ctypes.POINTER(ScanArgs), vp, ci] + [vp] * 10 + [vp]
    lib.r2l_scan_block_bwd.restype = ci
    lib.r2l_dt_proj.argtypes = [vp, vp, ci, ci, ci, vp, vp]
    lib.r2l_dt_proj.restype = ci
    lib.r2l_sidecar_workspace_size.argtypes = [ctypes.POINTER(SidecarWeights), ci, ci]
    lib.r2l_sidecar_workspace_size.restype = sz
    lib.r2l_sidecar_forward.argtypes = [ctypes.POINTER(SidecarWeights), ci, ci, ci, cf, vp, vp, sz, vp]
    lib.r2l_sidecar_forward.restype = ci
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


def make_scan_args(x, dt, B, C, z, A, D, dt_bias, conv_w=None, conv_b=None, block_len=None,
                   conv_state=None, conv_state_out=None) -> ScanArgs:
    """Build an r2l_scan_args from device tensors (x, dt, z [b, L, d]; B, C [b, L, n];
    conv_state / conv_state_out [b, d, conv_width - 1] fp32 for forward scans)."""
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
    cs_shape = (batch, d_inner, max(conv_width - 1, 0))
    _check_dev("conv_state", conv_state, torch.float32, cs_shape)
    _check_dev("conv_state_out", conv_state_out, torch.float32, cs_shape)
    return ScanArgs(batch, seqlen, seqlen if block_len is None else int(block_len), d_inner, d_state, conv_width,
                    _DTYPE_CODE[io], _ptr(x), _ptr(dt), _ptr(B), _ptr(C), _ptr(z), _ptr(A), _ptr(D),
                    _ptr(dt_bias), _ptr(conv_w), _ptr(conv_b), _ptr(conv_state), _ptr(conv_state_out))


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
    ``fwd`` may also hold ``conv_state`` / ``conv_state_out`` (the convolution's cached tokens).
    Returns (y, h_last).
    """
    lib = load()
    fa = make_scan_args(x, fwd["dt"], fwd["B"], fwd["C"], z, fwd["A"], fwd["D"], fwd["dt_bias"],
                        fwd.get("conv_w"), fwd.get("conv_b"), conv_state=fwd.get("conv_state"),
                        conv_state_out=fwd.get("conv_state_out"))
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


def r2l_scan_block_bwd(x, dt, B, C, z, A, D, dt_bias, dy, *, block_len: int, conv_w=None, conv_b=None,
                       stream=None) -> Dict[str, torch.Tensor]:
    """Gradients of r2l_scan_block (with the width-4 convolution when conv_w, conv_b are given)
    given dy = dL/dy; all fp32.

    Returns dx, ddt, dB, dC, dz (None without a gate), dA, dD, ddt_bias, dconv_w and dconv_b (None
    without the convolution).
    """
    lib = load()
    a = make_scan_args(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, block_len)
    batch, seqlen, d_inner = x.shape
    d_state = B.shape[-1]
    _check_dev("dy", dy, None, x.shape)
    if dy.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported dy dtype {dy.dtype}")
    f32 = dict(dtype=torch.float32, device=x.device)
    g = {"dx": torch.empty(x.shape, **f32), "ddt": torch.empty(x.shape, **f32),
         "dB": torch.empty((batch, seqlen, d_state), **f32), "dC": torch.empty((batch, seqlen, d_state), **f32),
         "dz": torch.empty(x.shape, **f32) if z is not None else None,
         "dA": torch.empty((d_inner, d_state), **f32), "dD": torch.empty(d_inner, **f32),
         "ddt_bias": torch.empty(d_inner, **f32),
         "dconv_w": torch.empty((d_inner, 4), **f32) if conv_w is not None else None,
         "dconv_b": torch.empty(d_inner, **f32) if conv_w is not None else None}
    st = lib.r2l_scan_block_bwd(ctypes.byref(a), _ptr(dy), _DTYPE_CODE[dy.dtype], _ptr(g["dx"]), _ptr(g["ddt"]),
                                _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dz"]), _ptr(g["dA"]), _ptr(g["dD"]),
                                _ptr(g["ddt_bias"]), _ptr(g["dconv_w"]), _ptr(g["dconv_b"]), _stream(stream))
    _raise(st, "r2l_scan_block_bwd")
    return g


def bidir_scan(x, z, fwd: Dict[str, torch.Tensor], rev: Dict[str, torch.Tensor], *, rev_block_len: int,
               h0: Optional[torch.Tensor] = None, h_last: Optional[torch.Tensor] = None, want_h_last: bool = True,
               y: Optional[torch.Tensor] = None, y_dtype: Optional[torch.dtype] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """(y_f + y_r) * SiLU(z) for any reverse block length (rev_block_len = seqlen: the whole window).

    Same arguments as fwd_scan_from_state; the two directions run as separate ungated scans into
    ``workspace`` (allocated here when omitted).  Returns (y, h_last).
    """
    lib = load()
    fa = make_scan_args(x, fwd["dt"], fwd["B"], fwd["C"], z, fwd["A"], fwd["D"], fwd["dt_bias"],
                        fwd.get("conv_w"), fwd.get("conv_b"), conv_state=fwd.get("conv_state"),
                        conv_state_out=fwd.get("conv_state_out"))
    ra = make_scan_args(x, rev["dt"], rev["B"], rev["C"], z, rev["A"], rev["D"], rev["dt_bias"],
                        rev.get("conv_w"), rev.get("conv_b"), rev_block_len)
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
    need = int(lib.r2l_bidir_scan_workspace_size(ctypes.byref(fa)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    st = lib.r2l_bidir_scan(ctypes.byref(fa), ctypes.byref(ra), _ptr(h0), _ptr(h_last), _ptr(y), _DTYPE_CODE[y_dtype],
                            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _raise(st, "r2l_bidir_scan")
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


def r2l_decode_step(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, hidden: torch.Tensor, W_out: torch.Tensor,
                    s: float, *, block_len: int, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step: y = r2l_scan_block(...), then hidden <- hidden + s * y @ W_out^T in place
    (W_out and hidden pulled into L2 while the scan runs).  hidden is [b * L, d_model] or
    [b, L, d_model]; returns y."""
    lib = load()
    args = make_scan_args(x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, block_len)
    dtype = hidden.dtype
    if dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported dtype {dtype}")
    if y is None:
        y = torch.empty(x.shape, dtype=dtype, device=x.device)
    _check_dev("y", y, dtype, x.shape)
    batch, seqlen, d_inner = x.shape
    d_model = hidden.shape[-1]
    _check_dev("hidden", hidden, dtype, (batch * seqlen, d_model) if hidden.dim() == 2 else (batch, seqlen, d_model))
    _check_dev("W_out", W_out, dtype, (d_model, d_inner))
    st = lib.r2l_decode_step(ctypes.byref(args), _ptr(y), _ptr(hidden), _ptr(W_out), float(s), d_model,
                             _DTYPE_CODE[dtype], _stream(stream))
    _raise(st, "r2l_decode_step")
    return y


def r2l_device_status(stream=None) -> int:
    """Synchronise and read/clear the library's device status word (R2L_OK or R2L_ERR_TIMEOUT)."""
    return int(load().r2l_device_status(_stream(stream)))


def r2l_wait_selftest(stream=None) -> None:
    """Enqueue the bounded-wait self-test (see r2l.h); r2l_device_status() then reports the timeout."""
    _raise(load().r2l_wait_selftest(_stream(stream)), "r2l_wait_selftest")


def r2l_abi_version() -> int:
    return int(load().r2l_abi_version())


# ----------------------------------------------------------------------------- sidecar front-end

def r2l_in_proj(hidden: torch.Tensor, W_in: torch.Tensor, conv_w: Optional[torch.Tensor],
                conv_b: Optional[torch.Tensor], batch: int, seqlen: int, block_len: int,
                u: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """u = SiLU(conv(x)) (right to left inside each block) and z from hidden [M, d_model] (bf16)."""
    lib = load()
    M, d_model = hidden.shape
    d_inner = W_in.shape[0] // 2
    _check_dev("hidden", hidden, torch.bfloat16)
    _check_dev("W_in", W_in, torch.bfloat16, (2 * d_inner, d_model))
    _check_dev("conv_w", conv_w, torch.float32, (d_inner, 4) if conv_w is not None else None)
    _check_dev("conv_b", conv_b, torch.float32, (d_inner,) if conv_b is not None else None)
    if M != batch * seqlen:
        raise ValueError("hidden must have batch * seqlen rows")
    u = torch.empty((M, d_inner), dtype=torch.bfloat16, device=hidden.device) if u is None else u
    z = torch.empty((M, d_inner), dtype=torch.bfloat16, device=hidden.device) if z is None else z
    _check_dev("u", u, torch.bfloat16, (M, d_inner))
    _check_dev("z", z, torch.bfloat16, (M, d_inner))
    st = lib.r2l_in_proj(_ptr(hidden), _ptr(W_in), _ptr(conv_w), _ptr(conv_b), batch, seqlen, block_len, d_model,
                         d_inner, _ptr(u), _ptr(z), _stream(stream))
    _raise(st, "r2l_in_proj")
    return u, z


def r2l_x_proj(u: torch.Tensor, W_x: torch.Tensor, dt_rank: int, workspace: Optional[torch.Tensor] = None,
               stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(dt_low [M, dt_rank], B [M, d_state], C [M, d_state]) = split(u @ W_x^T) (bf16)."""
    lib = load()
    M, d_inner = u.shape
    d_state = (W_x.shape[0] - dt_rank) // 2
    _check_dev("u", u, torch.bfloat16)
    _check_dev("W_x", W_x, torch.bfloat16, (dt_rank + 2 * d_state, d_inner))
    need = int(lib.r2l_x_proj_workspace_size(M, d_inner, dt_rank, d_state))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=u.device)
    dev = u.device
    dt_low = torch.empty((M, dt_rank), dtype=torch.bfloat16, device=dev)
    B = torch.empty((M, d_state), dtype=torch.bfloat16, device=dev)
    C = torch.empty((M, d_state), dtype=torch.bfloat16, device=dev)
    st = lib.r2l_x_proj(_ptr(u), _ptr(W_x), M, d_inner, dt_rank, d_state, _ptr(dt_low), _ptr(B), _ptr(C),
                        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _raise(st, "r2l_x_proj")
    return dt_low, B, C


def r2l_x_proj_noalloc(u: torch.Tensor, W_x: torch.Tensor, dt_rank: int,
                       stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """r2l_x_proj with the split reduction's partial sums in the library's own device scratch."""
    lib = load()
    M, d_inner = u.shape
    d_state = (W_x.shape[0] - dt_rank) // 2
    _check_dev("u", u, torch.bfloat16)
    _check_dev("W_x", W_x, torch.bfloat16, (dt_rank + 2 * d_state, d_inner))
    dev = u.device
    dt_low = torch.empty((M, dt_rank), dtype=torch.bfloat16, device=dev)
    B = torch.empty((M, d_state), dtype=torch.bfloat16, device=dev)
    C = torch.empty((M, d_state), dtype=torch.bfloat16, device=dev)
    st = lib.r2l_x_proj_noalloc(_ptr(u), _ptr(W_x), M, d_inner, dt_rank, d_state, _ptr(dt_low), _ptr(B), _ptr(C),
                                _stream(stream))
    _raise(st, "r2l_x_proj_noalloc")
    return dt_low, B, C


def r2l_dt_proj(dt_low: torch.Tensor, W_dt: torch.Tensor, stream=None) -> torch.Tensor:
    """dt [M, d_inner] = dt_low @ W_dt^T (bf16)."""
    lib = load()
    M, dt_rank = dt_low.shape
    d_inner = W_dt.shape[0]
    _check_dev("dt_low", dt_low, torch.bfloat16)
    _check_dev("W_dt", W_dt, torch.bfloat16, (d_inner, dt_rank))
    dt = torch.empty((M, d_inner), dtype=torch.bfloat16, device=dt_low.device)
    st = lib.r2l_dt_proj(_ptr(dt_low), _ptr(W_dt), M, dt_rank, d_inner, _ptr(dt), _stream(stream))
    _raise(st, "r2l_dt_proj")
    return dt


def make_sidecar_weights(w: Dict[str, Optional[torch.Tensor]]) -> SidecarWeights:
    """r2l_sidecar_weights from device tensors W_in, conv_w, conv_b, W_x, W_dt, A, D, dt_bias, W_out."""
    d2, d_model = w["W_in"].shape
    d_inner = d2 // 2
    d_state = w["A"].shape[1]
    dt_rank = w["W_dt"].shape[1]
    for k in ("W_in", "W_x", "W_dt", "W_out"):
        _check_dev(k, w[k], torch.bfloat16)
    _check_dev("W_x", w["W_x"], torch.bfloat16, (dt_rank + 2 * d_state, d_inner))
    _check_dev("W_out", w["W_out"], torch.bfloat16, (d_model, d_inner))
    for k in ("A", "D", "dt_bias"):
        _check_dev(k, w[k], torch.float32)
    conv_w = w.get("conv_w")
    _check_dev("conv_w", conv_w, torch.float32, (d_inner, 4) if conv_w is not None else None)
    return SidecarWeights(d_model, d_inner, d_state, dt_rank, 0 if conv_w is None else 4,
                          _ptr(w["W_in"]), _ptr(conv_w), _ptr(w.get("conv_b")), _ptr(w["W_x"]), _ptr(w["W_dt"]),
                          _ptr(w["A"]), _ptr(w["D"]), _ptr(w["dt_bias"]), _ptr(w["W_out"]))


def sidecar_workspace_size(sw: SidecarWeights, batch: int, seqlen: int) -> int:
    return int(load().r2l_sidecar_workspace_size(ctypes.byref(sw), batch, seqlen))


def r2l_sidecar_forward(hidden: torch.Tensor, weights, batch: int, seqlen: int, block_len: int, s: float,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """hidden [batch*seqlen, d_model] (bf16) += s * sidecar(hidden), in place; returns hidden.

    ``weights`` is a dict of device tensors or a prebuilt SidecarWeights; ``workspace`` a device
    byte buffer of at least sidecar_workspace_size bytes (allocated here when omitted).
    """
    lib = load()
    sw = weights if isinstance(weights, SidecarWeights) else make_sidecar_weights(weights)
    _check_dev("hidden", hidden, torch.bfloat16, (batch * seqlen, sw.d_model))
    if workspace is None:
        workspace = torch.empty(max(sidecar_workspace_size(sw, batch, seqlen), 256), dtype=torch.uint8,
                                device=hidden.device)
    st = lib.r2l_sidecar_forward(ctypes.byref(sw), batch, seqlen, block_len, float(s), _ptr(hidden),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _raise(st, "r2l_sidecar_forward")
    return hidden
