"""fp64 CPU oracle of the right-to-left selective-scan sidecar.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The GPU library does not
import, link or call it, and it shares no code with the GPU path.

The arithmetic lives in ``r2l_oracle.c`` (plain C, double precision, built with
``-ffp-contract=off`` so the compiler keeps the written operation order).  This
module only compiles it, marshals numpy arrays and composes the two directions
of the partial-bidirectional mixer.

Parity pins (tests/test_oracle_pins.py) tie every function here to closed forms,
brute force, library routines and the invariants the pages state; no function
is "parity unpinned".
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "r2l_oracle.c")
_LIB = os.path.join(_HERE, "libr2l_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # R2L_ORACLE_LIB lets the mutation test load a deliberately broken copy.
        path = os.environ.get("R2L_ORACLE_LIB") or build()
        lib = ctypes.CDLL(path)
        dp = ctypes.c_void_p
        L = ctypes.c_long
        lib.r2l_oracle_scan.argtypes = [ctypes.c_int, L, L, L, L, L, L] + [dp] * 13
        lib.r2l_oracle_scan.restype = ctypes.c_int
        lib.r2l_oracle_residual.argtypes = [L, L, L, dp, dp, dp, ctypes.c_double, dp]
        lib.r2l_oracle_residual.restype = ctypes.c_int
        _lib = lib
    return _lib


def _c(a: Optional[np.ndarray]):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def scan(x, dt, B, C, z, A, D, dt_bias, conv_w=None, conv_b=None, *, reverse: bool = True,
         block_len: Optional[int] = None, h0=None, want_h_last: bool = False):
    """Selective scan of ``x`` [batch, seqlen, d_inner] (see r2l_oracle.c for the definition).

    Returns ``y`` or ``(y, h_last)`` when ``want_h_last`` (forward scans only).
    """
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    batch, seqlen, d_inner = x.shape
    d_state = np.shape(A)[1]
    conv_width = 0 if conv_w is None else np.shape(conv_w)[1]
    if block_len is None:
        block_len = seqlen
    keep = []
    ptrs = []
    for a in (x, dt, B, C, z, A, D, dt_bias, conv_w, conv_b, h0):
        arr, p = _c(a)
        keep.append(arr)
        ptrs.append(p)
    h_last = np.zeros((batch, d_inner, d_state)) if want_h_last else None
    y = np.zeros((batch, seqlen, d_inner))
    rc = lib.r2l_oracle_scan(1 if reverse else 0, batch, seqlen, block_len, d_inner, d_state,
                             conv_width, *ptrs,
                             None if h_last is None else h_last.ctypes.data_as(ctypes.c_void_p),
                             y.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("r2l_oracle_scan rejected its arguments")
    return (y, h_last) if want_h_last else y


def silu(v):
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def mamba_h(x, z, fwd: dict, rev: Optional[dict], h0=None, block_len: Optional[int] = None
            ) -> Tuple[np.ndarray, np.ndarray]:
    """Partial-bidirectional mixer ("Training Hybrid Block Diffusion Language Models with
    Partial Bidirectionality", Methodology item 1): forward scan resumed from the cached
    boundary state ``h0`` plus a reverse scan confined to each active block; the two
    direction outputs are summed before the single output gate SiLU(z).

    ``fwd``/``rev`` hold each direction's own dt, B, C, A, D, dt_bias (and optional
    conv_w/conv_b); x and z are shared.  Returns (y, h_last).
    """
    y_f, h_last = scan(x, fwd["dt"], fwd["B"], fwd["C"], None, fwd["A"], fwd["D"], fwd["dt_bias"],
                       fwd.get("conv_w"), fwd.get("conv_b"), reverse=False, h0=h0, want_h_last=True)
    y = y_f
    if rev is not None:
        y_r = scan(x, rev["dt"], rev["B"], rev["C"], None, rev["A"], rev["D"], rev["dt_bias"],
                   rev.get("conv_w"), rev.get("conv_b"), reverse=True, block_len=block_len)
        y = y_f + y_r
    if z is not None:
        y = y * silu(z)
    return y, h_last


def residual(hidden, y, W_out, s: float) -> np.ndarray:
    """out = hidden + s * y @ W_out^T  (R2LM residual correction gated by s)."""
    lib = _load()
    hidden = np.ascontiguousarray(hidden, dtype=np.float64)
    y = np.ascontiguousarray(y, dtype=np.float64)
    W_out = np.ascontiguousarray(W_out, dtype=np.float64)
    M, d_model = hidden.shape
    d_inner = y.shape[1]
    out = np.empty_like(hidden)
    rc = lib.r2l_oracle_residual(M, d_model, d_inner, hidden.ctypes.data_as(ctypes.c_void_p),
                                 y.ctypes.data_as(ctypes.c_void_p), W_out.ctypes.data_as(ctypes.c_void_p),
                                 float(s), out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("r2l_oracle_residual rejected its arguments")
    return out
