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
        lib.r2l_oracle_scan.argtypes = [ctypes.c_int, L, L, L, L, L, L] + [dp] * 15
        lib.r2l_oracle_scan.restype = ctypes.c_int
        lib.r2l_oracle_residual.argtypes = [L, L, L, dp, dp, dp, ctypes.c_double, dp]
        lib.r2l_oracle_residual.restype = ctypes.c_int
        lib.r2l_oracle_linear.argtypes = [L, L, L, dp, dp, dp]
        lib.r2l_oracle_linear.restype = ctypes.c_int
        lib.r2l_oracle_conv_silu.argtypes = [ctypes.c_int, L, L, L, L, L, dp, dp, dp, dp]
        lib.r2l_oracle_conv_silu.restype = ctypes.c_int
        lib.r2l_oracle_scan_bwd.argtypes = [L, L, L, L, L, L] + [dp] * 21
        lib.r2l_oracle_scan_bwd.restype = ctypes.c_int
        _lib = lib
    return _lib


def _c(a: Optional[np.ndarray]):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def scan(x, dt, B, C, z, A, D, dt_bias, conv_w=None, conv_b=None, *, reverse: bool = True,
         block_len: Optional[int] = None, h0=None, want_h_last: bool = False, conv_state=None,
         want_conv_state: bool = False):
    """Selective scan of ``x`` [batch, seqlen, d_inner] (see r2l_oracle.c for the definition).

    Returns ``y``, with ``h_last`` and then ``conv_state_out`` appended (as a tuple) when
    ``want_h_last`` / ``want_conv_state`` are set (forward scans only).
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
    cs_in, cs_ptr = _c(conv_state)
    h_last = np.zeros((batch, d_inner, d_state)) if want_h_last else None
    cs_out = np.zeros((batch, d_inner, max(conv_width - 1, 0))) if want_conv_state else None
    y = np.zeros((batch, seqlen, d_inner))

    def _p(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    rc = lib.r2l_oracle_scan(1 if reverse else 0, batch, seqlen, block_len, d_inner, d_state,
                             conv_width, *ptrs, _p(h_last), cs_ptr, _p(cs_out), _p(y))
    if rc != 0:
        raise ValueError("r2l_oracle_scan rejected its arguments")
    extra = ([h_last] if want_h_last else []) + ([cs_out] if want_conv_state else [])
    return tuple([y] + extra) if extra else y


def silu(v):
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def mamba_h(x, z, fwd: dict, rev: Optional[dict], h0=None, block_len: Optional[int] = None,
            want_conv_state: bool = False) -> Tuple[np.ndarray, ...]:
    """Partial-bidirectional mixer ("Training Hybrid Block Diffusion Language Models with
    Partial Bidirectionality", Methodology item 1): forward scan resumed from the cached
    boundary state ``h0`` plus a reverse scan confined to each active block; the two
    direction outputs are summed before the single output gate SiLU(z).

    ``fwd``/``rev`` hold each direction's own dt, B, C, A, D, dt_bias (and optional
    conv_w/conv_b); x and z are shared.  ``fwd`` may hold ``conv_state``, the forward
    convolution's cached prefix inputs.  Returns (y, h_last), plus the forward
    direction's new convolution state when ``want_conv_state``.
    """
    res = scan(x, fwd["dt"], fwd["B"], fwd["C"], None, fwd["A"], fwd["D"], fwd["dt_bias"],
               fwd.get("conv_w"), fwd.get("conv_b"), reverse=False, h0=h0, want_h_last=True,
               conv_state=fwd.get("conv_state"), want_conv_state=want_conv_state)
    y_f, h_last = res[0], res[1]
    y = y_f
    if rev is not None:
        y_r = scan(x, rev["dt"], rev["B"], rev["C"], None, rev["A"], rev["D"], rev["dt_bias"],
                   rev.get("conv_w"), rev.get("conv_b"), reverse=True, block_len=block_len)
        y = y_f + y_r
    if z is not None:
        y = y * silu(z)
    return (y, h_last, res[2]) if want_conv_state else (y, h_last)


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


def linear(X, W) -> np.ndarray:
    """out = X @ W^T in fp64 (X [M, K], W [N, K])."""
    lib = _load()
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = X.shape
    N = W.shape[0]
    out = np.empty((M, N))
    rc = lib.r2l_oracle_linear(M, N, K, X.ctypes.data_as(ctypes.c_void_p), W.ctypes.data_as(ctypes.c_void_p),
                               out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0 or W.shape[1] != K:
        raise ValueError("r2l_oracle_linear rejected its arguments")
    return out


def conv_silu(x, conv_w, conv_b, *, reverse: bool = True, block_len: Optional[int] = None) -> np.ndarray:
    """u = SiLU(conv(x)) of x [batch, seqlen, d_inner], causal in scan order (see r2l_oracle.c)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    conv_w = np.ascontiguousarray(conv_w, dtype=np.float64)
    conv_b = np.ascontiguousarray(conv_b, dtype=np.float64)
    batch, seqlen, d_inner = x.shape
    u = np.empty_like(x)
    rc = lib.r2l_oracle_conv_silu(1 if reverse else 0, batch, seqlen, seqlen if block_len is None else block_len,
                                  d_inner, conv_w.shape[1], x.ctypes.data_as(ctypes.c_void_p),
                                  conv_w.ctypes.data_as(ctypes.c_void_p), conv_b.ctypes.data_as(ctypes.c_void_p),
                                  u.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("r2l_oracle_conv_silu rejected its arguments")
    return u


def round_bf16(a) -> np.ndarray:
    """Each element rounded to the nearest bfloat16 value (ties to even) the way a bf16 store of an
    fp32 value is: fp64 -> fp32 (nearest), then bf16 keeps fp32's sign and exponent and the top 7 of
    its 23 mantissa bits, rounding the 16 dropped bits to nearest, ties to even.  Returns fp64."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    bits = a32.view(np.uint32).astype(np.uint64)
    kept_lsb = (bits >> 16) & 1
    r = ((bits + 0x7FFF + kept_lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def sidecar(hidden, w: dict, batch: int, seqlen: int, block_len: int, s: float,
            store_bf16: bool = False) -> Tuple[np.ndarray, dict]:
    """The whole right-to-left sidecar on the active tokens, hidden [batch*seqlen, d_model] -> hidden.

    "Bifocal Diffusion Language Models", section 2: projections of the hidden states go through a
    right-to-left Mamba selective scan inside each block, and s * out_proj(y) is added back.  The
    projections are the standard Mamba-1 ones (the pages do not spell them out):
      [x | z] = hidden W_in^T (x = first d_inner columns),  u = SiLU(conv(x)) right to left,
      [dt_low | B | C] = u W_x^T (in that order),  dt = dt_low W_dt^T,
      y = scan(u, dt, B, C, z),  out = hidden + s * y W_out^T.
    ``w`` holds W_in, conv_w, conv_b (or None), W_x, W_dt, A, D, dt_bias, W_out.  Returns the new
    hidden state and the intermediates (u, z, dt_low, B, C, dt, y), each [batch*seqlen, ...].

    ``store_bf16``: a bf16 sidecar keeps its activations in bf16 between the steps, so each of z, u,
    dt_low, B, C, dt and y is rounded to bf16 (``round_bf16``) where it is produced, and the next
    step reads the rounded value.  The convolution takes the unrounded x (it is applied where x is
    produced), and every step still computes in fp64.
    """
    keep = round_bf16 if store_bf16 else (lambda a: a)
    hidden = np.asarray(hidden, dtype=np.float64)
    M = hidden.shape[0]
    d_inner = np.shape(w["W_in"])[0] // 2
    d_state = np.shape(w["A"])[1]
    dt_rank = np.shape(w["W_dt"])[1]
    xz = linear(hidden, w["W_in"])
    x, z = xz[:, :d_inner], keep(xz[:, d_inner:])
    if w.get("conv_w") is not None:
        u = conv_silu(x.reshape(batch, seqlen, d_inner), w["conv_w"], w["conv_b"], reverse=True,
                      block_len=block_len).reshape(M, d_inner)
    else:
        u = x
    u = keep(u)
    dbl = keep(linear(u, w["W_x"]))
    dt_low, Bm, Cm = dbl[:, :dt_rank], dbl[:, dt_rank:dt_rank + d_state], dbl[:, dt_rank + d_state:]
    dt = keep(linear(dt_low, w["W_dt"]))
    r3 = lambda a: np.ascontiguousarray(a).reshape(batch, seqlen, -1)
    y = keep(scan(r3(u), r3(dt), r3(Bm), r3(Cm), r3(z), w["A"], w["D"], w["dt_bias"], None, None, reverse=True,
                  block_len=block_len).reshape(M, d_inner))
    out = residual(hidden, y, w["W_out"], s)
    return out, {"u": u, "z": z, "dt_low": dt_low, "B": Bm, "C": Cm, "dt": dt, "y": y}


def scan_bwd(x, dt, B, C, z, A, D, dt_bias, dy, *, block_len: Optional[int] = None, conv_w=None,
             conv_b=None) -> dict:
    """Gradients of the right-to-left block scan given dL/dy (see r2l_oracle.c), with the width-W
    convolution front-end when conv_w [d_inner][W] and conv_b [d_inner] are given.

    Returns a dict with dx, ddt, dB, dC, dz (None without a gate), dA, dD, ddt_bias, dconv_w and
    dconv_b (both None without the convolution).
    """
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    batch, seqlen, d_inner = x.shape
    d_state = np.shape(A)[1]
    if (conv_w is None) != (conv_b is None):
        raise ValueError("conv_w and conv_b go together")
    W = 0 if conv_w is None else np.shape(conv_w)[1]
    ins = [np.ascontiguousarray(a, dtype=np.float64) if a is not None else None
           for a in (dt, B, C, z, A, D, dt_bias, conv_w, conv_b, dy)]
    out = {"dx": np.empty_like(x), "ddt": np.empty_like(x), "dB": np.empty((batch, seqlen, d_state)),
           "dC": np.empty((batch, seqlen, d_state)), "dz": np.empty_like(x) if z is not None else None,
           "dA": np.empty((d_inner, d_state)), "dD": np.empty(d_inner), "ddt_bias": np.empty(d_inner),
           "dconv_w": np.empty((d_inner, W)) if W else None, "dconv_b": np.empty(d_inner) if W else None}
    p = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.r2l_oracle_scan_bwd(batch, seqlen, seqlen if block_len is None else block_len, d_inner, d_state, W,
                                 p(x), *[p(a) for a in ins],
                                 *[p(out[k]) for k in ("dx", "ddt", "dB", "dC", "dz", "dA", "dD", "ddt_bias",
                                                       "dconv_w", "dconv_b")])
    if rc != 0:
        raise ValueError("r2l_oracle_scan_bwd rejected its arguments")
    return out
