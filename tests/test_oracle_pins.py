"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test below would fail under a plausible slip in the oracle: a dropped D skip,
a sign error in A, ZOH instead of Euler B, an exclusive instead of inclusive state,
scanning the wrong way, a flipped convolution, a missing per-block reset, a state
hand-off off by one token, a transposed W_out, or the gate applied per direction.

Sources of truth used: hand-derived worked examples (tests/golden), closed forms
(single token, geometric sums, pure decay of a cached state), an O(L^2) brute-force
evaluation of the recurrence's explicit solution, library routines for the parts
that are textbook functions (numpy logaddexp for softplus, scipy expit for the
sigmoid, torch conv1d for the causal convolution, numpy matmul for the residual),
and the invariants the pages state (identity at s = 0, exact cacheability of the
forward boundary state, block-confined reverse scan).
"""

import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import workloads as W
from conftest import rel_err

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def rand_inputs(batch, seqlen, d_inner, conv=0, gate=True, wid=90, layer=0, direction=""):
    t = W.scan_inputs(wid, batch, seqlen, d_inner, 16, conv, io="f32", layer=layer, gate=gate,
                      direction=direction)
    return {k: W.as_f64(v) for k, v in t.items()}


def call_scan(o, p, **kw):
    return o.scan(p["x"], p["dt"], p["B"], p["C"], p.get("z"), p["A"], p["D"], p["dt_bias"],
                  p.get("conv_w"), p.get("conv_b"), **kw)


# ----------------------------------------------------------------------------- brute force

def softplus_lib(v):
    return np.logaddexp(0.0, v)


def silu_lib(v):
    return v * expit(v)


def conv_lib(x, w, b, reverse, block_len):
    """Causal depthwise conv + SiLU in scan order, via torch conv1d per block (reverse) or
    over the whole sequence (forward).  x [L, d]; w [d, W]; b [d]."""
    L, d = x.shape
    Wd = w.shape[1]
    out = np.empty_like(x)
    wt = torch.from_numpy(w).reshape(d, 1, Wd)
    bt = torch.from_numpy(b)
    segs = [(s, s + block_len) for s in range(0, L, block_len)] if reverse else [(0, L)]
    for s0, s1 in segs:
        seg = x[s0:s1]
        if reverse:
            seg = seg[::-1]
        inp = torch.from_numpy(np.ascontiguousarray(seg.T)).reshape(1, d, -1)
        r = torch.nn.functional.conv1d(torch.nn.functional.pad(inp, (Wd - 1, 0)), wt, bt, groups=d)
        r = r.reshape(d, -1).numpy().T
        if reverse:
            r = r[::-1]
        out[s0:s1] = silu_lib(r)
    return out


def brute_scan(p, reverse=True, block_len=None, h0=None):
    """Explicit solution of the linear recurrence, one output at a time.

    reverse: h_t = sum_{s=t}^{e} exp(A * sum_{r=t}^{s-1} delta_r) * delta_s B_s u_s
    forward: h_t = exp(A * sum_{r=0}^{t} delta_r) h0 + sum_{s=0}^{t} exp(A * sum_{r=s+1}^{t} delta_r) delta_s B_s u_s
    """
    x, dt, Bm, Cm, z = p["x"], p["dt"], p["B"], p["C"], p.get("z")
    A, D, bias = p["A"], p["D"], p["dt_bias"]
    bsz, L, d_inner = x.shape
    block_len = block_len or L
    y = np.zeros_like(x)
    hl = np.zeros((bsz, d_inner, A.shape[1]))
    for b in range(bsz):
        delta = softplus_lib(dt[b] + bias[None, :])  # [L, d]
        u = x[b] if p.get("conv_w") is None else conv_lib(x[b], p["conv_w"], p["conv_b"], reverse, block_len)
        for d in range(d_inner):
            segs = [(s, s + block_len) for s in range(0, L, block_len)] if reverse else [(0, L)]
            for s0, s1 in segs:
                for t in range(s0, s1):
                    h = np.zeros(A.shape[1])
                    if reverse:
                        for s in range(t, s1):
                            h += np.exp(A[d] * delta[t:s, d].sum()) * delta[s, d] * Bm[b, s] * u[s, d]
                    else:
                        if h0 is not None:
                            h += np.exp(A[d] * delta[0:t + 1, d].sum()) * h0[b, d]
                        for s in range(0, t + 1):
                            h += np.exp(A[d] * delta[s + 1:t + 1, d].sum()) * delta[s, d] * Bm[b, s] * u[s, d]
                        if t == L - 1:
                            hl[b, d] = h
                    yv = float(Cm[b, t] @ h) + D[d] * u[t, d]
                    if z is not None:
                        yv *= silu_lib(z[b, t, d])
                    y[b, t, d] = yv
    return y, hl


# ----------------------------------------------------------------------------- golden

def _gold_params(c):
    L = len(c["x"])
    one = lambda v: np.array(v, dtype=np.float64)
    p = {
        "x": one(c["x"]).reshape(1, L, 1),
        "dt": one(c["dt"]).reshape(1, L, 1),
        "B": one(c["B"]).reshape(1, L, 1),
        "C": one(c["C"]).reshape(1, L, 1),
        "z": one(c["z"]).reshape(1, L, 1) if "z" in c else None,
        "A": one([[c["A"]]]),
        "D": one([c["D"]]),
        "dt_bias": one([c["dt_bias"]]),
        "conv_w": one([c["conv_w"]]) if "conv_w" in c else None,
        "conv_b": one([c["conv_b"]]) if "conv_w" in c else None,
    }
    return p


@pytest.mark.parametrize("idx", range(7))
def test_hand_worked_cases(oracle_lib, idx):
    c = json.load(open(GOLD))["cases"][idx]
    p = _gold_params(c)
    if c["reverse"]:
        y = call_scan(oracle_lib, p, reverse=True)
    else:
        h0 = np.full((1, 1, 1), float(c.get("h0", 0.0)))
        y, hl = call_scan(oracle_lib, p, reverse=False, h0=h0, want_h_last=True)
        if "h_last" in c:
            assert hl[0, 0, 0] == pytest.approx(c["h_last"], rel=1e-15, abs=1e-15)
    np.testing.assert_allclose(y.reshape(-1), c["y"], rtol=1e-14, atol=1e-15, err_msg=c["name"])


@pytest.mark.parametrize("idx", range(2))
def test_hand_worked_residual(oracle_lib, idx):
    c = json.load(open(GOLD))["residual"][idx]
    out = oracle_lib.residual(np.array(c["hidden"], float), np.array(c["y"], float),
                              np.array(c["W_out"], float), c["s"])
    np.testing.assert_array_equal(out, np.array(c["out"], float))


# ----------------------------------------------------------------------------- closed forms

def test_single_token_closed_form(oracle_lib):
    """L = 1: y = (C.(delta B x) + D x) * SiLU(z), delta = softplus(dt + dt_bias)."""
    p = rand_inputs(3, 1, 5)
    p["D"] = np.linspace(-1.5, 2.0, 5)
    y = call_scan(oracle_lib, p, reverse=True)
    delta = softplus_lib(p["dt"] + p["dt_bias"])  # [b,1,d]
    cb = np.einsum("btn,btn->bt", p["C"], p["B"])[..., None]
    ref = (delta * p["x"] * cb + p["D"] * p["x"]) * silu_lib(p["z"])
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-14)
    # the forward direction is the same single step
    yf = call_scan(oracle_lib, p, reverse=False)
    np.testing.assert_allclose(yf, ref, rtol=1e-13, atol=1e-14)


def test_softplus_large_argument(oracle_lib):
    """dt + dt_bias > 20: delta equals its argument (softplus saturation; the dropped
    log1p(exp(-v)) term is below exp(-20)/20 ~ 1e-10 relative)."""
    p = rand_inputs(1, 1, 4, gate=False)
    p["dt"] = np.full_like(p["dt"], 30.0)
    y = call_scan(oracle_lib, p, reverse=True)
    delta = softplus_lib(p["dt"] + p["dt_bias"])
    cb = np.einsum("btn,btn->bt", p["C"], p["B"])[..., None]
    np.testing.assert_allclose(y, delta * p["x"] * cb + p["D"] * p["x"], rtol=2e-10)


@pytest.mark.parametrize("reverse", [True, False])
def test_geometric_sum(oracle_lib, reverse):
    """Constant delta, B, x per channel: the state k tokens into the scan (inclusive) is
    delta B x (1 - a^k) / (1 - a) with a = exp(delta A)."""
    L, d = 12, 3
    p = rand_inputs(1, L, d, gate=False)
    p["x"][:] = np.array([0.7, -1.3, 2.0])[None, None, :]
    p["dt"][:] = np.array([0.1, -0.4, 0.3])[None, None, :]
    p["B"][:] = p["B"][:, :1, :]  # same B at every token
    Cn = np.zeros(16)
    Cn[5] = 1.0
    p["C"][:] = Cn
    p["D"] = np.zeros(d)
    y = call_scan(oracle_lib, p, reverse=reverse)
    delta = softplus_lib(p["dt"][0, 0] + p["dt_bias"])  # [d]
    a = np.exp(delta * p["A"][:, 5])
    for t in range(L):
        k = (L - t) if reverse else (t + 1)
        ref = delta * p["B"][0, 0, 5] * p["x"][0, 0] * (1 - a ** k) / (1 - a)
        np.testing.assert_allclose(y[0, t], ref, rtol=1e-12)


def test_cached_state_pure_decay(oracle_lib):
    """x = 0: the forward output is only the cached state decaying:
    y_t = sum_n C_tn exp((t+1) delta A_n) h0_n and h_last = exp(L delta A) h0."""
    L, d = 6, 2
    p = rand_inputs(2, L, d, gate=False)
    p["x"][:] = 0.0
    p["dt"][:] = p["dt"][:, :1, :]
    h0 = W.as_f64(W.boundary_state(91, 2, d))
    y, hl = call_scan(oracle_lib, p, reverse=False, h0=h0, want_h_last=True)
    delta = softplus_lib(p["dt"][:, 0, :] + p["dt_bias"])  # [b, d]
    for b in range(2):
        for t in range(L):
            dec = np.exp((t + 1) * delta[b][:, None] * p["A"])  # [d, n]
            ref = (dec * h0[b] * p["C"][b, t][None, :]).sum(-1)
            np.testing.assert_allclose(y[b, t], ref, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(hl[b], np.exp(L * delta[b][:, None] * p["A"]) * h0[b], rtol=1e-12)


# ----------------------------------------------------------------------------- brute force

@pytest.mark.parametrize("conv", [0, 4])
@pytest.mark.parametrize("block_len", [16, 4])
def test_reverse_matches_bruteforce(oracle_lib, conv, block_len):
    p = rand_inputs(2, 16, 3, conv=conv)
    y = call_scan(oracle_lib, p, reverse=True, block_len=block_len)
    ref, _ = brute_scan(p, reverse=True, block_len=block_len)
    assert rel_err(y, ref) < 1e-12


@pytest.mark.parametrize("conv", [0, 4])
def test_forward_from_state_matches_bruteforce(oracle_lib, conv):
    p = rand_inputs(2, 11, 3, conv=conv)
    h0 = W.as_f64(W.boundary_state(92, 2, 3))
    y, hl = call_scan(oracle_lib, p, reverse=False, h0=h0, want_h_last=True)
    ref, ref_hl = brute_scan(p, reverse=False, h0=h0)
    assert rel_err(y, ref) < 1e-12
    assert rel_err(hl, ref_hl) < 1e-12


def test_conv_matches_torch_conv1d(oracle_lib):
    """With B = 0 the state stays zero and y = D u: the convolution front-end alone,
    checked against torch conv1d applied to each reversed block."""
    p = rand_inputs(2, 24, 5, conv=4, gate=False)
    p["B"][:] = 0.0
    p["D"] = np.ones(5)
    for bl in (24, 8, 6):
        y = call_scan(oracle_lib, p, reverse=True, block_len=bl)
        for b in range(2):
            np.testing.assert_allclose(y[b], conv_lib(p["x"][b], p["conv_w"], p["conv_b"], True, bl),
                                       rtol=1e-13, atol=1e-14)
    yf = call_scan(oracle_lib, p, reverse=False)
    for b in range(2):
        np.testing.assert_allclose(yf[b], conv_lib(p["x"][b], p["conv_w"], p["conv_b"], False, 24),
                                   rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------- invariants

@pytest.mark.parametrize("conv", [0, 4])
def test_reverse_is_flip_forward_flip(oracle_lib, conv):
    """Reversing, scanning left-to-right and reversing back is the right-to-left scan
    (exact: both loops perform the same operations on the same values)."""
    p = rand_inputs(2, 20, 4, conv=conv)
    y = call_scan(oracle_lib, p, reverse=True)
    fl = {k: (v[:, ::-1].copy() if k in ("x", "dt", "B", "C", "z") and v is not None else v) for k, v in p.items()}
    yf = call_scan(oracle_lib, fl, reverse=False)
    np.testing.assert_array_equal(y, yf[:, ::-1])
    # and direction matters on asymmetric input
    y_wrong = call_scan(oracle_lib, p, reverse=False)
    assert rel_err(y_wrong, y) > 1e-2


@pytest.mark.parametrize("conv", [0, 4])
def test_block_confinement(oracle_lib, conv):
    """Reverse outputs of block k do not depend on tokens outside block k, and a multi-block
    scan equals independent scans of each block."""
    L, bl = 32, 8
    p = rand_inputs(1, L, 3, conv=conv)
    y = call_scan(oracle_lib, p, reverse=True, block_len=bl)
    q = {k: (v.copy() if v is not None else None) for k, v in p.items()}
    rng = np.random.default_rng(5)
    for key in ("x", "dt", "B", "C", "z"):
        q[key][:, :8] = rng.standard_normal(q[key][:, :8].shape)
        q[key][:, 16:] = rng.standard_normal(q[key][:, 16:].shape)
    yq = call_scan(oracle_lib, q, reverse=True, block_len=bl)
    np.testing.assert_array_equal(y[:, 8:16], yq[:, 8:16])
    for s0 in range(0, L, bl):
        part = {k: (v[:, s0:s0 + bl] if k in ("x", "dt", "B", "C", "z") and v is not None else v) for k, v in p.items()}
        np.testing.assert_array_equal(call_scan(oracle_lib, part, reverse=True), y[:, s0:s0 + bl])


def test_prefix_cache_continuation(oracle_lib):
    """Scanning a clean prefix, caching its forward boundary state and continuing from it
    equals scanning the whole sequence (exactly)."""
    L, cut = 24, 16
    p = rand_inputs(2, L, 3)
    h0 = W.as_f64(W.boundary_state(93, 2, 3))
    y, hl = call_scan(oracle_lib, p, reverse=False, h0=h0, want_h_last=True)
    pre = {k: (v[:, :cut] if k in ("x", "dt", "B", "C", "z") and v is not None else v) for k, v in p.items()}
    suf = {k: (v[:, cut:] if k in ("x", "dt", "B", "C", "z") and v is not None else v) for k, v in p.items()}
    y1, h_mid = call_scan(oracle_lib, pre, reverse=False, h0=h0, want_h_last=True)
    y2, h_end = call_scan(oracle_lib, suf, reverse=False, h0=h_mid, want_h_last=True)
    np.testing.assert_array_equal(np.concatenate([y1, y2], 1), y)
    np.testing.assert_array_equal(h_end, hl)


def _cut(p, a, b):
    return {k: (v[:, a:b] if k in ("x", "dt", "B", "C", "z") and v is not None else v) for k, v in p.items()}


def test_conv_state_layout_and_continuation(oracle_lib):
    """With the width-4 convolution, the state handed across a cut is the three inputs before
    it, newest first (written out here by hand from x), and resuming from it reproduces the
    uncut scan, whose convolution is pinned to torch conv1d above."""
    L, cut = 24, 13
    p = rand_inputs(2, L, 5, conv=4, wid=95)
    h0 = W.as_f64(W.boundary_state(95, 2, 5))
    y, hl = call_scan(oracle_lib, p, reverse=False, h0=h0, want_h_last=True)
    y1, h_mid, cs = call_scan(oracle_lib, _cut(p, 0, cut), reverse=False, h0=h0, want_h_last=True,
                              want_conv_state=True)
    by_hand = np.stack([p["x"][:, cut - 1 - j, :] for j in range(3)], axis=-1)  # [b, d, 3]
    np.testing.assert_array_equal(cs, by_hand)
    y2, h_end, cs_end = call_scan(oracle_lib, _cut(p, cut, L), reverse=False, h0=h_mid, want_h_last=True,
                                  conv_state=by_hand, want_conv_state=True)
    np.testing.assert_array_equal(np.concatenate([y1, y2], 1), y)
    np.testing.assert_array_equal(h_end, hl)
    np.testing.assert_array_equal(cs_end, np.stack([p["x"][:, L - 1 - j, :] for j in range(3)], axis=-1))
    # without the convolution state the continuation differs (the padding would be zeros)
    y2z = call_scan(oracle_lib, _cut(p, cut, L), reverse=False, h0=h_mid)
    assert not np.allclose(y2z[:, :3], y[:, cut:cut + 3])


@pytest.mark.parametrize("chunk", [1, 2, 5])
def test_conv_state_chunked_decode(oracle_lib, chunk):
    """Decoding in chunks shorter than the convolution window (the state then mixes new inputs
    with cached ones) equals one scan over the whole sequence."""
    L = 11
    p = rand_inputs(1, L, 4, conv=4, wid=96)
    y = call_scan(oracle_lib, p, reverse=False)
    h, cs, parts = None, None, []
    for a in range(0, L, chunk):
        yc, h, cs = call_scan(oracle_lib, _cut(p, a, min(a + chunk, L)), reverse=False, h0=h, want_h_last=True,
                              conv_state=cs, want_conv_state=True)
        parts.append(yc)
    np.testing.assert_array_equal(np.concatenate(parts, 1), y)


def test_conv_state_zero_is_default_and_rejected_where_meaningless(oracle_lib):
    p = rand_inputs(1, 6, 4, conv=4, wid=97)
    y = call_scan(oracle_lib, p, reverse=False)
    np.testing.assert_array_equal(call_scan(oracle_lib, p, reverse=False, conv_state=np.zeros((1, 4, 3))), y)
    with pytest.raises(ValueError):
        call_scan(oracle_lib, p, reverse=True, conv_state=np.zeros((1, 4, 3)))
    with pytest.raises(ValueError):
        call_scan(oracle_lib, dict(p, conv_w=None, conv_b=None), reverse=False, want_conv_state=True)


def test_linearity_in_x(oracle_lib):
    """Without conv and gate, y is linear in x for fixed delta, B, C."""
    p = rand_inputs(1, 10, 3, gate=False)
    q = rand_inputs(1, 10, 3, gate=False, layer=1)
    y1 = call_scan(oracle_lib, p, reverse=True)
    p2 = dict(p, x=q["x"])
    y2 = call_scan(oracle_lib, p2, reverse=True)
    p3 = dict(p, x=2.5 * p["x"] - 0.75 * q["x"])
    y3 = call_scan(oracle_lib, p3, reverse=True)
    assert rel_err(y3, 2.5 * y1 - 0.75 * y2) < 1e-12


def test_mamba_h_combination(oracle_lib):
    """Forward-from-state plus block-confined reverse: (y_f + y_r) * SiLU(z), with the gate
    applied once to the sum, and h_last from the forward direction only."""
    L, bl = 8, 4
    pf = rand_inputs(2, L, 3, wid=94)
    pr = rand_inputs(2, L, 3, wid=94, direction="_r")
    assert np.array_equal(pf["x"], pr["x"]) and np.array_equal(pf["z"], pr["z"])
    h0 = W.as_f64(W.boundary_state(94, 2, 3))
    y, hl = oracle_lib.mamba_h(pf["x"], pf["z"], pf, pr, h0=h0, block_len=bl)
    nz_f = dict(pf, z=None)
    nz_r = dict(pr, z=None)
    yf, hf = brute_scan(nz_f, reverse=False, h0=h0)
    yr, _ = brute_scan(nz_r, reverse=True, block_len=bl)
    assert rel_err(y, (yf + yr) * silu_lib(pf["z"])) < 1e-12
    assert rel_err(hl, hf) < 1e-12
    # the gate must not be applied per direction
    assert rel_err(y, yf * silu_lib(pf["z"]) + yr * silu_lib(pf["z"]) ** 2) > 1e-3


# ----------------------------------------------------------------------------- residual

def test_residual_matches_matmul(oracle_lib):
    rng = np.random.default_rng(3)
    M, dm, di = 5, 7, 3
    hidden = rng.standard_normal((M, dm))
    y = rng.standard_normal((M, di))
    Wm = rng.standard_normal((dm, di))
    out = oracle_lib.residual(hidden, y, Wm, 0.05)
    np.testing.assert_allclose(out, hidden + 0.05 * (y @ Wm.T), rtol=1e-14, atol=1e-14)


def test_residual_s0_identity(oracle_lib):
    rng = np.random.default_rng(4)
    hidden = rng.standard_normal((4, 6))
    out = oracle_lib.residual(hidden, rng.standard_normal((4, 3)), rng.standard_normal((6, 3)), 0.0)
    np.testing.assert_array_equal(out, hidden)


def test_rejects_bad_arguments(oracle_lib):
    p = rand_inputs(1, 6, 2)
    with pytest.raises(ValueError):
        call_scan(oracle_lib, p, reverse=True, block_len=4)  # does not divide 6
    with pytest.raises(ValueError):
        call_scan(oracle_lib, p, reverse=True, h0=np.zeros((1, 2, 16)))  # reverse emits/takes no state


# ----------------------------------------------------------------------------- sidecar front-end

def test_linear_matches_numpy(oracle_lib):
    rng = np.random.default_rng(7)
    X, Wm = rng.standard_normal((13, 24)), rng.standard_normal((9, 24))
    assert rel_err(oracle_lib.linear(X, Wm), X @ Wm.T) < 1e-13


@pytest.mark.parametrize("reverse", [True, False])
def test_conv_silu_matches_torch_conv1d(oracle_lib, reverse):
    p = rand_inputs(2, 24, 5, conv=4, wid=98)
    bl = 8 if reverse else 24
    u = oracle_lib.conv_silu(p["x"], p["conv_w"], p["conv_b"], reverse=reverse, block_len=bl)
    for b in range(2):
        assert rel_err(u[b], conv_lib(p["x"][b], p["conv_w"], p["conv_b"], reverse, bl)) < 1e-12
    # the scan's built-in convolution is the same map: scanning u without one gives identical bits
    y_conv = call_scan(oracle_lib, p, reverse=reverse, block_len=bl)
    y_u = call_scan(oracle_lib, dict(p, x=u, conv_w=None, conv_b=None), reverse=reverse, block_len=bl)
    np.testing.assert_array_equal(y_conv, y_u)


def _sidecar_case(conv=4, wid=99):
    batch, seqlen, bl, d_model, d_inner, dt_rank = 2, 16, 8, 64, 64, 16
    w = {k: (W.as_f64(v) if v is not None else None)
         for k, v in W.sidecar_weights(wid, d_model, d_inner, dt_rank=dt_rank, conv_width=conv).items()}
    hidden = W.as_f64(W.normal(wid, 0, "hidden", (batch * seqlen, d_model)))
    return w, hidden, batch, seqlen, bl


@pytest.mark.parametrize("conv", [4, 0])
def test_sidecar_matches_independent_recomputation(oracle_lib, conv):
    """numpy matmuls for the projections, torch conv1d for the convolution and the explicit
    O(L^2) solution of the recurrence for the scan."""
    w, hidden, batch, seqlen, bl = _sidecar_case(conv)
    out, it = oracle_lib.sidecar(hidden, w, batch, seqlen, bl, 0.05)
    d_inner, dt_rank, N = w["W_in"].shape[0] // 2, w["W_dt"].shape[1], w["A"].shape[1]
    xz = hidden @ w["W_in"].T
    x, z = xz[:, :d_inner].reshape(batch, seqlen, d_inner), xz[:, d_inner:].reshape(batch, seqlen, d_inner)
    u = np.stack([conv_lib(x[b], w["conv_w"], w["conv_b"], True, bl) for b in range(batch)]) if conv else x
    dbl = u.reshape(batch * seqlen, d_inner) @ w["W_x"].T
    dt = dbl[:, :dt_rank] @ w["W_dt"].T
    p = {"x": u, "dt": dt.reshape(batch, seqlen, d_inner), "B": dbl[:, dt_rank:dt_rank + N].reshape(batch, seqlen, N),
         "C": dbl[:, dt_rank + N:].reshape(batch, seqlen, N), "z": z, "A": w["A"], "D": w["D"],
         "dt_bias": w["dt_bias"]}
    y, _ = brute_scan(p, reverse=True, block_len=bl)
    ref = hidden + 0.05 * (y.reshape(batch * seqlen, d_inner) @ w["W_out"].T)
    assert rel_err(it["u"], u.reshape(batch * seqlen, d_inner)) < 1e-12
    assert rel_err(it["y"], y.reshape(batch * seqlen, d_inner)) < 1e-10
    assert rel_err(out, ref) < 1e-12


def test_round_bf16_hand_values(oracle_lib):
    """bf16 keeps 7 mantissa bits: the spacing above 1 is 2^-7.  Halfway cases go to the even
    neighbour, anything past halfway goes up, and the sign is kept."""
    e = 2.0 ** -8
    cases = [(1.0, 1.0), (1.0 + e, 1.0), (1.0 + 3 * e, 1.0 + 4 * e), (1.0 + e + 2.0 ** -20, 1.0 + 2 * e),
             (-(1.0 + e), -1.0), (1.0 + e - 2.0 ** -20, 1.0), (3.0, 3.0), (0.0, 0.0), (1.0 / 3.0, 0.333984375),
             (1000.0, 1000.0), (1001.0, 1000.0), (1003.0, 1004.0)]
    got = oracle_lib.round_bf16(np.array([c[0] for c in cases]))
    np.testing.assert_array_equal(got, np.array([c[1] for c in cases]))


def test_round_bf16_matches_torch(oracle_lib):
    """Against torch's float32 -> bfloat16 conversion (round to nearest even) on random values
    spread over many binades, including exact ties."""
    rng = np.random.default_rng(11)
    v = rng.standard_normal(20000) * np.exp2(rng.integers(-40, 40, 20000))
    ties = (rng.integers(1, 1 << 8, 512).astype(np.float64) * 2 + 1) * 2.0 ** -9  # m.5 ulp of [1, 2)
    v = np.concatenate([v, 1.0 + ties / 2.0 ** 8, -(1.0 + ties / 2.0 ** 8)]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle_lib.round_bf16(v.astype(np.float64)), ref)


@pytest.mark.parametrize("conv", [4, 0])
def test_sidecar_bf16_store_matches_independent_recomputation(oracle_lib, conv):
    """With bf16 storage of the activations: numpy matmuls, torch conv1d, the explicit O(L^2)
    solution of the recurrence, and torch's bfloat16 conversion at each stored activation."""
    w, hidden, batch, seqlen, bl = _sidecar_case(conv, wid=97)
    out, it = oracle_lib.sidecar(hidden, w, batch, seqlen, bl, 0.5, store_bf16=True)
    d_inner, dt_rank, N = w["W_in"].shape[0] // 2, w["W_dt"].shape[1], w["A"].shape[1]
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).double().numpy()
    xz = hidden @ w["W_in"].T
    x, z = xz[:, :d_inner].reshape(batch, seqlen, d_inner), bf(xz[:, d_inner:]).reshape(batch, seqlen, d_inner)
    u = np.stack([conv_lib(x[b], w["conv_w"], w["conv_b"], True, bl) for b in range(batch)]) if conv else x
    u = bf(u)
    dbl = bf(u.reshape(batch * seqlen, d_inner) @ w["W_x"].T)
    dt = bf(dbl[:, :dt_rank] @ w["W_dt"].T)
    p = {"x": u, "dt": dt.reshape(batch, seqlen, d_inner), "B": dbl[:, dt_rank:dt_rank + N].reshape(batch, seqlen, N),
         "C": dbl[:, dt_rank + N:].reshape(batch, seqlen, N), "z": z, "A": w["A"], "D": w["D"],
         "dt_bias": w["dt_bias"]}
    y, _ = brute_scan(p, reverse=True, block_len=bl)
    y = bf(y.reshape(batch * seqlen, d_inner))
    ref = hidden + 0.5 * (y @ w["W_out"].T)
    for k, v in (("z", z), ("u", u), ("dt", dt), ("y", y)):
        np.testing.assert_array_equal(it[k], v.reshape(batch * seqlen, d_inner), err_msg=k)
    np.testing.assert_array_equal(np.concatenate([it["dt_low"], it["B"], it["C"]], 1), dbl)
    assert rel_err(out, ref) < 1e-12
    # the stored activations moved the output: the unrounded chain differs
    out64, _ = oracle_lib.sidecar(hidden, w, batch, seqlen, bl, 0.5)
    assert not np.array_equal(out, out64) and rel_err(out, out64) < 0.05


def test_sidecar_identities(oracle_lib):
    """s = 0 and a z half of zeros (SiLU(0) = 0 closes the gate) both leave hidden bit-identical,
    while a live sidecar changes it."""
    w, hidden, batch, seqlen, bl = _sidecar_case()
    np.testing.assert_array_equal(oracle_lib.sidecar(hidden, w, batch, seqlen, bl, 0.0)[0], hidden)
    d_inner = w["W_in"].shape[0] // 2
    closed = dict(w, W_in=np.concatenate([w["W_in"][:d_inner], np.zeros_like(w["W_in"][d_inner:])]))
    np.testing.assert_array_equal(oracle_lib.sidecar(hidden, closed, batch, seqlen, bl, 0.05)[0], hidden)
    assert not np.array_equal(oracle_lib.sidecar(hidden, w, batch, seqlen, bl, 0.05)[0], hidden)


def test_sidecar_is_block_confined(oracle_lib):
    """Tokens of one block do not affect another block's output (the convolution and the scan
    both stop at the block edge); token rows are independent through the projections."""
    w, hidden, batch, seqlen, bl = _sidecar_case()
    out, _ = oracle_lib.sidecar(hidden, w, batch, seqlen, bl, 0.05)
    h2 = hidden.copy()
    h2[bl:2 * bl] += 1.0  # second block of the first sequence
    out2, _ = oracle_lib.sidecar(h2, w, batch, seqlen, bl, 0.05)
    np.testing.assert_array_equal(out2[:bl], out[:bl])
    np.testing.assert_array_equal(out2[2 * bl:], out[2 * bl:])
    assert not np.array_equal(out2[bl:2 * bl], out[bl:2 * bl])


# ----------------------------------------------------------------------------- scan backward

def _fd_grad(oracle_lib, p, key, w, bl, eps=1e-6):
    """Central differences of L = sum(w * y) with respect to every element of p[key]."""
    base = p[key]
    g = np.zeros_like(base)
    flat = base.reshape(-1)
    for i in range(flat.size):
        old = flat[i]
        flat[i] = old + eps
        lp = float(np.sum(w * call_scan(oracle_lib, p, reverse=True, block_len=bl)))
        flat[i] = old - eps
        lm = float(np.sum(w * call_scan(oracle_lib, p, reverse=True, block_len=bl)))
        flat[i] = old
        g.reshape(-1)[i] = (lp - lm) / (2 * eps)
    return g


@pytest.mark.parametrize("gate,conv", [(True, 0), (False, 0), (True, 4), (False, 4)])
def test_scan_bwd_matches_finite_differences(oracle_lib, gate, conv):
    """Every gradient of the backward oracle against central differences of the (pinned) forward
    oracle, on two batch rows of two 4-token blocks (5-token blocks with the width-4 convolution,
    so that its taps reach past a block edge), 3 channels and 4 states."""
    bl = 5 if conv else 4
    t = W.scan_inputs(91, 2, 2 * bl, 3, 4, conv, io="f32", gate=gate)
    p = {k: (W.as_f64(v) if v is not None else None) for k, v in t.items()}
    w = np.random.default_rng(5).standard_normal(p["x"].shape)
    g = oracle_lib.scan_bwd(p["x"], p["dt"], p["B"], p["C"], p["z"], p["A"], p["D"], p["dt_bias"], w, block_len=bl,
                            conv_w=p["conv_w"], conv_b=p["conv_b"])
    names = {"x": "dx", "dt": "ddt", "B": "dB", "C": "dC", "A": "dA", "D": "dD", "dt_bias": "ddt_bias"}
    if gate:
        names["z"] = "dz"
    else:
        assert g["dz"] is None
    if conv:
        names["conv_w"] = "dconv_w"
        names["conv_b"] = "dconv_b"
    else:
        assert g["dconv_w"] is None and g["dconv_b"] is None
    for k, gk in names.items():
        fd = _fd_grad(oracle_lib, p, k, w, bl)
        # central differences with eps = 1e-6 carry ~1e-10 of rounding (fp64 L / eps): the bound is
        # 1e-6 of the gradient's scale, with that scale floored at 1e-3 (dA is ~1e-4 here)
        assert np.max(np.abs(g[gk] - fd)) <= 1e-6 * max(float(np.abs(fd).max()), 1e-3), k


def test_scan_bwd_block_confinement_and_linearity(oracle_lib):
    """dy confined to one block gives zero gradients for the other blocks' inputs, and the
    gradients are linear in dy."""
    t = W.scan_inputs(92, 1, 12, 2, 4, 0, io="f32")
    p = {k: (W.as_f64(v) if v is not None else None) for k, v in t.items()}
    args = (p["x"], p["dt"], p["B"], p["C"], p["z"], p["A"], p["D"], p["dt_bias"])
    w1 = np.zeros_like(p["x"])
    w1[:, 4:8] = np.random.default_rng(6).standard_normal(w1[:, 4:8].shape)
    g1 = oracle_lib.scan_bwd(*args, w1, block_len=4)
    for k in ("dx", "ddt", "dz", "dB", "dC"):
        assert np.all(g1[k][:, :4] == 0) and np.all(g1[k][:, 8:] == 0), k
    w2 = np.random.default_rng(7).standard_normal(p["x"].shape)
    g2 = oracle_lib.scan_bwd(*args, w2, block_len=4)
    g3 = oracle_lib.scan_bwd(*args, 2.0 * w1 - 0.5 * w2, block_len=4)
    for k in g1:
        if g1[k] is None:  # no convolution: dconv_w, dconv_b
            continue
        assert rel_err(g3[k], 2.0 * g1[k] - 0.5 * g2[k]) < 1e-12, k
