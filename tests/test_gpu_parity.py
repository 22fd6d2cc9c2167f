"""GPU parity: libr2l (through its C ABI) against the fp64 oracle on the same seeded bytes.

Tolerances (max over elements of |gpu - oracle| / max(|oracle|, rms(oracle))):
  fp32 inputs, fp32 outputs      : 1e-5
  bf16 inputs, fp32 outputs      : 2e-3   (fp32 state; inputs are exact in both)
  bf16 outputs (scan or residual): 2e-3 + 2^-8  (rounding an output to bf16 alone costs up to 2^-8)
Bit-exact checks (GPU against GPU, same kernel order of operations): reverse == flip(forward(flip)),
prefix + cached-state continuation == one shot, block confinement, s = 0 identity.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from conftest import rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-3
TOL_BF16_OUT = 2e-3 + 2.0 ** -8


@pytest.fixture(scope="module")
def r2l():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import reverse_mamba_selective_b200 as pkg

    pkg.load()
    oracle.build()
    return pkg


def dev(p):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in p.items()}


def f64(p):
    return {k: W.as_f64(v) if isinstance(v, torch.Tensor) else v for k, v in p.items()}


def gpu_rev(r2l, g, block_len, y_dtype=torch.float32):
    y = r2l.r2l_scan_block(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"],
                           g["conv_w"], g["conv_b"], block_len=block_len, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return y


def oracle_rev(o, block_len, rows=None, chans=None):
    """Oracle on a subset of batch rows / channels (rows and channels are independent)."""
    o = dict(o)
    if rows is not None:
        for k in ("x", "dt", "B", "C", "z"):
            if o[k] is not None:
                o[k] = o[k][rows]
    if chans is not None:
        for k in ("x", "dt", "z"):
            if o[k] is not None:
                o[k] = o[k][..., chans]
        for k in ("A", "D", "dt_bias", "conv_w", "conv_b"):
            if o[k] is not None:
                o[k] = o[k][chans]
    return oracle.scan(o["x"], o["dt"], o["B"], o["C"], o["z"], o["A"], o["D"], o["dt_bias"], o["conv_w"],
                       o["conv_b"], reverse=True, block_len=block_len)


def check_status(r2l):
    assert r2l.r2l_device_status() == r2l.R2L_OK


# ----------------------------------------------------------------------------- config 0 (tiny, fp32)

def test_tiny_f32_scan_and_residual(r2l):
    wl = W.WORKLOADS["tiny_f32"]
    p = W.scan_inputs(wl.wid, wl.batch, wl.seqlen, wl.d_inner, io="f32")
    y = gpu_rev(r2l, dev(p), wl.block_len)
    ref = oracle_rev(f64(p), wl.block_len)
    assert rel_err(y.cpu().numpy(), ref) < TOL_F32
    res = W.residual_inputs(wl.wid, wl.tokens, wl.d_model, wl.d_inner, io="f32")
    for s in (0.0, 0.05):
        hidden = res["hidden"].cuda()
        before = hidden.clone()
        r2l.r2l_residual_apply(hidden, y.reshape(wl.tokens, wl.d_inner), res["W_out"].cuda(), s)
        torch.cuda.synchronize()
        if s == 0.0:
            assert torch.equal(hidden.view(torch.int32), before.view(torch.int32))
        # the oracle's own chain: its scan output feeds its residual
        ref_h = oracle.residual(W.as_f64(res["hidden"]), ref.reshape(wl.tokens, wl.d_inner), W.as_f64(res["W_out"]), s)
        assert rel_err(hidden.cpu().numpy(), ref_h) < TOL_F32
    check_status(r2l)


# ----------------------------------------------------------------------------- reverse scan, bf16

@pytest.mark.parametrize("batch,seqlen,block_len,d_inner,conv,gate", [
    (3, 32, 32, 2048, 4, True),    # decode-step shape, few rows
    (2, 96, 32, 256, 4, True),     # several blocks per row
    (2, 40, 20, 72, 4, True),      # ragged: block not a multiple of the stage, partial channel tile
    (2, 64, 16, 136, 0, False),    # no conv, no gate, 136 = 4*32 + 8 channels
    (1, 1, 1, 8, 4, True),         # single token, minimum width
    (4, 200, 200, 64, 0, True),    # long block through several stages
    (2, 520, 520, 96, 4, True),    # long block, ragged last stage
])
def test_reverse_scan_bf16_parity(r2l, batch, seqlen, block_len, d_inner, conv, gate):
    p = W.scan_inputs(1, batch, seqlen, d_inner, conv_width=conv, io="bf16", gate=gate, layer=7)
    g = dev(p)
    y = gpu_rev(r2l, g, block_len)
    ref = oracle_rev(f64(p), block_len)
    assert rel_err(y.cpu().numpy(), ref) < TOL_BF16
    yb = gpu_rev(r2l, g, block_len, torch.bfloat16)
    assert rel_err(yb.float().cpu().numpy(), ref) < TOL_BF16_OUT
    check_status(r2l)


def test_reverse_scan_f32_inputs_multiblock(r2l):
    p = W.scan_inputs(0, 2, 48, 64, conv_width=4, io="f32", layer=3)
    y = gpu_rev(r2l, dev(p), 16)
    assert rel_err(y.cpu().numpy(), oracle_rev(f64(p), 16)) < TOL_F32


def test_decode_step_full_size(r2l):
    """R2LM parallel-decode sidecar step at full size: scan (all 64 rows vs oracle) + residual
    (sampled rows vs oracle, identical launch to the benchmark)."""
    wl = W.WORKLOADS["decode_b64_blk32"]
    p = W.scan_inputs(wl.wid, wl.batch, wl.seqlen, wl.d_inner, conv_width=wl.conv_width, io="bf16")
    g = dev(p)
    ref = oracle_rev(f64(p), wl.block_len)
    y32 = gpu_rev(r2l, g, wl.block_len, torch.float32)
    assert rel_err(y32.cpu().numpy(), ref) < TOL_BF16
    y = gpu_rev(r2l, g, wl.block_len, torch.bfloat16)
    assert rel_err(y.float().cpu().numpy(), ref) < TOL_BF16_OUT
    res = W.residual_inputs(wl.wid, wl.tokens, wl.d_model, wl.d_inner, io="bf16")
    hidden = res["hidden"].cuda()
    r2l.r2l_residual_apply(hidden, y.reshape(wl.tokens, wl.d_inner), res["W_out"].cuda(), wl.s)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(wl.tokens, 96, replace=False)
    # the oracle's own chain: its scan output feeds its residual
    yr = ref.reshape(wl.tokens, wl.d_inner)
    ref_h = oracle.residual(W.as_f64(res["hidden"])[rows], yr[rows], W.as_f64(res["W_out"]), wl.s)
    assert rel_err(hidden.float().cpu().numpy()[rows], ref_h) < TOL_BF16_OUT
    # the residual launch alone, same shape and launch configuration, on a seeded bf16 y: nearly
    # every element equals the oracle's value rounded once to bf16
    y_in = W.normal(wl.wid, 0, "u_probe", (wl.tokens, wl.d_inner), std=0.25)
    hidden = res["hidden"].cuda()
    r2l.r2l_residual_apply(hidden, y_in.cuda(), res["W_out"].cuda(), wl.s)
    torch.cuda.synchronize()
    ref_h = oracle.residual(W.as_f64(res["hidden"])[rows], W.as_f64(y_in)[rows], W.as_f64(res["W_out"]), wl.s)
    got = hidden.float().cpu().numpy()[rows]
    assert rel_err(got, ref_h) < TOL_BF16_OUT
    ref_b = torch.from_numpy(ref_h).float().to(torch.bfloat16).float().numpy()
    assert np.mean(got == ref_b) > 0.98
    check_status(r2l)


@pytest.mark.parametrize("case", ["full", "small", "one_block", "s0"])
def test_decode_step_entry_point(r2l, case):
    """r2l_decode_step (scan + residual in one call, the residual's operands pulled into L2 during
    the scan) gives r2l_scan_block followed by r2l_residual_apply bit for bit, and the oracle's
    chain on sampled rows.  Cases: the decode step at full size (the benchmark's launch); 3 rows of
    5 blocks of 8 tokens (120 token rows, d_model 264); one 16-token block (the residual for up to
    64 rows); s = 0 (hidden untouched)."""
    if case == "full":
        wl = W.WORKLOADS["decode_b64_blk32"]
        b, L, blk, d, dm, s = wl.batch, wl.seqlen, wl.block_len, wl.d_inner, wl.d_model, wl.s
        wid = wl.wid
    elif case == "one_block":
        b, L, blk, d, dm, s, wid = 1, 16, 16, 256, 256, 0.05, 12
    else:
        b, L, blk, d, dm, s, wid = 3, 40, 8, 192, 264, (0.05 if case == "small" else 0.0), 11
    p = W.scan_inputs(wid, b, L, d, conv_width=4, io="bf16")
    g = dev(p)
    res = W.residual_inputs(wid, b * L, dm, d, io="bf16")
    Wm = res["W_out"].cuda()
    h1, h2 = res["hidden"].cuda(), res["hidden"].cuda()
    y1 = r2l.r2l_decode_step(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], g["conv_w"],
                             g["conv_b"], h1, Wm, s, block_len=blk)
    y2 = gpu_rev(r2l, g, blk, torch.bfloat16)
    r2l.r2l_residual_apply(h2, y2.reshape(b * L, d), Wm, s)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))
    if s == 0.0:
        assert torch.equal(h1.cpu().view(torch.int16), res["hidden"].view(torch.int16))
    rows = np.arange(b * L) if b * L <= 128 else np.random.default_rng(2).choice(b * L, 64, replace=False)
    brows = np.unique(rows // L)
    ref_y = oracle_rev(f64(p), blk, rows=brows).reshape(-1, d)
    # token row r sits at (position of batch row r // L among brows) * L + r % L in ref_y
    at = {int(bb): i for i, bb in enumerate(brows)}
    yr = ref_y[[at[int(r // L)] * L + int(r % L) for r in rows]]
    assert rel_err(y1.reshape(b * L, d).float().cpu().numpy()[rows], yr) < TOL_BF16_OUT
    ref_h = oracle.residual(W.as_f64(res["hidden"])[rows], yr, W.as_f64(res["W_out"]), s)
    assert rel_err(h1.float().cpu().numpy()[rows], ref_h) < TOL_BF16_OUT
    check_status(r2l)


# ----------------------------------------------------------------------------- residual GEMM shapes

@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (2048, 2048, 2048), (100, 264, 72), (300, 512, 1000),
                                   (16, 2048, 2048), (1, 8, 8), (257, 776, 136),
                                   (1024, 2048, 512), (896, 1920, 2048), (512, 2048, 2048),
                                   (256, 2048, 2048), (48, 1032, 384),  # 32- and 16-column tiles
                                   # 256-column tiles: ragged M, N and K; a last row tile with 8
                                   # valid rows (M 1800); more tiles than SMs (N 4096)
                                   (2000, 2056, 1000), (1800, 2048, 2048), (4096, 1024, 512),
                                   (2048, 4096, 256),
                                   # up to 64 token rows: swapped operands, K split over a cluster
                                   # (ragged N; odd chunk counts of K; 1 to 8 K ranges; a single row);
                                   # 65 to 128 rows on the general kernel
                                   (128, 2048, 2048), (1, 2048, 2048), (33, 520, 1088), (64, 4096, 4096),
                                   (16, 8192, 512), (100, 2048, 64), (17, 264, 192), (80, 1024, 2048)])
def test_residual_bf16_parity(r2l, M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    hidden = torch.randn(M, N, generator=g).to(torch.bfloat16)
    y = torch.randn(M, K, generator=g).to(torch.bfloat16)
    Wm = (torch.randn(N, K, generator=g) / math.sqrt(K)).to(torch.bfloat16)
    h = hidden.cuda()
    r2l.r2l_residual_apply(h, y.cuda(), Wm.cuda(), 0.05)
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 300 else np.union1d(np.random.default_rng(1).choice(M, 128, replace=False),
                                                    np.arange(M - 8, M))
    ref = oracle.residual(W.as_f64(hidden)[rows], W.as_f64(y)[rows], W.as_f64(Wm), 0.05)
    assert rel_err(h.float().cpu().numpy()[rows], ref) < TOL_BF16_OUT
    check_status(r2l)


def test_residual_s0_bit_identity(r2l):
    """s = 0 leaves hidden bit-identical, including negative zeros (identity at initialisation)."""
    hidden = torch.randn(256, 512).to(torch.bfloat16)
    hidden[0, :7] = -0.0
    h = hidden.cuda()
    r2l.r2l_residual_apply(h, torch.randn(256, 128).to(torch.bfloat16).cuda(),
                           torch.randn(512, 128).to(torch.bfloat16).cuda(), 0.0)
    torch.cuda.synchronize()
    assert torch.equal(h.cpu().view(torch.int16), hidden.view(torch.int16))


# ----------------------------------------------------------------------------- prefill (long L)

def test_prefill_long_scan_sampled(r2l):
    """The prefill workload at full size (8 rows, one 4096-token reverse block, d_inner 2048) in the
    benchmark's launch configuration: fp32 outputs of every row on 256 channels (four 64-channel
    groups spread over the channel range, so several warps and CTAs) against the oracle over all
    4096 tokens at the bf16-input bound; bf16 outputs of the same launch at the bf16-output bound."""
    wl = W.WORKLOADS["prefill_b8_L4096"]
    p = W.scan_inputs(wl.wid, wl.batch, wl.seqlen, wl.d_inner, io="bf16")
    g = dev(p)
    chans = np.concatenate([np.arange(c, c + 64) for c in (0, 576, 1216, wl.d_inner - 64)])
    ref = oracle_rev(f64(p), wl.block_len, chans=chans)
    y32 = gpu_rev(r2l, g, wl.block_len, torch.float32)
    got = y32.cpu().numpy()[..., chans]
    assert rel_err(got, ref) < TOL_BF16
    # both ends of the block: the first tokens of the scan (right edge) and the last (left edge)
    assert rel_err(got[:, -64:], ref[:, -64:]) < TOL_BF16 and rel_err(got[:, :64], ref[:, :64]) < TOL_BF16
    del y32
    y = gpu_rev(r2l, g, wl.block_len, torch.bfloat16)
    assert rel_err(y.float().cpu().numpy()[..., chans], ref) < TOL_BF16_OUT
    assert torch.isfinite(y.float()).all()
    check_status(r2l)


# ----------------------------------------------------------------------------- partial bidirectionality

def mamba_h_inputs(wid, batch, seqlen, d_inner, conv=0, io="bf16", h0_std=0.1):
    pf = W.scan_inputs(wid, batch, seqlen, d_inner, conv_width=conv, io=io)
    pr = W.scan_inputs(wid, batch, seqlen, d_inner, conv_width=conv, io=io, direction="_r")
    h0 = W.boundary_state(wid, batch, d_inner, std=h0_std)
    return pf, pr, h0


def gpu_mamba_h(r2l, pf, pr, h0, block_len, y_dtype=torch.float32, rev=True):
    gf, gr = dev(pf), dev(pr)
    gr["x"], gr["z"] = gf["x"], gf["z"]
    y, hl = r2l.fwd_scan_from_state(gf["x"], gf["z"], gf, gr if rev else None, h0=h0.cuda(),
                                    rev_block_len=block_len, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return y, hl


@pytest.mark.parametrize("batch,seqlen,block_len,d_inner,conv", [
    (32, 16, 16, 4096, 0),   # the partial-bidirectional workload at full size
    (3, 64, 16, 136, 0),     # forward carried over 4 blocks, reverse confined to each
    (2, 48, 24, 72, 4),      # with the conv front-end in both directions
    (2, 5, 5, 64, 0),        # block shorter than a stage
])
def test_mamba_h_parity(r2l, batch, seqlen, block_len, d_inner, conv):
    pf, pr, h0 = mamba_h_inputs(3, batch, seqlen, d_inner, conv)
    y, hl = gpu_mamba_h(r2l, pf, pr, h0, block_len)
    ref, ref_hl = oracle.mamba_h(W.as_f64(pf["x"]), W.as_f64(pf["z"]), f64(pf), f64(pr), h0=W.as_f64(h0),
                                 block_len=block_len)
    assert rel_err(y.cpu().numpy(), ref) < TOL_BF16
    assert rel_err(hl.cpu().numpy(), ref_hl) < TOL_BF16
    check_status(r2l)


def test_forward_only_from_state(r2l):
    pf, _, h0 = mamba_h_inputs(5, 2, 300, 64)
    y, hl = gpu_mamba_h(r2l, pf, pf, h0, 300, rev=False)
    ref, ref_hl = oracle.mamba_h(W.as_f64(pf["x"]), W.as_f64(pf["z"]), f64(pf), None, h0=W.as_f64(h0))
    assert rel_err(y.cpu().numpy(), ref) < TOL_BF16
    assert rel_err(hl.cpu().numpy(), ref_hl) < TOL_BF16


def test_h_last_may_alias_h0(r2l):
    pf, pr, h0 = mamba_h_inputs(6, 4, 16, 256)
    gf, gr = dev(pf), dev(pr)
    gr["x"], gr["z"] = gf["x"], gf["z"]
    hd = h0.cuda()
    y1, hl1 = r2l.fwd_scan_from_state(gf["x"], gf["z"], gf, gr, h0=hd.clone(), rev_block_len=16)
    y2, hl2 = r2l.fwd_scan_from_state(gf["x"], gf["z"], gf, gr, h0=hd, h_last=hd, rev_block_len=16)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(hl1, hl2) and hl2.data_ptr() == hd.data_ptr()


# ----------------------------------------------------------------------------- bit-exact GPU invariants

@pytest.mark.parametrize("conv", [0, 4])
def test_flip_by_indexing_is_bit_exact(r2l, conv):
    """Right-to-left scan == flip(left-to-right scan of the flipped block), bit for bit."""
    p = W.scan_inputs(8, 4, 32, 256, conv_width=conv, io="bf16")
    g = dev(p)
    y = gpu_rev(r2l, g, 32)
    fl = {k: (v.flip(1).contiguous() if k in ("x", "dt", "B", "C", "z") else v) for k, v in g.items()}
    yf, _ = r2l.fwd_scan_from_state(fl["x"], fl["z"], fl, None, h0=None, want_h_last=False, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y, yf.flip(1))


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_balanced_launch_is_bit_exact(r2l, y_dtype):
    """The decode shape (64 rows x 2048 channels, 32-token blocks) runs as a balanced launch: 12 warps
    of each CTA take 64 channels (two per lane) and 4 take 32 (one per lane).  Per channel both
    kinds perform the same operations, so the reverse scan, and the forward scan from a state with
    its end state, equal bit for bit the plain launches of 8-row slices of the same inputs."""
    p = W.scan_inputs(21, 64, 32, 2048, conv_width=4, io="bf16")
    g = dev(p)
    rows = lambda a, b: {k: (v[a:b].contiguous() if k in ("x", "dt", "B", "C", "z") else v) for k, v in g.items()}
    y = gpu_rev(r2l, g, 32, y_dtype=y_dtype)
    assert torch.equal(y, torch.cat([gpu_rev(r2l, rows(r, r + 8), 32, y_dtype=y_dtype) for r in range(0, 64, 8)]))
    h0 = (torch.randn(64, 2048, 16, generator=torch.Generator().manual_seed(5)) * 0.1).cuda()
    yf, hl = r2l.fwd_scan_from_state(g["x"], g["z"], g, None, h0=h0, y_dtype=y_dtype)
    parts = [r2l.fwd_scan_from_state(rows(r, r + 8)["x"], rows(r, r + 8)["z"], rows(r, r + 8), None,
                                     h0=h0[r:r + 8].contiguous(), y_dtype=y_dtype) for r in range(0, 64, 8)]
    torch.cuda.synchronize()
    assert torch.equal(yf, torch.cat([a for a, _ in parts]))
    assert torch.equal(hl, torch.cat([b for _, b in parts]))
    check_status(r2l)


@pytest.mark.parametrize("block", [16, 64])
def test_small_launch_scan_is_bit_exact(r2l, block):
    """One decoding request (1 row, a 16- or 64-token block, 2048 channels) is too small to fill the
    GPU and runs on the four-lanes-per-channel kernel (8 rows on the plain launch); their rows equal
    bit for bit those of the same rows scanned inside a 64-row batch (the balanced launch), and the
    oracle at 2e-3."""
    p = W.scan_inputs(23, 64, block, 2048, conv_width=4, io="bf16")
    g = dev(p)
    y_all = gpu_rev(r2l, g, block)
    for r, n in ((0, 1), (37, 1), (63, 1), (24, 8)):
        part = {k: (v[r:r + n].contiguous() if k in ("x", "dt", "B", "C", "z") else v) for k, v in g.items()}
        yp = gpu_rev(r2l, part, block)
        assert torch.equal(yp, y_all[r:r + n])
    ref = oracle_rev(f64(p), block, rows=[37])
    assert rel_err(y_all[37:38].cpu().numpy(), ref) < TOL_BF16
    check_status(r2l)


def test_prefix_cache_continuation_is_bit_exact(r2l):
    """Forward scan of a prefix, its h_last passed as h0 to the rest == one-shot forward scan."""
    pf, _, h0 = mamba_h_inputs(9, 3, 96, 128)
    g = dev(pf)
    hd = h0.cuda()
    y_all, h_all = r2l.fwd_scan_from_state(g["x"], g["z"], g, None, h0=hd, y_dtype=torch.float32)
    cut = 40
    part = lambda a, b: {k: (v[:, a:b].contiguous() if k in ("x", "dt", "B", "C", "z") else v) for k, v in g.items()}
    g1, g2 = part(0, cut), part(cut, 96)
    y1, h_mid = r2l.fwd_scan_from_state(g1["x"], g1["z"], g1, None, h0=hd, y_dtype=torch.float32)
    y2, h_end = r2l.fwd_scan_from_state(g2["x"], g2["z"], g2, None, h0=h_mid, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([y1, y2], 1), y_all)
    assert torch.equal(h_end, h_all)


@pytest.mark.parametrize("batch,seqlen,rev_block,d_inner,conv,io", [
    (2, 320, 320, 136, 4, "bf16"),  # fully bidirectional: the reverse pass covers the whole window
    (3, 240, 80, 64, 0, "bf16"),    # reverse blocks longer than the fused kernel's 64 tokens
    (2, 64, 16, 128, 4, "f32"),     # fp32 inputs, active-block reverse
])
def test_bidir_scan_parity(r2l, batch, seqlen, rev_block, d_inner, conv, io):
    """Two-pass bidirectional scan (any reverse block length) against the oracle's mixer."""
    pf, pr, h0 = mamba_h_inputs(13, batch, seqlen, d_inner, conv, io=io)
    gf, gr = dev(pf), dev(pr)
    gr["x"], gr["z"] = gf["x"], gf["z"]
    y, hl = r2l.bidir_scan(gf["x"], gf["z"], gf, gr, rev_block_len=rev_block, h0=h0.cuda(), y_dtype=torch.float32)
    torch.cuda.synchronize()
    ref, ref_hl = oracle.mamba_h(W.as_f64(pf["x"]), W.as_f64(pf["z"]), f64(pf), f64(pr), h0=W.as_f64(h0),
                                 block_len=rev_block)
    tol = TOL_F32 if io == "f32" else TOL_BF16
    assert rel_err(y.cpu().numpy(), ref) < tol
    assert rel_err(hl.cpu().numpy(), ref_hl) < tol
    # the forward direction is the forward-only kernel: the same boundary state bit for bit
    _, hl_f = r2l.fwd_scan_from_state(gf["x"], gf["z"], gf, None, h0=h0.cuda(), y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(hl, hl_f)
    check_status(r2l)


def test_bidir_scan_agrees_with_fused_path(r2l):
    """Where both apply (16-token reverse blocks) the two-pass and the fused paths agree to fp32
    rounding, and bf16 outputs are produced by the combine pass."""
    pf, pr, h0 = mamba_h_inputs(14, 4, 48, 256, 4)
    gf, gr = dev(pf), dev(pr)
    gr["x"], gr["z"] = gf["x"], gf["z"]
    y1, _ = r2l.fwd_scan_from_state(gf["x"], gf["z"], gf, gr, h0=h0.cuda(), rev_block_len=16, y_dtype=torch.float32)
    y2, _ = r2l.bidir_scan(gf["x"], gf["z"], gf, gr, rev_block_len=16, h0=h0.cuda(), y_dtype=torch.float32)
    yb, _ = r2l.bidir_scan(gf["x"], gf["z"], gf, gr, rev_block_len=16, h0=h0.cuda(), y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert rel_err(y2.cpu().numpy(), y1.cpu().double().numpy()) < 1e-5
    ref, _ = oracle.mamba_h(W.as_f64(pf["x"]), W.as_f64(pf["z"]), f64(pf), f64(pr), h0=W.as_f64(h0), block_len=16)
    assert rel_err(yb.float().cpu().numpy(), ref) < TOL_BF16_OUT
    check_status(r2l)


def conv_state_at(x, cut):
    """[b, d, 3] fp32: the three inputs before position ``cut``, newest first."""
    return torch.stack([x[:, cut - 1 - j, :].float() for j in range(3)], dim=-1).contiguous()


@pytest.mark.parametrize("io,fused", [("bf16", False), ("f32", False), ("bf16", True)])
def test_conv_state_parity(r2l, io, fused):
    """Forward scan with the width-4 convolution resumed from a cached convolution state and
    boundary state (alone, and fused with the block-confined reverse scan)."""
    batch, L, d, bl = 3, 48, 136, 16
    pf, pr, h0 = mamba_h_inputs(11, batch, L, d, conv=4, io=io)
    cs = W.conv_state(11, batch, d)
    gf, gr = dev(pf), dev(pr)
    gr["x"], gr["z"] = gf["x"], gf["z"]
    gf["conv_state"] = cs.cuda()
    gf["conv_state_out"] = torch.full_like(gf["conv_state"], float("nan"))
    y, hl = r2l.fwd_scan_from_state(gf["x"], gf["z"], gf, gr if fused else None, h0=h0.cuda(), rev_block_len=bl,
                                    y_dtype=torch.float32)
    torch.cuda.synchronize()
    of = dict(f64(pf), conv_state=W.as_f64(cs))
    ref, ref_hl, ref_cs = oracle.mamba_h(of["x"], of["z"], of, f64(pr) if fused else None, h0=W.as_f64(h0),
                                         block_len=bl, want_conv_state=True)
    tol = TOL_F32 if io == "f32" else TOL_BF16
    assert rel_err(y.cpu().numpy(), ref) < tol
    assert rel_err(hl.cpu().numpy(), ref_hl) < tol
    np.testing.assert_array_equal(gf["conv_state_out"].cpu().numpy(), ref_cs)
    check_status(r2l)


@pytest.mark.parametrize("chunk", [1, 3, 16])
def test_conv_state_chunked_decode_is_bit_exact(r2l, chunk):
    """Decoding chunk by chunk with h and the convolution state updated in place (h_last
    aliasing h0, conv_state_out aliasing conv_state) == one forward scan, bit for bit."""
    batch, L, d = 2, 40, 128
    pf, _, h0 = mamba_h_inputs(12, batch, L, d, conv=4)
    g = dev(pf)
    hd = h0.cuda()
    y_all, h_all = r2l.fwd_scan_from_state(g["x"], g["z"], g, None, h0=hd, y_dtype=torch.float32)
    h = hd.clone()
    cs = torch.zeros(batch, d, 3, device="cuda")
    parts = []
    for a in range(0, L, chunk):
        gc = {k: (v[:, a:min(a + chunk, L)].contiguous() if k in ("x", "dt", "B", "C", "z") else v)
              for k, v in g.items()}
        gc["conv_state"], gc["conv_state_out"] = cs, cs
        yc, _ = r2l.fwd_scan_from_state(gc["x"], gc["z"], gc, None, h0=h, h_last=h, y_dtype=torch.float32)
        parts.append(yc)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, 1), y_all)
    assert torch.equal(h, h_all)
    assert torch.equal(cs, conv_state_at(g["x"], L))
    check_status(r2l)


@pytest.mark.parametrize("conv", [0, 4])
def test_block_confinement_on_gpu(r2l, conv):
    p = W.scan_inputs(10, 2, 96, 128, conv_width=conv, io="bf16")
    g = dev(p)
    y = gpu_rev(r2l, g, 32)
    q = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in g.items()}
    for k in ("x", "dt", "B", "C", "z"):
        q[k][:, :32] = torch.randn_like(q[k][:, :32].float()).to(q[k].dtype)
        q[k][:, 64:] = torch.randn_like(q[k][:, 64:].float()).to(q[k].dtype)
    yq = gpu_rev(r2l, q, 32)
    assert torch.equal(y[:, 32:64], yq[:, 32:64])


# ----------------------------------------------------------------------------- serving sweep

@pytest.mark.parametrize("batch", W.SWEEP_BATCHES)
@pytest.mark.parametrize("block", W.SWEEP_BLOCKS)
def test_serving_sweep_layers(r2l, batch, block):
    """14 independent sidecars per step, each seeded separately; layers 0 and 13 checked on
    sampled rows against the oracle, fp32 outputs at the bf16-input bound and bf16 outputs at the
    bf16-output bound; every layer checked for finite outputs."""
    wl = W.sweep_workload(batch, block)
    rows = np.unique(np.array([0, batch // 2, batch - 1]))
    for layer in range(wl.layers):
        p = W.scan_inputs(wl.wid, batch, block, wl.d_inner, io="bf16", layer=layer)
        g = dev(p)
        y = gpu_rev(r2l, g, block, torch.bfloat16)
        assert torch.isfinite(y.float()).all()
        if layer in (0, wl.layers - 1):
            ref = oracle_rev(f64(p), block, rows=rows)
            y32 = gpu_rev(r2l, g, block, torch.float32)
            assert rel_err(y32.cpu().numpy()[rows], ref) < TOL_BF16
            assert rel_err(y.float().cpu().numpy()[rows], ref) < TOL_BF16_OUT
    check_status(r2l)


# ----------------------------------------------------------------------------- edge cases

def test_outputs_stay_inside_their_extent(r2l):
    """Canary NaNs around y: every element of y is written, nothing outside it."""
    p = W.scan_inputs(11, 3, 40, 72, conv_width=4, io="bf16")
    g = dev(p)
    n = 3 * 40 * 72
    buf = torch.full((n + 256,), float("nan"), device="cuda")
    y = buf[64:64 + n].view(3, 40, 72)
    r2l.r2l_scan_block(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], g["conv_w"],
                       g["conv_b"], block_len=20, y=y)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    assert torch.isnan(buf[:64]).all() and torch.isnan(buf[64 + n:]).all()


def test_empty_batch_is_noop(r2l):
    p = W.scan_inputs(12, 1, 8, 64, io="bf16")
    g = dev(p)
    e = {k: (v[:0] if k in ("x", "dt", "B", "C", "z") else v) for k, v in g.items()}
    y = r2l.r2l_scan_block(e["x"], e["dt"], e["B"], e["C"], e["z"], e["A"], e["D"], e["dt_bias"], block_len=8)
    assert y.shape == (0, 8, 64)


def test_misaligned_pointer_rejected(r2l):
    p = W.scan_inputs(13, 1, 8, 64, io="bf16")
    g = dev(p)
    big = torch.zeros(8 * 64 + 1, dtype=torch.bfloat16, device="cuda")
    x_bad = big[1:].view(1, 8, 64)  # 2-byte offset
    with pytest.raises(r2l.R2LError) as ei:
        r2l.r2l_scan_block(x_bad, g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], block_len=8)
    assert ei.value.status == r2l.R2L_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- launch shapes, both directions

@pytest.mark.parametrize("batch,d_inner,conv,path", [
    (48, 1024, 4, "several CTAs per SM"),
    (24, 1024, 4, "about one wave"),
    (3, 1024, 0, "few warps: narrow CTAs"),
])
def test_scan_shapes_both_directions(r2l, batch, d_inner, conv, path):
    p = W.scan_inputs(14, batch, 32, d_inner, conv_width=conv, io="bf16")
    y = gpu_rev(r2l, dev(p), 32)
    rows = np.unique(np.array([0, batch // 2, batch - 1]))
    ref = oracle_rev(f64(p), 32, rows=rows)
    assert rel_err(y.cpu().numpy()[rows], ref) < TOL_BF16, path
    # forward direction through the same path, from a cached state
    h0 = W.boundary_state(14, batch, d_inner)
    g = dev(p)
    yf, hl = r2l.fwd_scan_from_state(g["x"], g["z"], g, None, h0=h0.cuda(), y_dtype=torch.float32)
    torch.cuda.synchronize()
    reff, refh = oracle.mamba_h(W.as_f64(p["x"])[rows], W.as_f64(p["z"])[rows],
                                {k: (v[rows] if k in ("dt", "B", "C") else v) for k, v in f64(p).items()}, None,
                                h0=W.as_f64(h0)[rows])
    assert rel_err(yf.cpu().numpy()[rows], reff) < TOL_BF16, path
    assert rel_err(hl.cpu().numpy()[rows], refh) < TOL_BF16, path


# ----------------------------------------------------------------------------- scan backward

def _bwd_case(wid, batch, seqlen, d_inner, io, gate, dy_dtype):
    p = W.scan_inputs(wid, batch, seqlen, d_inner, io=io, gate=gate)
    dy = W.normal(wid, 0, "u_probe", (batch, seqlen, d_inner), io="bf16" if dy_dtype == torch.bfloat16 else "f32")
    return p, dy


@pytest.mark.parametrize("batch,seqlen,block_len,d_inner,io,gate,dy_dtype", [
    (3, 64, 32, 64, "bf16", True, torch.float32),    # two blocks per row, gate
    (2, 48, 16, 128, "bf16", False, torch.bfloat16),  # no gate, bf16 dy
    (2, 64, 64, 32, "f32", True, torch.float32),     # the longest block, fp32 inputs
    (5, 20, 20, 48, "bf16", True, torch.float32),    # a block that is not a power of two
    (2, 36, 18, 32, "f32", True, torch.float32),     # 18-token blocks: the last 4-token chunk holds 2
    (3, 6, 3, 16, "f32", True, torch.bfloat16),      # blocks shorter than one chunk
])
def test_scan_bwd_parity(r2l, batch, seqlen, block_len, d_inner, io, gate, dy_dtype):
    p, dy = _bwd_case(15, batch, seqlen, d_inner, io, gate, dy_dtype)
    g = dev(p)
    got = r2l.r2l_scan_block_bwd(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], dy.cuda(),
                                 block_len=block_len)
    torch.cuda.synchronize()
    o = f64(p)
    ref = oracle.scan_bwd(o["x"], o["dt"], o["B"], o["C"], o["z"], o["A"], o["D"], o["dt_bias"], W.as_f64(dy),
                          block_len=block_len)
    tol = TOL_F32 if io == "f32" else TOL_BF16
    for k, v in ref.items():
        if v is None:
            assert got[k] is None
            continue
        assert rel_err(got[k].cpu().numpy(), v) < tol, k
    check_status(r2l)


def test_scan_bwd_decode_step_full_size(r2l):
    """The decode-step shapes (64 x 32-token blocks, d_inner 2048, gate) against the full oracle."""
    p, dy = _bwd_case(16, 64, 32, 2048, "bf16", True, torch.float32)
    g = dev(p)
    got = r2l.r2l_scan_block_bwd(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], dy.cuda(),
                                 block_len=32)
    torch.cuda.synchronize()
    o = f64(p)
    ref = oracle.scan_bwd(o["x"], o["dt"], o["B"], o["C"], o["z"], o["A"], o["D"], o["dt_bias"], W.as_f64(dy),
                          block_len=32)
    for k, v in ref.items():
        if v is None:  # no convolution
            assert got[k] is None, k
            continue
        assert rel_err(got[k].cpu().numpy(), v) < TOL_BF16, k
    check_status(r2l)


@pytest.mark.parametrize("batch,seqlen,block_len,d_inner,io,gate", [
    (2, 64, 32, 64, "bf16", True),    # decode-step blocks with the width-4 convolution front-end
    (3, 36, 18, 48, "f32", False),    # ragged last chunk; taps past the block edge read zero
    (2, 6, 3, 16, "f32", True),       # blocks shorter than the convolution window
    (8, 32, 32, 512, "bf16", True),   # a larger slice of the decode step
])
def test_scan_bwd_conv_parity(r2l, batch, seqlen, block_len, d_inner, io, gate):
    """The gradient through the convolution front-end (dx of the raw x, dconv_w, dconv_b and all the
    scan's own gradients) against the oracle."""
    p = W.scan_inputs(18, batch, seqlen, d_inner, 16, 4, io=io, gate=gate)
    dy = W.normal(18, 0, "u_probe", (batch, seqlen, d_inner), io="f32")
    g = dev(p)
    got = r2l.r2l_scan_block_bwd(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], dy.cuda(),
                                 block_len=block_len, conv_w=g["conv_w"], conv_b=g["conv_b"])
    torch.cuda.synchronize()
    o = f64(p)
    ref = oracle.scan_bwd(o["x"], o["dt"], o["B"], o["C"], o["z"], o["A"], o["D"], o["dt_bias"], W.as_f64(dy),
                          block_len=block_len, conv_w=o["conv_w"], conv_b=o["conv_b"])
    tol = TOL_F32 if io == "f32" else TOL_BF16
    assert ref["dconv_w"] is not None and ref["dconv_b"] is not None
    for k, v in ref.items():
        if v is None:
            assert got[k] is None, k
            continue
        assert rel_err(got[k].cpu().numpy(), v) < tol, k
    check_status(r2l)


def test_empty_inputs_on_the_newer_paths(r2l):
    """Zero-sized batches are no-ops for the bidirectional scan and the sidecar; the scan gradient
    still writes its parameter sums (zeros)."""
    p = W.scan_inputs(17, 1, 32, 64, io="bf16")
    g = dev(p)
    e = {k: (v[:0] if k in ("x", "dt", "B", "C", "z") else v) for k, v in g.items()}
    y, _ = r2l.bidir_scan(e["x"], e["z"], e, e, rev_block_len=32, y_dtype=torch.float32)
    assert y.shape == (0, 32, 64)
    dy = torch.zeros((0, 32, 64), device="cuda")
    grads = r2l.r2l_scan_block_bwd(e["x"], e["dt"], e["B"], e["C"], e["z"], e["A"], e["D"], e["dt_bias"], dy,
                                   block_len=32)
    torch.cuda.synchronize()
    for k in ("dA", "dD", "ddt_bias"):
        assert torch.count_nonzero(grads[k]) == 0
    gc = dev(W.scan_inputs(17, 1, 32, 64, 16, 4, io="bf16"))
    ec = {k: (v[:0] if k in ("x", "dt", "B", "C", "z") else v) for k, v in gc.items()}
    grads = r2l.r2l_scan_block_bwd(ec["x"], ec["dt"], ec["B"], ec["C"], ec["z"], ec["A"], ec["D"], ec["dt_bias"], dy,
                                   block_len=32, conv_w=ec["conv_w"], conv_b=ec["conv_b"])
    torch.cuda.synchronize()
    for k in ("dA", "dD", "ddt_bias", "dconv_w", "dconv_b"):
        assert torch.count_nonzero(grads[k]) == 0, k
    w = dev(W.sidecar_weights(17, 64, 64, dt_rank=16))
    hidden = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    assert r2l.r2l_sidecar_forward(hidden, w, 0, 32, 32, 0.05).shape == (0, 64)
    check_status(r2l)
