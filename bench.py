#!/usr/bin/env python
"""Benchmark of the R2LM parallel-decode sidecar step on B200.

One step = the whole hot path over one batch: the right-to-left selective scan of a
64 x 32-token generation block (d_inner 2048, d_state 16, width-4 conv, gate) followed by
the s-gated residual hidden += s * y . W_out^T (d_model 2048): one r2l_decode_step call of
libr2l's C ABI (two kernels; the scan pulls the residual's W_out and hidden into L2 as it runs).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The K timed steps are replayed from CUDA graphs captured after the warm-up (the same call per
step, captured on a side stream); per-kernel times come from each kernel alone, K launches replayed
the same way, and the end-to-end figure from direct calls with host buffers.

N > 1 is launched with torchrun (one rank per GPU); every rank runs its own batch of 64
(independent problems, no data-path collective: weak scaling).  Rank 0 prints one JSON line.
--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload (the method's only other implementation here).
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "R2L scan tokens/s & HBM GB/s (frac of peak), B=64 blk=32 d_inner=2048"
WL = W.WORKLOADS["decode_b64_blk32"]
NSETS = 6  # rotating input sets: 6 x 48.5 MiB > 2 x 126 MB L2
GRAPH_STEPS = 100 * NSETS  # decode steps per captured CUDA graph in the timed region
SCAN_KERNEL_SRC = os.path.join(ROOT, "reverse_mamba_selective_b200", "csrc", "scan_kernels.cuh")
GEMM_KERNEL_SRC = os.path.join(ROOT, "reverse_mamba_selective_b200", "csrc", "residual_tc.cuh")
FE_KERNEL_SRC = os.path.join(ROOT, "reverse_mamba_selective_b200", "csrc", "frontend_tc.cuh")
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def scan_bytes_per_step(wl=WL) -> int:
    """Algorithmic HBM bytes of one scan launch: x, dt, z in + y out (bf16) per (b, t, d),
    B and C (bf16) per (b, t, n), and the fp32 parameters once."""
    tok = wl.batch * wl.seqlen
    act = tok * wl.d_inner * 2 * 4 + tok * wl.d_state * 2 * 2
    params = wl.d_inner * wl.d_state * 4 + 2 * wl.d_inner * 4 + (wl.d_inner * 5 * 4 if wl.conv_width else 0)
    return act + params


def residual_bytes_per_step(wl=WL) -> int:
    """Algorithmic bytes of the residual GEMM: y and W_out read once, hidden read + written (bf16)."""
    M = wl.batch * wl.seqlen
    return M * wl.d_inner * 2 + wl.d_model * wl.d_inner * 2 + 2 * M * wl.d_model * 2


def residual_flops_per_step(wl=WL) -> int:
    return 2 * wl.batch * wl.seqlen * wl.d_model * wl.d_inner


# MUFU transcendental operations the scan issues per (token, channel): 16 state exponentials,
# one for softplus, and 2^x + reciprocal for each of the two SiLUs (conv front-end and gate).
SCAN_MUFU_PER_ELEMENT = 16 + 1 + (2 if WL.conv_width else 0) + 2
B200_SMS = 148
MUFU_PER_CLK_PER_SM = 16  # special-function results per clock per SM (2^x, lg2, reciprocal)


def scan_mufu_ops_per_step(wl=WL) -> int:
    return wl.batch * wl.seqlen * wl.d_inner * SCAN_MUFU_PER_ELEMENT


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


def file_hash(path: str) -> str:
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def profiled_traffic(kernel: str, src: str):
    """DRAM bytes per launch from a committed ncu summary, or None if the kernel changed since."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    d = json.load(open(PROFILE_TRAFFIC)).get(kernel)
    if not d or d.get("source_sha256_16") != file_hash(src):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(gpu_index), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in out.strip().splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- reference arm (CPU oracle)

_SAMPLES = {}


def _row_sample(row: int, wl=WL):
    """Seeded inputs of one batch row of the decode step, widened to fp64 (drawn once, not timed)."""
    key = row % 4
    if key not in _SAMPLES:
        p = W.scan_inputs(wl.wid, 1, wl.seqlen, wl.d_inner, conv_width=wl.conv_width, io="bf16", layer=key)
        res = W.residual_inputs(wl.wid, wl.seqlen, wl.d_model, wl.d_inner, io="bf16", layer=key)
        f = {k: W.as_f64(v) for k, v in p.items()}
        y_in = np.full((wl.seqlen, wl.d_inner), 0.5)  # the residual's cost does not depend on the values
        _SAMPLES[key] = (f, W.as_f64(res["hidden"]), W.as_f64(res["W_out"]), y_in)
    return _SAMPLES[key]


def _channel_slice(f, c0: int, c1: int):
    c = slice(c0, c1)
    return {k: (f[k][..., c] if k in ("x", "dt", "z") else f[k][c] if k in ("A", "D", "dt_bias", "conv_w", "conv_b")
                else f[k]) for k in f}


def _oracle_part(part, wl=WL):
    """One unit of oracle work: the reverse scan of a channel range of one batch row, or the
    residual of a token range of one row."""
    import oracle

    if part[0] == "scan":
        sub = part[1]
        oracle.scan(sub["x"], sub["dt"], sub["B"], sub["C"], sub["z"], sub["A"], sub["D"], sub["dt_bias"],
                    sub["conv_w"], sub["conv_b"], reverse=True, block_len=wl.block_len)
    else:
        _, hid, Wo, y_in = part
        oracle.residual(hid, y_in, Wo, wl.s)


def oracle_step_sample(chans: int, toks: int, row: int = 0, wl=WL):
    """Time the fp64 oracle on a sample of one batch row of the decode step and scale it to the
    whole row: the reverse scan of `chans` of its d_inner channels (channels are independent)
    and the residual of `toks` of its tokens (all d_model outputs).  Returns (seconds for one
    full row, tokens of that row)."""
    import oracle

    oracle.build()
    f, hid, Wo, y_in = _row_sample(row, wl)
    sub = _channel_slice(f, 0, chans)
    t0 = time.perf_counter()
    oracle.scan(sub["x"], sub["dt"], sub["B"], sub["C"], sub["z"], sub["A"], sub["D"], sub["dt_bias"],
                sub["conv_w"], sub["conv_b"], reverse=True, block_len=wl.block_len)
    t1 = time.perf_counter()
    oracle.residual(hid[:toks], y_in[:toks], Wo, wl.s)
    t2 = time.perf_counter()
    return (t1 - t0) * (wl.d_inner / chans) + (t2 - t1) * (wl.seqlen / toks), wl.seqlen


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_rows_all_cores(rows: int, chans: int = 64, toks: int = 1, wl=WL):
    """The oracle on `rows` full batch rows of the decode step on every host core this process may
    run on: each row's scan is cut into ranges of `chans` channels and its residual into ranges of
    `toks` tokens (channels and tokens are independent), and the units run on a thread pool (the
    oracle's C calls release the GIL).  Returns (wall seconds, tokens, threads)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    oracle.build()
    threads = host_cores()
    units = []
    for r in range(rows):
        f, hid, Wo, y_in = _row_sample(r, wl)
        units += [("scan", _channel_slice(f, c, c + chans)) for c in range(0, wl.d_inner, chans)]
        units += [("residual", hid[t:t + toks], Wo, y_in[t:t + toks]) for t in range(0, wl.seqlen, toks)]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(_oracle_part, units[:threads]))  # start the pool's threads and load the oracle library
        t0 = time.perf_counter()
        list(ex.map(_oracle_part, units))
        secs = time.perf_counter() - t0
    return secs, rows * wl.seqlen, min(threads, len(units))


def cpu_baseline(rows: int = 64):
    """The oracle on `rows` full batch rows of the decode step (all channels, all 32 tokens of
    each): once on one thread and once on every host core, each scaled to tokens/s; the default
    covers the whole step (~5-10 s single-threaded)."""
    secs, tokens = 0.0, 0
    for r in range(rows):
        s, t = oracle_step_sample(WL.d_inner, WL.seqlen, row=r)
        secs += s
        tokens += t
    rows_mc = max(rows, host_cores() // 8)
    secs_mc, tokens_mc, threads = oracle_rows_all_cores(rows_mc)
    return {"value": tokens_mc / secs_mc, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows_mc} batch rows ({tokens_mc} tokens) of the decode step through the fp64 C oracle on "
                      f"{threads} host threads (each row cut into 64-channel and 1-token units): reverse scan of all "
                      f"{WL.d_inner} channels + residual of every token ({secs_mc:.2f} s wall; inputs of 4 distinct "
                      f"seeded rows reused)",
            "single_thread": {"value": tokens / secs, "unit": "tokens/s", "cores": 1,
                              "sample": f"{rows} batch rows ({tokens} tokens), one thread, {secs:.2f} s"}}


def run_reference(args, rank, world):
    """Reference arm: the fp64 oracle on the host cores, one bounded sample of the decode step per
    step; the sample shrinks with K so that the whole run ends within a few minutes."""
    if rank != 0:
        return
    small = args.steps + args.warmup <= 60
    rows = 8 if small else 1  # batch rows of the decode step per timed step, all channels and tokens
    for i in range(args.warmup):
        oracle_rows_all_cores(1)
    total, tokens, threads = 0.0, 0, 1
    for i in range(args.steps):
        s, t, threads = oracle_rows_all_cores(rows)
        total += s
        tokens += t
    value = tokens / total
    sample = (f"each step: {rows} batch row(s) of the decode step through the fp64 C oracle on {threads} host "
              f"threads: reverse scan of all {WL.d_inner} channels and residual of all {WL.seqlen} tokens per row")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {"workload": WL.name},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank timing over all ranks (identity without a process group)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- our arm

class StepSet:
    """Device-resident inputs/outputs of one decode step, plus prebuilt C-ABI arguments."""

    def __init__(self, r2l, seed_layer: int, device):
        p = W.scan_inputs(WL.wid, WL.batch, WL.seqlen, WL.d_inner, conv_width=WL.conv_width, io="bf16",
                          layer=seed_layer)
        res = W.residual_inputs(WL.wid, WL.tokens, WL.d_model, WL.d_inner, io="bf16", layer=seed_layer)
        self.host = {**p, **res}
        self.dev = {k: (v.to(device) if v is not None else None) for k, v in self.host.items()}
        d = self.dev
        self.y = torch.empty((WL.batch, WL.seqlen, WL.d_inner), dtype=torch.bfloat16, device=device)
        self.args = r2l.make_scan_args(d["x"], d["dt"], d["B"], d["C"], d["z"], d["A"], d["D"], d["dt_bias"],
                                       d["conv_w"], d["conv_b"], WL.block_len)
        self.args_ref = ctypes.byref(self.args)


# ----------------------------------------------------------------------------- the whole sidecar

DT_RANK = -(-WL.d_model // 16)  # standard Mamba-1 sizing: ceil(d_model / 16) = 128


class SidecarSet:
    """Device-resident weights, hidden state and workspaces of one sidecar (hidden -> hidden),
    plus separate intermediate buffers for timing the stages one at a time."""

    def __init__(self, r2l, lib, layer: int, device):
        M, D, Dm = WL.tokens, WL.d_inner, WL.d_model
        w = W.sidecar_weights(WL.wid, Dm, D, d_state=WL.d_state, dt_rank=DT_RANK, conv_width=WL.conv_width,
                              layer=layer)
        self.w = {k: (v.to(device) if v is not None else None) for k, v in w.items()}
        self.sw = r2l.make_sidecar_weights(self.w)
        self.sw_ref = ctypes.byref(self.sw)
        self.hidden = W.normal(WL.wid, layer, "hidden", (M, Dm)).to(device)
        self.ws = torch.empty(r2l.sidecar_workspace_size(self.sw, WL.batch, WL.seqlen), dtype=torch.uint8,
                              device=device)
        bf = dict(dtype=torch.bfloat16, device=device)
        self.u, self.z, self.dt, self.y = (torch.empty((M, D), **bf) for _ in range(4))
        self.dt_low = torch.empty((M, DT_RANK), **bf)
        self.B, self.C = (torch.empty((M, WL.d_state), **bf) for _ in range(2))
        self.part = torch.empty(lib.r2l_x_proj_workspace_size(M, D, DT_RANK, WL.d_state), dtype=torch.uint8,
                                device=device)
        r3 = lambda t: t.view(WL.batch, WL.seqlen, -1)
        self.scan_args = r2l.make_scan_args(r3(self.u), r3(self.dt), r3(self.B), r3(self.C), r3(self.z),
                                            self.w["A"], self.w["D"], self.w["dt_bias"], None, None, WL.block_len)


def sidecar_flops(M=WL.tokens, D=WL.d_inner, Dm=WL.d_model, R=DT_RANK, N=WL.d_state):
    return {"in_proj": 2 * M * 2 * D * Dm, "x_proj": 2 * M * (R + 2 * N) * D, "dt_proj": 2 * M * D * R,
            "residual": 2 * M * Dm * D}


def measure_sidecar(r2l, lib, device, stream, K: int, warmup: int, dist, rank: int):
    """Time the whole sidecar (hidden -> hidden: in_proj + conv, x_proj, dt_proj, the right-to-left
    scan and the residual, six launches) with the same discipline as the headline step: first as
    K direct calls through the C ABI, then replayed from a CUDA graph (no host work between
    launches, as a serving loop would run it), and each stage alone from a graph over the same
    rotating sets."""
    sets = [SidecarSet(r2l, lib, 200 + 100 * rank + i, device) for i in range(NSETS)]
    M, D, Dm, R, N = WL.tokens, WL.d_inner, WL.d_model, DT_RANK, WL.d_state
    bfc = r2l.R2L_BF16

    def chk(rc, what):
        if rc:
            raise r2l.R2LError(rc, what)

    def fused(i, sh):
        st = sets[i % NSETS]
        # the sign of s alternates between a set's uses so that hidden stays near its initial scale
        sgn = -1.0 if (i // NSETS) % 2 else 1.0
        chk(lib.r2l_sidecar_forward(st.sw_ref, WL.batch, WL.seqlen, WL.block_len, ctypes.c_float(sgn * WL.s),
                                    st.hidden.data_ptr(), st.ws.data_ptr(), st.ws.numel(), sh), "r2l_sidecar_forward")

    stages = {
        "in_proj": lambda st, sh: chk(lib.r2l_in_proj(st.hidden.data_ptr(), st.w["W_in"].data_ptr(),
                                                      st.w["conv_w"].data_ptr(), st.w["conv_b"].data_ptr(), WL.batch,
                                                      WL.seqlen, WL.block_len, Dm, D, st.u.data_ptr(), st.z.data_ptr(),
                                                      sh), "r2l_in_proj"),
        "x_proj": lambda st, sh: chk(lib.r2l_x_proj(st.u.data_ptr(), st.w["W_x"].data_ptr(), M, D, R, N,
                                                    st.dt_low.data_ptr(), st.B.data_ptr(), st.C.data_ptr(),
                                                    st.part.data_ptr(), st.part.numel(), sh), "r2l_x_proj"),
        "dt_proj": lambda st, sh: chk(lib.r2l_dt_proj(st.dt_low.data_ptr(), st.w["W_dt"].data_ptr(), M, R, D,
                                                      st.dt.data_ptr(), sh), "r2l_dt_proj"),
        "scan": lambda st, sh: chk(lib.r2l_scan_block(ctypes.byref(st.scan_args), st.y.data_ptr(), bfc, sh),
                                   "r2l_scan_block"),
        "residual": lambda st, sh: chk(lib.r2l_residual_apply(st.hidden.data_ptr(), st.y.data_ptr(),
                                                              st.w["W_out"].data_ptr(), ctypes.c_float(WL.s), M, Dm, D,
                                                              bfc, sh), "r2l_residual_apply"),
    }
    sh0 = stream.cuda_stream
    for i in range(max(warmup, NSETS)):
        fused(i, sh0)
    for st in sets:  # valid intermediates for the stage-alone runs
        for fn in stages.values():
            fn(st, sh0)
    torch.cuda.synchronize()
    if r2l.r2l_device_status() != r2l.R2L_OK:
        raise RuntimeError("device status not OK after the sidecar warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def graph_of(launch, count):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(device)
        cs.wait_stream(stream)
        with torch.cuda.graph(g, stream=cs, capture_error_mode="thread_local"):
            for i in range(count):
                launch(i, cs.cuda_stream)
        torch.cuda.synchronize()
        return g

    def time_replays(g, reps):
        g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(K):
        fused(i, sh0)
    e1.record(stream)
    torch.cuda.synchronize()
    step_ms = max_over_ranks(e0.elapsed_time(e1), dist, device) / K
    per_graph = 4 * NSETS  # steps captured per graph (each set used four times, s alternating)
    g = graph_of(fused, per_graph)
    reps = max(1, K // per_graph)
    if dist is not None:
        dist.barrier()
    step_graph_ms = max_over_ranks(time_replays(g, reps), dist, device) / (reps * per_graph)
    del g
    stage_us = {}
    for name, fn in stages.items():
        gs = graph_of(lambda i, sh, fn=fn: fn(sets[i % NSETS], sh), per_graph)
        stage_us[name] = 1e3 * time_replays(gs, max(1, min(reps, 50))) / (max(1, min(reps, 50)) * per_graph)
        del gs
    if r2l.r2l_device_status() != r2l.R2L_OK:
        raise RuntimeError("device status not OK after the sidecar timing")
    return step_ms, step_graph_ms, stage_us


# ----------------------------------------------------------------------------- scan backward

# MUFU operations the gradient needs per (token, channel) at least: the 16 state exponentials
# (computed once, if every state were kept), one exponential for the softplus and its slope (the
# slope's reciprocal is one more) and the gate's SiLU (2).  The kernel keeps only a checkpoint every
# 4 tokens, so it issues the state exponentials up to three times (forward pass, chunk recompute,
# adjoint); its count is reported beside the roofline, which uses the minimum.
SCAN_BWD_MUFU_PER_ELEMENT = 16 + 1 + 1 + 2
SCAN_BWD_CHUNK = 4


def scan_bwd_mufu_issued(block_len: int) -> float:
    """MUFU operations the gradient kernel issues per (token, channel): the forward pass (16 + the
    softplus) skips the leftmost chunk of each block; the chunk recompute (16 + the softplus + the
    slope's reciprocal) and the adjoint (16 + the gate's 2) cover every token."""
    first = (block_len - min(SCAN_BWD_CHUNK, block_len)) / block_len
    return first * (16 + 1) + (16 + 1 + 1) + (16 + 2)


def measure_scan_bwd(r2l, device, stream, K: int, dist):
    """Gradient of the right-to-left block scan on the decode-step shapes (64 x 32-token blocks,
    d_inner 2048, gate, no convolution: the sidecar runs its convolution in in_proj), over six
    rotating input sets; one call = the kernel that zeroes the accumulated gradients + the gradient
    kernel."""
    lib = r2l.load()
    sets = []
    for i in range(NSETS):
        p = {k: (v.to(device) if v is not None else None)
             for k, v in W.scan_inputs(WL.wid, WL.batch, WL.seqlen, WL.d_inner, layer=300 + i).items()}
        dy = W.normal(WL.wid, 300 + i, "u_probe", (WL.batch, WL.seqlen, WL.d_inner), io="f32").to(device)
        a = r2l.make_scan_args(p["x"], p["dt"], p["B"], p["C"], p["z"], p["A"], p["D"], p["dt_bias"], None, None,
                               WL.block_len)
        f32 = dict(dtype=torch.float32, device=device)
        g = [torch.empty((WL.batch, WL.seqlen, WL.d_inner), **f32), torch.empty((WL.batch, WL.seqlen, WL.d_inner), **f32),
             torch.empty((WL.batch, WL.seqlen, 16), **f32), torch.empty((WL.batch, WL.seqlen, 16), **f32),
             torch.empty((WL.batch, WL.seqlen, WL.d_inner), **f32), torch.empty((WL.d_inner, 16), **f32),
             torch.empty(WL.d_inner, **f32), torch.empty(WL.d_inner, **f32)]
        sets.append((p, dy, a, g))
    sh = stream.cuda_stream

    def launch(i):
        p, dy, a, g = sets[i % NSETS]
        rc = lib.r2l_scan_block_bwd(ctypes.byref(a), dy.data_ptr(), r2l.R2L_F32, *[t.data_ptr() for t in g], None,
                                    None, sh)
        if rc:
            raise r2l.R2LError(rc, "r2l_scan_block_bwd")

    for i in range(max(3, NSETS)):
        launch(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    e0.record(stream)
    for i in range(K):
        launch(i)
    e1.record(stream)
    torch.cuda.synchronize()
    us = 1e3 * max_over_ranks(e0.elapsed_time(e1), dist, device) / K
    if r2l.r2l_device_status() != r2l.R2L_OK:
        raise RuntimeError("device status not OK after the backward timing")
    sm_mhz = measured_peaks().get("sm_max_mhz") or 1965.0
    mufu_peak = B200_SMS * MUFU_PER_CLK_PER_SM * sm_mhz * 1e6 / 1e12
    mufu = WL.tokens * WL.d_inner * SCAN_BWD_MUFU_PER_ELEMENT / (us * 1e-6) / 1e12
    issued = scan_bwd_mufu_issued(WL.block_len)
    return {"workload": f"gradient of the reverse block scan, batch {WL.batch}, block {WL.block_len}, "
                        f"d_inner {WL.d_inner}, d_state 16, gate, no conv",
            "us_per_launch": us, "tokens_per_s": WL.tokens / (us * 1e-6), "steps": K,
            "roofline": {"bound": "alu", "achieved": mufu, "peak": mufu_peak, "frac": mufu / mufu_peak,
                         "unit": "Top/s (MUFU transcendental results)",
                         "work": f"{SCAN_BWD_MUFU_PER_ELEMENT} MUFU ops per (token, channel), the minimum",
                         "issued_per_element": issued, "issued_frac": mufu * issued / SCAN_BWD_MUFU_PER_ELEMENT
                         / mufu_peak}}


# ----------------------------------------------------------------------------- comparators

MH = W.WORKLOADS["mamba_h_b32_blk16"]
MH_PREFIX = 1024  # tokens of clean prefix behind the active block


def measure_comparators(r2l, device, stream, K: int, dist):
    """One denoising step of a Mamba mixer layer on the partial-bidirectional workload (batch 32,
    d_inner 4096, 16-token active block behind a 1024-token prefix), two ways:
      * partial bidirectionality: the forward scan resumes from the cached prefix state over the
        active block and the reverse scan is confined to it (fused kernel, 16 tokens);
      * full-window bidirectionality (the earlier hybrids' way): the reverse states depend on the
        active tokens, so nothing of the prefix can be cached and both directions rescan the whole
        1040-token window (two-pass scan, reverse block = window).
    Inputs for the full window are drawn on the device (timing only)."""
    B_, L_, D_ = MH.batch, MH.seqlen, MH.d_inner
    psets = []  # 8 rotating sets of ~21 MB each (> L2), as for the headline step
    for i in range(8):
        pf = {k: (v.to(device) if v is not None else None) for k, v in W.scan_inputs(MH.wid, B_, L_, D_, layer=i).items()}
        pr = {k: (v.to(device) if v is not None else None)
              for k, v in W.scan_inputs(MH.wid, B_, L_, D_, layer=i, direction="_r").items()}
        pr["x"], pr["z"] = pf["x"], pf["z"]
        h0 = W.boundary_state(MH.wid, B_, D_, std=MH.h0_std, layer=i).to(device)
        psets.append((pf, pr, h0, torch.empty((B_, L_, D_), dtype=torch.bfloat16, device=device), torch.empty_like(h0)))
    pf = psets[0][0]
    hl = torch.empty_like(psets[0][2])
    Lw = MH_PREFIX + L_
    g = torch.Generator(device=device)
    g.manual_seed(4242)
    rnd = lambda *shape, std=1.0: (torch.randn(*shape, generator=g, device=device) * std).to(torch.bfloat16)
    wf = {"x": rnd(B_, Lw, D_), "z": rnd(B_, Lw, D_), "dt": rnd(B_, Lw, D_, std=0.5), "B": rnd(B_, Lw, 16),
          "C": rnd(B_, Lw, 16), "A": pf["A"], "D": pf["D"], "dt_bias": pf["dt_bias"]}
    wr = dict(wf, dt=rnd(B_, Lw, D_, std=0.5), B=rnd(B_, Lw, 16), C=rnd(B_, Lw, 16), dt_bias=psets[0][1]["dt_bias"])
    yw = torch.empty((B_, Lw, D_), dtype=torch.bfloat16, device=device)
    fa = r2l.make_scan_args(wf["x"], wf["dt"], wf["B"], wf["C"], wf["z"], wf["A"], wf["D"], wf["dt_bias"])
    ws = torch.empty(r2l.load().r2l_bidir_scan_workspace_size(ctypes.byref(fa)), dtype=torch.uint8, device=device)

    turn = [0]

    def partial():
        pf_, pr_, h0_, y_, hl_ = psets[turn[0] % len(psets)]
        turn[0] += 1
        r2l.fwd_scan_from_state(pf_["x"], pf_["z"], pf_, pr_, h0=h0_, h_last=hl_, rev_block_len=L_, y=y_)

    def full():
        r2l.bidir_scan(wf["x"], wf["z"], wf, wr, rev_block_len=Lw, h_last=hl, y=yw, workspace=ws)

    out = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for name, fn, k in (("partial_us", partial, K), ("full_window_us", full, max(3, K // 50))):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        out[name] = 1e3 * max_over_ranks(e0.elapsed_time(e1), dist, device) / k
    if r2l.r2l_device_status() != r2l.R2L_OK:
        raise RuntimeError("device status not OK after the comparator timing")
    return {
        "workload": f"one Mamba mixer layer per denoising step: batch {B_}, d_inner {D_}, d_state 16, "
                    f"{L_}-token active block behind a {MH_PREFIX}-token prefix",
        "partial_bidirectional_us": out["partial_us"],
        "full_window_bidirectional_us": out["full_window_us"],
        "ratio": out["full_window_us"] / out["partial_us"],
        "note": "partial: forward from the cached prefix state + reverse confined to the active block (one fused "
                "launch); full window: both directions over all 1040 tokens (two scans + combine), as needed when "
                "the reverse states depend on the active tokens",
    }


# ----------------------------------------------------------------------------- --workloads

def measure_workloads(r2l, device, stream, which="all"):
    """Timings of the other workloads (parity-test configurations, not the headline): the prefill
    reverse scan, the serving sweep (14 sidecars per step, one CUDA graph per step) and the residual
    GEMM at a few shapes beside torch.matmul.  Inputs are drawn on the device with the workloads'
    distributions (timing only; the parity tests use the seeded host inputs)."""
    lib = r2l.load()
    g = torch.Generator(device=device)
    g.manual_seed(777)
    bf = torch.bfloat16

    def rnd(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=device) * std).to(bf)

    def scan_set(batch, seqlen, d, layer):
        base = W.scan_inputs(4, 1, 1, d, layer=layer)  # A, D, dt_bias from the seeded initialisers
        return {"x": rnd(batch, seqlen, d), "dt": rnd(batch, seqlen, d, std=0.5), "z": rnd(batch, seqlen, d),
                "B": rnd(batch, seqlen, 16), "C": rnd(batch, seqlen, 16), "A": base["A"].to(device),
                "D": base["D"].to(device), "dt_bias": base["dt_bias"].to(device)}

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def time_us(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return 1e3 * e0.elapsed_time(e1) / reps

    out = {}
    sh = stream.cuda_stream
    if which in ("all", "prefill"):
        wl = W.WORKLOADS["prefill_b8_L4096"]
        p = scan_set(wl.batch, wl.seqlen, wl.d_inner, 0)
        a = r2l.make_scan_args(p["x"], p["dt"], p["B"], p["C"], p["z"], p["A"], p["D"], p["dt_bias"], None, None,
                               wl.block_len)
        y = torch.empty_like(p["x"])
        us = time_us(lambda: lib.r2l_scan_block(ctypes.byref(a), y.data_ptr(), r2l.R2L_BF16, sh), 20)
        out["prefill_b8_L4096"] = {"what": "reverse scan, one 4096-token block, d_inner 2048, gate", "us": us,
                                   "tokens_per_s": wl.tokens / (us * 1e-6)}
        del p, a, y
    sweep = {}
    for batch in (W.SWEEP_BATCHES if which in ("all", "sweep") else ()):
        for block in W.SWEEP_BLOCKS:
            M = batch * block
            layers = []
            for layer in range(W.SWEEP_LAYERS):
                q = scan_set(batch, block, 2048, layer)
                q["args"] = r2l.make_scan_args(q["x"], q["dt"], q["B"], q["C"], q["z"], q["A"], q["D"], q["dt_bias"],
                                               None, None, block)
                q["y"] = torch.empty_like(q["x"])
                q["hidden"] = rnd(M, 2048)
                q["W_out"] = rnd(2048, 2048, std=2048 ** -0.5)
                layers.append(q)
            graph = torch.cuda.CUDAGraph()
            cs = torch.cuda.Stream(device)
            cs.wait_stream(stream)
            with torch.cuda.graph(graph, stream=cs, capture_error_mode="thread_local"):
                h = cs.cuda_stream
                for q in layers:
                    # one sidecar: the scan, pulling W_out and hidden into L2, then the residual
                    lib.r2l_decode_step(ctypes.byref(q["args"]), q["y"].data_ptr(), q["hidden"].data_ptr(),
                                        q["W_out"].data_ptr(), ctypes.c_float(0.05), 2048, r2l.R2L_BF16, h)
            torch.cuda.synchronize()
            us = time_us(graph.replay, 20)
            sweep[f"b{batch}_blk{block}"] = {"us_per_step": us, "tokens_per_s": M / (us * 1e-6)}
            if batch == 8:
                # the batch-8 points: several repeats on the same box, to separate run-to-run spread
                sweep[f"b{batch}_blk{block}"]["repeats_us"] = [time_us(graph.replay, 20) for _ in range(5)]
            del graph, layers
            torch.cuda.empty_cache()
    if sweep:
        out["serving_sweep_14_layers"] = sweep
    gemm = {}
    shapes = ((2048, 2048, 2048), (2048, 2048, 8192), (1024, 2048, 2048), (256, 2048, 2048), (16, 2048, 2048))
    for (M, N, K) in (shapes if which in ("all", "gemm") else ()):
        yv, Wm, hv = rnd(M, K), rnd(N, K, std=K ** -0.5), rnd(M, N)
        us = time_us(lambda: lib.r2l_residual_apply(hv.data_ptr(), yv.data_ptr(), Wm.data_ptr(), ctypes.c_float(0.05),
                                                    M, N, K, r2l.R2L_BF16, sh), 50)
        ref = time_us(lambda: torch.matmul(yv, Wm.t()), 50)
        gemm[f"{M}x{N}x{K}"] = {"us": us, "tflops": 2 * M * N * K / (us * 1e-6) / 1e12, "torch_matmul_us": ref}
    if gemm:
        out["residual_gemm"] = gemm
    if r2l.r2l_device_status() != r2l.R2L_OK:
        raise RuntimeError("device status not OK after the workload timings")
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sidecar-steps", type=int, default=2000,
                    help="steps of the whole-sidecar (hidden -> hidden) measurement; 0 skips it")
    ap.add_argument("--workloads", nargs="?", const="all", default=None, choices=["all", "prefill", "sweep", "gemm"],
                    help="time the other workloads (prefill, serving sweep, GEMM shapes; all of them by default) "
                         "instead of the headline step and print them as one JSON object")
    ap.add_argument("--bwd-steps", type=int, default=500,
                    help="launches of the scan-gradient measurement; 0 skips it")
    ap.add_argument("--comparator-steps", type=int, default=500,
                    help="steps of the partial vs full-window bidirectional comparison; 0 skips it")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))

    if args.impl == "reference":
        run_reference(args, rank, world)
        if dist is not None:
            dist.destroy_process_group()
        return

    import reverse_mamba_selective_b200 as r2l

    args.warmup = max(args.warmup, 3)
    lib = r2l.load()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    if args.workloads:
        res = measure_workloads(r2l, device, stream, args.workloads)
        if rank == 0:
            print(json.dumps({"workload_timings": res, "clock": "see nvidia-smi; not sampled in this mode"}), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return
    sh = stream.cuda_stream
    sets = [StepSet(r2l, 100 * rank + i, device) for i in range(NSETS)]
    M, D, Dm = WL.tokens, WL.d_inner, WL.d_model
    s_c = ctypes.c_float(WL.s)

    def scan(st, h=sh):
        rc = lib.r2l_scan_block(st.args_ref, st.y.data_ptr(), r2l.R2L_BF16, h)
        if rc:
            raise r2l.R2LError(rc, "r2l_scan_block")

    def resid(st, h=sh):
        rc = lib.r2l_residual_apply(st.dev["hidden"].data_ptr(), st.y.data_ptr(), st.dev["W_out"].data_ptr(), s_c,
                                    M, Dm, D, r2l.R2L_BF16, h)
        if rc:
            raise r2l.R2LError(rc, "r2l_residual_apply")

    def step(st, h=sh):
        """One decode step through the one-call entry point (the scan pulls the residual's W_out and
        hidden into L2 while it runs)."""
        rc = lib.r2l_decode_step(st.args_ref, st.y.data_ptr(), st.dev["hidden"].data_ptr(), st.dev["W_out"].data_ptr(),
                                 s_c, Dm, r2l.R2L_BF16, h)
        if rc:
            raise r2l.R2LError(rc, "r2l_decode_step")

    def capture_steps(first, count, launch=None):
        """One CUDA graph of `count` decode steps (or launches of `launch`) on the rotating sets,
        starting at step `first`."""
        launch = launch or step
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(device)
        cs.wait_stream(stream)
        with torch.cuda.graph(g, stream=cs, capture_error_mode="thread_local"):
            for i in range(first, first + count):
                launch(sets[i % NSETS], cs.cuda_stream)
        torch.cuda.synchronize()
        return g

    # the clock sampler starts first: its start-up sleep must not leave the GPU idle (and clocking
    # down) between the warm-up steps and the timed region
    clocks = ClockSampler(local)
    time.sleep(0.25)
    for i in range(args.warmup):
        step(sets[i % NSETS])
    torch.cuda.synchronize()
    if r2l.r2l_device_status() != r2l.R2L_OK:
        raise RuntimeError("device status not OK after warm-up")

    K = args.steps
    # the K timed steps are replayed from CUDA graphs captured here, before the timed region: the
    # same two kernels per step on the same rotating inputs, without host launch work between
    # steps.  Chunks of GRAPH_STEPS steps (a multiple of NSETS, so every chunk starts on set 0) and
    # one graph for the remainder make exactly K steps.
    chunk = min(K, GRAPH_STEPS)
    n_full, rem = divmod(K, chunk)
    g_main = capture_steps(0, chunk)
    g_rem = capture_steps(n_full * chunk, rem) if rem else None
    g_main.replay()  # the first replay uploads the graph; untimed
    if g_rem is not None:
        g_rem.replay()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # timed region: K steps, events only at its ends (events between kernels would add their own
    # cost and break the overlap of each kernel's launch with its predecessor's tail)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(n_full):
        g_main.replay()
    if g_rem is not None:
        g_rem.replay()
    stop.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    elapsed_ms = start.elapsed_time(stop)
    del g_main, g_rem
    # per-kernel durations: each kernel alone, K launches on the same rotating sets replayed from
    # CUDA graphs the same way, events at the ends: its average launch duration in a stream of its
    # own launches (events around every launch would break each launch's overlap with its
    # predecessor's tail and add their own cost)
    def kernel_ms(launch):
        gm = capture_steps(0, chunk, launch)
        gr = capture_steps(n_full * chunk, rem, launch) if rem else None
        gm.replay()
        if gr is not None:
            gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_full):
            gm.replay()
        if gr is not None:
            gr.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    scan_ms, res_ms = kernel_ms(scan), kernel_ms(resid)
    clk = clocks.stop()
    if r2l.r2l_device_status() != r2l.R2L_OK:
        raise RuntimeError("device status not OK after the timed region")

    elapsed_ms = max_over_ranks(elapsed_ms, dist, device)

    # ---- end to end: pinned host inputs copied in and the result copied out every step, inside
    # the timed region.  Two device sets alternate so that the copies of one step overlap the
    # compute and the opposite-direction copy of its neighbours (PCIe is full duplex).
    Ke = max(1, min(args.e2e_steps, K))
    in_keys = ("x", "dt", "B", "C", "z", "hidden")
    ring = [sets[0], sets[1]]
    pinned = [{k: st.host[k].pin_memory() for k in in_keys} for st in ring]
    outs = [torch.empty_like(ring[0].host["hidden"]).pin_memory() for _ in ring]
    h2d = sum(pinned[0][k].numel() * pinned[0][k].element_size() for k in in_keys)
    d2h = outs[0].numel() * outs[0].element_size()
    copy_in = torch.cuda.Stream(device)
    copied = [torch.cuda.Event() for _ in ring]
    computed = [torch.cuda.Event() for _ in ring]

    def e2e_step(i):
        j = i % 2
        st = ring[j]
        with torch.cuda.stream(copy_in):
            copy_in.wait_event(computed[j])  # the previous use of this set has been read back
            for k in in_keys:
                st.dev[k].copy_(pinned[j][k], non_blocking=True)
            copied[j].record(copy_in)
        stream.wait_event(copied[j])
        step(st)
        outs[j].copy_(st.dev["hidden"], non_blocking=True)
        computed[j].record(stream)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_in.wait_stream(stream)
    for i in range(Ke):
        e2e_step(i)
    stream.wait_stream(copy_in)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dist, device)
    if dist is not None:
        dist.barrier()

    # ---- gradient of the reverse block scan
    scan_bwd = measure_scan_bwd(r2l, device, stream, args.bwd_steps, dist) if args.bwd_steps > 0 else None

    # ---- partial vs full-window bidirectional Mamba mixer
    comparators = None
    if args.comparator_steps > 0:
        comparators = measure_comparators(r2l, device, stream, args.comparator_steps, dist)

    # ---- the whole sidecar, hidden -> hidden (front-end projections included)
    sidecar = None
    if args.sidecar_steps > 0:
        Ksc = args.sidecar_steps
        sc_ms, sc_graph_ms, sc_stage_us = measure_sidecar(r2l, lib, device, stream, Ksc, args.warmup, dist, rank)
        fl = sidecar_flops()
        peak_tc = measured_peaks()["bf16_tflops_sustained"]
        in_tf = fl["in_proj"] / (sc_stage_us["in_proj"] * 1e-6) / 1e12
        sidecar = {
            "workload": f"{WL.name}, whole sidecar hidden -> hidden (dt_rank {DT_RANK})",
            "steps": Ksc, "ms_per_step": sc_ms, "tokens_per_s": WL.tokens * world / (sc_ms * 1e-3),
            "ms_per_step_graph": sc_graph_ms, "tokens_per_s_graph": WL.tokens * world / (sc_graph_ms * 1e-3),
            "launches_per_step": 6,
            "stage_us": sc_stage_us,
            "stage_timing": "each stage alone through its own entry point, replayed from a CUDA graph over the same "
                            "rotating sets (the whole-sidecar call fuses x_proj's products into in_proj, so its time "
                            "is below the sum of these)",
            "flops_per_step": sum(fl.values()),
            "in_proj": {"bound": "tensor", "achieved": in_tf, "peak": peak_tc, "unit": "TFLOP/s",
                        "frac": in_tf / peak_tc, "peak_source": "bf16_tflops_sustained (measured)",
                        "traffic": profiled_traffic("in_proj", FE_KERNEL_SRC)},
            "l2": f"{NSETS} rotating sets of weights, hidden and workspace (~{NSETS * 117:.0f} MiB)",
        }

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    peaks = measured_peaks()
    tokens_all = WL.tokens * world * K
    ms_per_step = elapsed_ms / K
    scan_us = 1e3 * scan_ms
    res_us = 1e3 * res_ms
    sb, rb, rf = scan_bytes_per_step(), residual_bytes_per_step(), residual_flops_per_step()
    scan_gbs = sb / (scan_us * 1e-6) / 1e9
    res_tflops = rf / (res_us * 1e-6) / 1e12
    kernels = {
        "scan": {"us_per_launch": scan_us, "algorithmic_bytes": sb, "achieved_gbs": scan_gbs,
                 "frac_of_hbm": scan_gbs / peaks["hbm_gbs"], "tokens_per_s": WL.tokens / (scan_us * 1e-6),
                 "dram_bytes_ncu": profiled_traffic("scan", SCAN_KERNEL_SRC)},
        "residual": {"us_per_launch": res_us, "algorithmic_bytes": rb, "flops": rf, "achieved_tflops": res_tflops,
                     "frac_of_bf16_sustained": res_tflops / peaks["bf16_tflops_sustained"],
                     "dram_bytes_ncu": profiled_traffic("residual", GEMM_KERNEL_SRC)},
    }
    # The scan is bound by special-function (MUFU) throughput and instruction issue, not by HBM:
    # its roofline is the MUFU peak of 148 SMs x 16 results/clk at the maximum SM clock.
    sm_mhz = peaks.get("sm_max_mhz") or 1965.0
    mufu_peak = B200_SMS * MUFU_PER_CLK_PER_SM * sm_mhz * 1e6 / 1e12  # Top/s
    mufu_achieved = scan_mufu_ops_per_step() / (scan_us * 1e-6) / 1e12
    kernels["scan"]["mufu_tops"] = mufu_achieved
    kernels["scan"]["frac_of_mufu_peak"] = mufu_achieved / mufu_peak
    if scan_us >= res_us:
        roof = {"kernel": "scan", "bound": "alu", "achieved": mufu_achieved, "peak": mufu_peak,
                "unit": "Top/s (MUFU transcendental results)", "frac": mufu_achieved / mufu_peak,
                "traffic": kernels["scan"]["dram_bytes_ncu"],
                "traffic_note": "ncu DRAM bytes of r2l_scan_block's scan (as timed here); as r2l_decode_step "
                                "launches it, it also pulls the residual's W_out and hidden (16.8 MB) into L2",
                "peak_source": f"derived: {B200_SMS} SMs x {MUFU_PER_CLK_PER_SM} MUFU results/clk x {sm_mhz:.0f} MHz",
                "work": f"{SCAN_MUFU_PER_ELEMENT} MUFU ops per (token, channel)",
                "hbm": {"achieved": scan_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": scan_gbs / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} hbm_gbs",
                        "algorithmic_bytes": sb}}
    else:
        roof = {"kernel": "residual", "bound": "tensor", "achieved": res_tflops, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": res_tflops / peaks["bf16_tflops_sustained"],
                "traffic": kernels["residual"]["dram_bytes_ncu"],
                "peak_source": f"{peaks['source']} bf16_tflops_sustained"}

    line = {
        "metric": METRIC,
        "value": tokens_all / (elapsed_ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; Qwen3-1.7B-sized activations, Mamba-1 initialisation)",
        "config": {"workload": WL.name, "batch_per_gpu": WL.batch, "global_batch": WL.batch * world,
                   "block_len": WL.block_len, "seq_len": WL.seqlen, "d_inner": D, "d_state": WL.d_state,
                   "d_model": Dm, "conv_width": WL.conv_width, "s": WL.s, "io_dtype": "bf16",
                   "state_dtype": "f32", "gemm": "bf16 tcgen05, f32 accumulate",
                   "parallelism": f"dp{world} (independent batches, no collective)",
                   "l2": f"{NSETS} rotating input sets (~{NSETS * 48.5:.0f} MiB > 2x 126 MB L2)"},
        "hbm_gbs_step": (sb + rb) / (ms_per_step * 1e-3) / 1e9,
        "roofline": roof,
        "kernels": kernels,
        "timing": "K steps (one r2l_decode_step call each: scan + residual) replayed from CUDA graphs "
                  f"captured before the timed region (chunks of {GRAPH_STEPS} steps + remainder), CUDA events "
                  "on the launching stream at its ends",
        "kernel_timing": "per-kernel durations: each kernel alone, K launches (r2l_scan_block, then "
                         "r2l_residual_apply on the scan's outputs; no L2 prefetch) on the same rotating sets, "
                         "replayed from CUDA graphs with CUDA events at the ends: elapsed / K",
        "gpu_launches": 2 * K,
        "clocks": clk,
        "e2e": {"value": WL.tokens * world * Ke / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke,
                "note": "pinned host inputs (x, dt, z, B, C, hidden) copied in and hidden copied out every step "
                        "through r2l_decode_step; two device sets alternate so copies overlap compute; weights "
                        "resident"},
    }
    if sidecar is not None:
        line["sidecar_step"] = sidecar
    if comparators is not None:
        line["bidirectional_comparators"] = comparators
    if scan_bwd is not None:
        line["scan_backward"] = scan_bwd
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
