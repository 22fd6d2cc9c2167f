"""Seeded synthetic inputs for the right-to-left selective-scan sidecar.

This module is shared by the oracle tests, the GPU parity tests, the smoke
check and the benchmark.  It holds shapes, seeds and value distributions only:
none of the scan's arithmetic lives here.  Every tensor is drawn once on the
host from its own counter-free PCG64 stream keyed by (workload id, layer,
tensor id), rounded to its storage dtype, and the same bytes are handed to the
GPU library and to the fp64 oracle.

Value recipe (the pages print no numbers for the scan itself, so the recipe is
the standard Mamba-1 initialisation on activations shaped like a Qwen3-1.7B
backbone, batched parallel decoding over short generation blocks):

* x, B, C, z, hidden ~ N(0, 1); dt ~ 0.5 * N(0, 1)
* dt_bias = inverse-softplus of dt_init, dt_init log-uniform on [1e-3, 1e-1]
* A = -exp(A_log) with A_log[d, n] = log(n + 1)            (fp32)
* D = 1                                                     (fp32)
* conv_w, conv_b ~ U(-1/2, 1/2)  (= +-1/sqrt(width) for width 4)
* W_out ~ N(0, 1) / sqrt(d_inner)
* h0 (cached forward boundary state) ~ N(0, 0.1^2)          (fp32)
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import numpy as np
import torch

# Tensor ids inside one (workload, layer) key.
TID = {
    "x": 1, "dt": 2, "B": 3, "C": 4, "z": 5, "dt_bias": 6, "conv_w": 7,
    "conv_b": 8, "hidden": 9, "W_out": 10, "h0": 11,
    # second (reverse) direction of the partial-bidirectional mixer
    "dt_r": 12, "B_r": 13, "C_r": 14, "dt_bias_r": 15,
    # cached convolution inputs of a resumed forward scan
    "conv_state": 16,
    # sidecar front-end weights
    "W_in": 17, "W_x": 18, "W_dt": 19, "u_probe": 20, "dt_low_probe": 21,
}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One workload shape.  ``io`` is the storage dtype of x/dt/z/B/C/y/hidden/W_out."""

    wid: int
    name: str
    batch: int
    seqlen: int
    block_len: int
    d_inner: int
    d_state: int = 16
    d_model: int = 0          # 0: no residual step in this workload
    conv_width: int = 0
    io: str = "bf16"
    s: float = 0.05
    h0_std: float = 0.0       # > 0: forward scan resumed from a cached state
    layers: int = 1

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


WORKLOADS: Dict[str, Workload] = {
    # Tiny oracle case: reverse scan only, fp32, s in {0, 0.05} through a 64x64 out-projection.
    "tiny_f32": Workload(0, "reverse scan b1 L64 d_inner64 d_state16 f32", 1, 64, 64, 64,
                         d_model=64, io="f32", s=0.05),
    # R2LM parallel-decode sidecar step (the headline workload).
    "decode_b64_blk32": Workload(1, "R2LM parallel-decode sidecar step b64 block32 d_model2048 "
                                    "d_inner2048 d_state16 conv4 s0.05",
                                 64, 32, 32, 2048, d_model=2048, conv_width=4, s=0.05),
    # Prompt prefill: one right-to-left scan over the whole 4096-token prompt.
    "prefill_b8_L4096": Workload(2, "prompt prefill reverse scan b8 L4096 d_inner2048 d_state16",
                                 8, 4096, 4096, 2048),
    # Partial bidirectionality: forward from cached h0 + block-confined reverse.
    "mamba_h_b32_blk16": Workload(3, "forward-from-state + block reverse b32 block16 d_inner4096",
                                  32, 16, 16, 4096, h0_std=0.1),
}

# Batch-serving sweep: 14 independent sidecars (every 2nd of 28 layers) per denoising step.
SWEEP_BATCHES = (1, 8, 32, 64, 128, 256)
SWEEP_BLOCKS = (16, 32, 64)
SWEEP_LAYERS = 14


def sweep_workload(batch: int, block: int) -> Workload:
    return Workload(4, f"serving sweep b{batch} block{block} d_inner2048 x14 layers",
                    batch, block, block, 2048, d_model=2048, conv_width=0, s=0.05,
                    layers=SWEEP_LAYERS)


def rng_for(wid: int, layer: int, tensor: str) -> np.random.Generator:
    """Independent PCG64 stream per (workload, layer, tensor)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(wid), int(layer), TID[tensor]])))


def _store(a64: np.ndarray, io: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a64, dtype=np.float32))
    if io == "bf16":
        return t.to(torch.bfloat16)  # round-to-nearest-even
    if io == "f32":
        return t
    raise ValueError(io)


def normal(wid, layer, tensor, shape, std=1.0, io="bf16") -> torch.Tensor:
    g = rng_for(wid, layer, tensor)
    return _store(g.standard_normal(size=shape) * std, io)


def uniform(wid, layer, tensor, shape, lo, hi, io="f32") -> torch.Tensor:
    g = rng_for(wid, layer, tensor)
    return _store(g.uniform(lo, hi, size=shape), io)


def dt_bias_init(wid, layer, d_inner, tensor="dt_bias") -> torch.Tensor:
    """Inverse-softplus of a log-uniform dt_init on [1e-3, 1e-1] (fp64, then fp32)."""
    g = rng_for(wid, layer, tensor)
    dt_init = np.exp(g.uniform(math.log(1e-3), math.log(1e-1), size=(d_inner,)))
    return _store(dt_init + np.log(-np.expm1(-dt_init)), "f32")


def a_init(d_inner: int, d_state: int) -> torch.Tensor:
    """A = -exp(A_log) with A_log[d, n] = log(n + 1), evaluated in fp64 and stored fp32."""
    a_log = np.log(np.arange(1, d_state + 1, dtype=np.float64))[None, :].repeat(d_inner, 0)
    return _store(-np.exp(a_log), "f32")


def scan_inputs(wid: int, batch: int, seqlen: int, d_inner: int, d_state: int = 16,
                conv_width: int = 0, io: str = "bf16", layer: int = 0, gate: bool = True,
                direction: str = "") -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of one selective scan as CPU tensors.

    ``direction='_r'`` draws the reverse direction's own dt/B/C/dt_bias (x, z shared).
    """
    sfx = direction
    out: Dict[str, Optional[torch.Tensor]] = {
        "x": normal(wid, layer, "x", (batch, seqlen, d_inner), io=io),
        "dt": normal(wid, layer, "dt" + sfx, (batch, seqlen, d_inner), std=0.5, io=io),
        "B": normal(wid, layer, "B" + sfx, (batch, seqlen, d_state), io=io),
        "C": normal(wid, layer, "C" + sfx, (batch, seqlen, d_state), io=io),
        "z": normal(wid, layer, "z", (batch, seqlen, d_inner), io=io) if gate else None,
        "A": a_init(d_inner, d_state),
        "D": torch.ones(d_inner, dtype=torch.float32),
        "dt_bias": dt_bias_init(wid, layer, d_inner, "dt_bias" + sfx),
        "conv_w": None,
        "conv_b": None,
    }
    if conv_width:
        out["conv_w"] = uniform(wid, layer, "conv_w", (d_inner, conv_width), -0.5, 0.5)
        out["conv_b"] = uniform(wid, layer, "conv_b", (d_inner,), -0.5, 0.5)
    return out


def residual_inputs(wid: int, M: int, d_model: int, d_inner: int, io: str = "bf16",
                    layer: int = 0) -> Dict[str, torch.Tensor]:
    return {
        "hidden": normal(wid, layer, "hidden", (M, d_model), io=io),
        "W_out": normal(wid, layer, "W_out", (d_model, d_inner), std=1.0 / math.sqrt(d_inner), io=io),
    }


def sidecar_weights(wid: int, d_model: int, d_inner: int, d_state: int = 16, dt_rank: Optional[int] = None,
                    conv_width: int = 4, layer: int = 0) -> Dict[str, Optional[torch.Tensor]]:
    """Random-init weights of one sidecar (standard Mamba-1 block shapes, bf16 matrices).

    Scales: W_in ~ N(0, 1/d_model) so that x, z ~ N(0, 1) for hidden ~ N(0, 1); W_x's dt rows
    ~ N(0, 1/d_inner) and its B, C rows ~ N(0, 8/d_inner) (u = SiLU of the convolution has an rms
    near 0.35, so B, C come out near unit scale); W_dt ~ N(0, 2/dt_rank) so that dt has a standard
    deviation near 0.5,
    as in the scan-only workloads.  A, D, dt_bias, conv_w, conv_b as in scan_inputs.
    """
    dt_rank = dt_rank or -(-d_model // 16)
    wx = normal(wid, layer, "W_x", (dt_rank + 2 * d_state, d_inner), std=1.0 / math.sqrt(d_inner), io="f32")
    wx[dt_rank:] *= math.sqrt(8.0)
    out: Dict[str, Optional[torch.Tensor]] = {
        "W_in": normal(wid, layer, "W_in", (2 * d_inner, d_model), std=1.0 / math.sqrt(d_model)),
        "conv_w": None,
        "conv_b": None,
        "W_x": wx.to(torch.bfloat16),
        "W_dt": normal(wid, layer, "W_dt", (d_inner, dt_rank), std=math.sqrt(2.0 / dt_rank)),
        "A": a_init(d_inner, d_state),
        "D": torch.ones(d_inner, dtype=torch.float32),
        "dt_bias": dt_bias_init(wid, layer, d_inner),
        "W_out": normal(wid, layer, "W_out", (d_model, d_inner), std=1.0 / math.sqrt(d_inner)),
    }
    if conv_width:
        out["conv_w"] = uniform(wid, layer, "conv_w", (d_inner, conv_width), -0.5, 0.5)
        out["conv_b"] = uniform(wid, layer, "conv_b", (d_inner,), -0.5, 0.5)
    return out


def boundary_state(wid: int, batch: int, d_inner: int, d_state: int = 16, std: float = 0.1,
                   layer: int = 0) -> torch.Tensor:
    return normal(wid, layer, "h0", (batch, d_inner, d_state), std=std, io="f32")


def conv_state(wid: int, batch: int, d_inner: int, conv_width: int = 4, layer: int = 0) -> torch.Tensor:
    """Cached convolution inputs [batch, d_inner, conv_width - 1] of a resumed forward scan.
    They are earlier x values, so they are drawn like x (bf16-exact) and held in fp32."""
    return normal(wid, layer, "conv_state", (batch, d_inner, conv_width - 1), io="bf16").float()


def as_f64(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """Exact widening of a stored tensor (bf16 -> fp32 -> fp64 is exact)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def shard_rows(total: int, world: int, rank: int) -> Sequence[int]:
    """Contiguous batch-row range owned by ``rank`` when independent rows are split over ``world`` ranks."""
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))
