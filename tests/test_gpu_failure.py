"""Failure detection on the GPU without a fault: a bounded device-side wait that runs out.

r2l_wait_selftest enqueues one CTA waiting on an mbarrier that nothing arrives at; the wait gives up
after its bound (2 s), sets the library's device status word and returns.  The host then reads
R2L_ERR_TIMEOUT once, the word is cleared, and the context still runs a scan correctly.
"""

import pytest
import torch

import oracle
import workloads as W
from conftest import rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def r2l():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import reverse_mamba_selective_b200 as pkg

    pkg.load()
    oracle.build()
    return pkg


def test_bounded_wait_reports_timeout_and_context_survives(r2l):
    assert r2l.r2l_device_status() == r2l.R2L_OK
    r2l.r2l_wait_selftest()
    assert r2l.r2l_device_status() == r2l.R2L_ERR_TIMEOUT
    assert r2l.r2l_device_status() == r2l.R2L_OK  # read once, then cleared
    p = W.scan_inputs(0, 1, 64, 64, io="f32")
    g = {k: (v.cuda() if v is not None else None) for k, v in p.items()}
    y = r2l.r2l_scan_block(g["x"], g["dt"], g["B"], g["C"], g["z"], g["A"], g["D"], g["dt_bias"], None, None,
                           block_len=64, y_dtype=torch.float32)
    torch.cuda.synchronize()
    o = {k: (W.as_f64(v) if v is not None else None) for k, v in p.items()}
    ref = oracle.scan(o["x"], o["dt"], o["B"], o["C"], o["z"], o["A"], o["D"], o["dt_bias"], reverse=True, block_len=64)
    assert rel_err(y.cpu().numpy(), ref) < 1e-5
    assert r2l.r2l_device_status() == r2l.R2L_OK
