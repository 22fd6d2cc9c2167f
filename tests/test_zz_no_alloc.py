"""r2l_x_proj_noalloc (partial sums in the library's own device scratch) against r2l_x_proj (partial
sums in a caller workspace): the same kernels in the same order, so the results must agree bit for
bit, on two calls in a row (the second reuses the scratch the first one wrote)."""

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def r2l():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import reverse_mamba_selective_b200 as pkg

    pkg.load()
    return pkg


@pytest.mark.parametrize("M,d_inner,dt_rank", [(2048, 2048, 128), (144, 192, 16), (300, 520, 64)])
def test_noalloc_matches_workspace_entry_point(r2l, M, d_inner, dt_rank):
    w = W.sidecar_weights(70, 64, d_inner, dt_rank=dt_rank)
    u1 = W.normal(70, 0, "u_probe", (M, d_inner), std=0.35).cuda()
    u2 = W.normal(70, 1, "u_probe", (M, d_inner), std=0.35).cuda()
    wx = w["W_x"].cuda()
    for u in (u1, u2):  # two calls in a row on different inputs
        ref = r2l.r2l_x_proj(u, wx, dt_rank)
        got = r2l.r2l_x_proj_noalloc(u, wx, dt_rank)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    assert r2l.r2l_device_status() == r2l.R2L_OK
