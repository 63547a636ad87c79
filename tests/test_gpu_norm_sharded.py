"""GPU parity of the hidden-sharded LayerNorm / RMSNorm (statistics from the
shards' local sums reduced over shards) against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import TOL_BF16, TOL_F32, assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["rms", "layer"])
@pytest.mark.parametrize("p,h", [(1, 512), (2, 512), (3, 1152), (4, 4096), (8, 8192), (8, 128), (8, 16384)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_norm_sharded_fwd_bwd(kind, p, h, dtype):
    """1500 rows: more than the backward's CTAs at every width, so each CTA
    carries its parameter-gradient partials over several rows."""
    from megatron_tensor_transformer_gemm_b200 import tp
    if dtype == "f32" and h > 8192:
        pytest.skip("fp32 rows are limited to 8192 columns")
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    rows = 1500
    g = torch.Generator().manual_seed(h + p)
    x = (torch.randn(rows, h, generator=g) * 1.5 + 0.2).to(tdt)
    gamma = (1 + 0.1 * torch.randn(h, generator=g)).to(tdt)
    beta = (0.1 * torch.randn(h, generator=g)).to(tdt)
    dy = torch.randn(rows, h, generator=g).to(tdt)
    hs = h // p
    sl = lambda t, i: t[..., i * hs:(i + 1) * hs].contiguous()
    xs = [dev(sl(x, i)) for i in range(p)]
    gs = [dev(sl(gamma, i)) for i in range(p)]
    bs = [dev(sl(beta, i)) for i in range(p)]
    dys = [dev(sl(dy, i)) for i in range(p)]
    ys = [torch.empty(rows, hs, dtype=tdt, device="cuda") for _ in range(p)]
    mean = torch.empty(rows, dtype=torch.float32, device="cuda")
    rstd = torch.empty(rows, dtype=torch.float32, device="cuda")
    plan = tp.Plan(h, 0, 0, p, dtype, "none")
    plan.norm_sharded_fwd(kind, rows, xs, gs, bs if kind == "layer" else None, ys, mean, rstd)
    okind = "rms" if kind == "rms" else "ln"
    X64 = [O.f64(sl(x, i)) for i in range(p)]
    G64 = [O.f64(sl(gamma, i)) for i in range(p)]
    B64 = [O.f64(sl(beta, i)) for i in range(p)]
    DY64 = [O.f64(sl(dy, i)) for i in range(p)]
    ref, stats = O.norm_sharded_fwd(X64, G64, B64, okind)
    assert_close(torch.cat(ys, 1), np.concatenate(ref, 1), tol, "Y")
    np.testing.assert_allclose(host(rstd), stats[1], rtol=1e-4)
    dxs = [torch.empty_like(a) for a in ys]
    dgs = [torch.empty(hs, dtype=torch.float32, device="cuda") for _ in range(p)]
    dbs = [torch.empty(hs, dtype=torch.float32, device="cuda") for _ in range(p)] if kind == "layer" else None
    plan.norm_sharded_bwd(kind, rows, xs, gs, dys, mean if kind == "layer" else None, rstd, dxs, dgs, dbs)
    rdx, rdg, rdb = O.norm_sharded_bwd(X64, G64, DY64, stats, okind)
    assert_close(torch.cat(dxs, 1), np.concatenate(rdx, 1), tol, "dX")
    assert_close(torch.cat(dgs)[None, :], np.concatenate(rdg)[None, :], max(tol, 1e-3), "dgamma")
    if kind == "layer":
        assert_close(torch.cat(dbs)[None, :], np.concatenate(rdb)[None, :], max(tol, 1e-3), "dbeta")
