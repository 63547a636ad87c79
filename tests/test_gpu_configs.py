"""Parity at the workloads' full sizes, in the launch configuration bench.py
times: every output is produced by the GPU in full; the oracle checks a fixed,
seeded sample of token rows (row-local outputs) and of intermediate units
(weight-gradient columns), each computed exactly from its definition."""
import numpy as np
import pytest
import torch

import oracle as O
import tp_synth
from gpu_helpers import TOL_BF16, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _rows(T, n):
    return tp_synth.sample_rows(T, n).numpy()


def _check_mlp_7b_sampled(m, inp, T, h, f, p, Y, dX):
    """Sampled rows of Y and dX and sampled units of dW1 and dW2 against the
    oracle (each sample computed exactly from its definition)."""
    rows = _rows(T, 48)
    fcols = np.sort(tp_synth.sample_rows(f, 12, seed=99).numpy())
    X, W1, W2, dY = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    ref = O.mlp_fwd_rows(X, W1, None, W2, None, "swiglu", rows)
    assert_close(host(Y)[rows], ref["Y"], TOL_BF16, "Y rows")
    smp = O.mlp_bwd_sampled(X, W1, None, W2, dY, "swiglu", rows, fcols)
    assert_close(host(dX)[rows], smp["dX_rows"], TOL_BF16, "dX rows")
    # weight gradients: gather the sampled units from the shards
    fp = f // p
    dW1 = [host(w) for w in m.dW1]
    dW2 = [host(w) for w in m.dW2]
    got_w1 = []
    for half in (0, 1):
        for j in fcols:
            i, jj = divmod(int(j), fp)
            got_w1.append(dW1[i][half * fp + jj])
    assert_close(np.array(got_w1), smp["dW1_rows"], TOL_BF16, "dW1 sampled rows")
    got_w2 = np.stack([dW2[int(j) // fp][:, int(j) % fp] for j in fcols], axis=1)
    assert_close(got_w2.T, smp["dW2_cols"].T, TOL_BF16, "dW2 sampled columns")
    from megatron_tensor_transformer_gemm_b200 import tp
    assert tp.device_status() == "TP_OK"


@pytest.mark.parametrize("fused", [False, True], ids=["partials", "fused"])
def test_mlp_7b_swiglu_full_size_sampled(fused):
    """hidden 4096, ffn 11008, tokens 32768, p 8; fused: the shard sums run
    inside the row GEMM and the column-backward dX GEMM (the launch
    configuration bench.py times by default)."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    T, h, f, p = 32768, 4096, 11008, 8
    inp = tp_synth.draw_mlp(T, h, f, "swiglu", torch.bfloat16, seed=0)
    m = TPMLP(h, f, p, "swiglu", "bf16", fused=fused)
    m.load_weights(dev(inp.W1), dev(inp.W2))
    Y = m.forward(dev(inp.X))
    dX = m.backward(dev(inp.dY))
    _check_mlp_7b_sampled(m, inp, T, h, f, p, Y, dX)


def _run_sp(seq, h, f, p, ln_random, seed=0):
    from megatron_tensor_transformer_gemm_b200.block import SPMLP
    X, g, b, W1, W2, dY = tp_synth.draw_sp_mlp(seq, h, f, p, torch.bfloat16, seed=seed,
                                               ln_affine_random=ln_random)
    sp = SPMLP(h, f, p, "swiglu")
    sp.mlp.load_weights(dev(W1), dev(W2))
    sp.gamma.copy_(dev(g))
    sp.beta.copy_(dev(b))
    t = seq // p
    Ys = sp.forward([dev(X[j * t:(j + 1) * t]) for j in range(p)])
    dXs = sp.backward([dev(dY[j * t:(j + 1) * t]) for j in range(p)])
    return sp, (X, g, b, W1, W2, dY), torch.cat(Ys, 0), torch.cat(dXs, 0)


def test_sp_mlp_reduced_size_full_check():
    """LN on sequence shards -> AG -> column -> row -> RS, and the backward, at a
    reduced size (seq 512, hidden 1024, ffn 3584, p 8) checked in full."""
    sp, (X, g, b, W1, W2, dY), Y, dX = _run_sp(512, 1024, 3584, 8, True, seed=3)
    X, g, b, W1, W2, dY = (O.f64(t) for t in (X, g, b, W1, W2, dY))
    ref = O.sp_mlp_fwd(X, g, b, W1, W2)
    rb = O.sp_mlp_bwd(X, g, W1, W2, ref, dY)
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, rb["dX"], TOL_BF16, "dX")
    assert_close(sp.dgamma[None, :], rb["dg"][None, :], TOL_BF16, "dgamma")
    assert_close(sp.dbeta[None, :], rb["db"][None, :], TOL_BF16, "dbeta")


def test_sp_mlp_full_size_sampled():
    """hidden 8192, ffn 28672, seq 8192, batch 1, p 8: sampled rows of Y and dX."""
    seq, h, f, p = 8192, 8192, 28672, 8
    sp, (X, g, b, W1, W2, dY), Y, dX = _run_sp(seq, h, f, p, False)
    rows = _rows(seq, 24)
    Xr = O.f64(X[rows])
    g64, b64, W1f, W2f = O.f64(g), O.f64(b), O.f64(W1), O.f64(W2)
    ref = O.sp_mlp_fwd(Xr, g64, b64, W1f, W2f)
    assert_close(host(Y)[rows], ref["Y"], TOL_BF16, "Y rows")
    rb = O.sp_mlp_bwd(Xr, g64, W1f, W2f, ref, O.f64(dY[rows]))
    assert_close(host(dX)[rows], rb["dX"], TOL_BF16, "dX rows")


def test_sp_mlp_reduced_size_fused():
    from megatron_tensor_transformer_gemm_b200.block import SPMLP
    seq, h, f, p = 512, 1024, 3584, 8
    X, g, b, W1, W2, dY = tp_synth.draw_sp_mlp(seq, h, f, p, torch.bfloat16, seed=4, ln_affine_random=True)
    sp = SPMLP(h, f, p, "swiglu", fused=True)
    sp.mlp.load_weights(dev(W1), dev(W2))
    sp.gamma.copy_(dev(g))
    sp.beta.copy_(dev(b))
    t = seq // p
    Y = torch.cat(sp.forward([dev(X[j * t:(j + 1) * t]) for j in range(p)]), 0)
    dX = torch.cat(sp.backward([dev(dY[j * t:(j + 1) * t]) for j in range(p)]), 0)
    X, g, b, W1, W2, dY = (O.f64(x) for x in (X, g, b, W1, W2, dY))
    ref = O.sp_mlp_fwd(X, g, b, W1, W2)
    rb = O.sp_mlp_bwd(X, g, W1, W2, ref, dY)
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, rb["dX"], TOL_BF16, "dX")
    assert_close(sp.dgamma[None, :], rb["dg"][None, :], TOL_BF16, "dgamma")
