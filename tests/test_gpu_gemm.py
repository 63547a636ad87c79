"""GPU parity of the tensor-core GEMM paths against the oracle's sharded steps.

Shapes span several 128x256 tiles and end in ragged tails in M (tokens), N
(output features) and K (reduction), including a final K block that is
partly out of bounds."""
import os

import numpy as np
import pytest
import torch

import oracle as O
import tp_synth
from gpu_helpers import TOL_BF16, TOL_F32, assert_close, dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _tp():
    from megatron_tensor_transformer_gemm_b200 import tp
    return tp


def _empty(*shape, dtype=torch.bfloat16):
    return torch.empty(*shape, dtype=dtype, device="cuda")


def _shard_w1(W1, act, p, i):
    return O.shard_gate_up(W1, p, i) if act == "swiglu" else O.shard_rows(W1, p, i)


CASES = [
    # (T, h, f, p, act, bias)
    (300, 192, 528, 2, "gelu", True),     # M tail 44, N = 264 (tail 8), K = 3 blocks
    (300, 200, 528, 2, "gelu", False),    # K = 200: last K block 8 wide
    (257, 256, 272, 2, "swiglu", False),  # 136 gate/up pairs: 128 + 8
    (129, 128, 1024, 4, "swiglu", False),
    (513, 136, 512, 1, "none", True),
]


@pytest.mark.parametrize("T,h,f,p,act,bias", CASES)
def test_column_forward(T, h, f, p, act, bias):
    tp = _tp()
    inp = tp_synth.draw_mlp(T, h, f, act, torch.bfloat16, seed=T + h, bias=bias, dy=False)
    plan = tp.Plan(h, f, 0, p, "bf16", act)
    n1 = (2 if act == "swiglu" else 1) * f // p
    W1s = [_empty(n1, h) for _ in range(p)]
    plan.shard_column("mlp", dev(inp.W1), W1s)
    b1s = None
    if bias:
        b1s = [_empty(n1) for _ in range(p)]
        plan.shard_column_bias("mlp", dev(inp.b1), b1s)
    Z = [_empty(T, n1) for _ in range(p)] if act != "none" else None
    H = [_empty(T, f // p) for _ in range(p)]
    plan.column_fwd("mlp", T, dev(inp.X), W1s, b1s, Z, H)
    X, W1 = O.f64(inp.X), O.f64(inp.W1)
    for i in range(p):
        bi = O.shard_vec(O.f64(inp.b1), p, i) if bias else None
        rz, rh = O.column_fwd_shard(X, _shard_w1(W1, act, p, i), bi, act)
        if Z is not None:
            assert_close(Z[i], rz, TOL_BF16, f"Z[{i}]")
        assert_close(H[i], rh, TOL_BF16, f"H[{i}]")
    # Z may be omitted (inference): H unchanged
    if Z is not None:
        H2 = [_empty(T, f // p) for _ in range(p)]
        plan.column_fwd("mlp", T, dev(inp.X), W1s, b1s, None, H2)
        for i in range(p):
            assert torch.equal(H2[i], H[i])


@pytest.mark.parametrize("T,K,h,p", [(300, 264, 192, 2), (129, 1376, 4096, 1), (1, 64, 256, 8)])
def test_row_forward_partials(T, K, h, p):
    tp = _tp()
    g = torch.Generator().manual_seed(T)
    Hs = [torch.randn(T, K, generator=g).to(torch.bfloat16) for _ in range(p)]
    W2 = (torch.randn(h, K * p, generator=g) * 0.02).to(torch.bfloat16)
    plan = tp.Plan(h, K * p, 0, p, "bf16", "gelu")
    W2s = [_empty(h, K) for _ in range(p)]
    plan.shard_row("mlp", dev(W2), W2s)
    P = [_empty(T, h) for _ in range(p)]
    plan.row_fwd_partial("mlp", T, [dev(x) for x in Hs], W2s, P)
    for i in range(p):
        assert_close(P[i], O.row_partial(O.f64(Hs[i]), O.shard_cols(O.f64(W2), p, i)), TOL_BF16, f"P[{i}]")


@pytest.mark.parametrize("T,h,f,p,act", [(300, 192, 528, 2, "gelu"), (257, 256, 272, 2, "swiglu"),
                                         (200, 128, 512, 4, "none")])
def test_row_backward(T, h, f, p, act):
    """dZ_i = act'(dY W2_i), dW2_i = dY^T H_i, db2 = sum dY, from independent
    inputs (Z_i, H_i drawn, not produced by the forward)."""
    tp = _tp()
    g = torch.Generator().manual_seed(T + 1)
    k = f // p
    nz = 2 * k if act == "swiglu" else k
    dY = torch.randn(T, h, generator=g).to(torch.bfloat16)
    W2 = (torch.randn(h, f, generator=g) * 0.05).to(torch.bfloat16)
    Zs = [torch.randn(T, nz, generator=g).to(torch.bfloat16) for _ in range(p)]
    Hs = [torch.randn(T, k, generator=g).to(torch.bfloat16) for _ in range(p)]
    plan = tp.Plan(h, f, 0, p, "bf16", act)
    W2s = [_empty(h, k) for _ in range(p)]
    plan.shard_row("mlp", dev(W2), W2s)
    dZ = [_empty(T, nz) for _ in range(p)]
    dW = [_empty(h, k) for _ in range(p)]
    db = torch.empty(h, dtype=torch.float32, device="cuda")
    plan.row_bwd("mlp", T, dev(dY), [dev(x) for x in Hs], W2s,
                 [dev(z) for z in Zs] if act != "none" else None, dZ, dW, db)
    for i in range(p):
        rdz, rdw = O.row_bwd_shard(O.f64(dY), O.f64(Hs[i]), O.shard_cols(O.f64(W2), p, i), O.f64(Zs[i]), act)
        assert_close(dZ[i], rdz, TOL_BF16, f"dZ[{i}]")
        assert_close(dW[i], rdw, TOL_BF16, f"dW2[{i}]")
    assert_close(db[None, :], O.bias_grad(O.f64(dY))[None, :], 1e-4, "db2")


@pytest.mark.parametrize("T,h,f,p,act,which", [(300, 192, 528, 2, "gelu", "mlp"),
                                               (257, 256, 272, 2, "swiglu", "mlp"),
                                               (130, 256, 0, 4, "none", "qkv")])
def test_column_backward(T, h, f, p, act, which):
    tp = _tp()
    g = torch.Generator().manual_seed(T + 2)
    heads = 8 if which == "qkv" else 0
    if which == "qkv":
        n = 3 * h // p
        Wfull = (torch.randn(3 * h, h, generator=g) * 0.05).to(torch.bfloat16)
    else:
        n = (2 if act == "swiglu" else 1) * f // p
        Wfull = (torch.randn(n * p, h, generator=g) * 0.05).to(torch.bfloat16)
    X = torch.randn(T, h, generator=g).to(torch.bfloat16)
    dZs = [torch.randn(T, n, generator=g).to(torch.bfloat16) for _ in range(p)]
    plan = tp.Plan(h, f, heads, p, "bf16", act)
    Ws = [_empty(n, h) for _ in range(p)]
    plan.shard_column(which, dev(Wfull), Ws)
    dW = [_empty(n, h) for _ in range(p)]
    db = [torch.empty(n, dtype=torch.float32, device="cuda") for _ in range(p)]
    dXp = [_empty(T, h) for _ in range(p)]
    plan.column_bwd(which, T, dev(X), [dev(z) for z in dZs], Ws, dW, db, dXp)
    Wf = O.f64(Wfull)
    for i in range(p):
        if which == "qkv":
            Wi = O.shard_qkv(Wf, heads, p, i)
        else:
            Wi = _shard_w1(Wf, act, p, i)
        rdw, rdb, rdx = O.column_bwd_shard(O.f64(X), O.f64(dZs[i]), Wi)
        assert_close(dW[i], rdw, TOL_BF16, f"dW1[{i}]")
        assert_close(db[i][None, :], rdb[None, :], 1e-4, f"db1[{i}]")
        assert_close(dXp[i], rdx, TOL_BF16, f"dX partial {i}")


@pytest.mark.parametrize("T,p", [(512, 8), (300, 2)])
def test_qkv_column_forward_by_heads(T, p):
    tp = _tp()
    h, H = 512, 8
    a = tp_synth.draw_attn_block(1, T, h, torch.bfloat16, seed=T, bias=True)
    plan = tp.Plan(h, 0, H, p, "bf16", "none")
    n = 3 * h // p
    Ws = [_empty(n, h) for _ in range(p)]
    bs = [_empty(n) for _ in range(p)]
    plan.shard_column("qkv", dev(a.Wqkv), Ws)
    plan.shard_column_bias("qkv", dev(a.bqkv), bs)
    out = [_empty(T, n) for _ in range(p)]
    plan.column_fwd("qkv", T, dev(a.X), Ws, bs, None, out)
    full = O.linear(O.f64(a.X), O.f64(a.Wqkv), O.f64(a.bqkv))
    d, hl = h // H, H // p
    for i in range(p):
        c0, c1 = i * hl * d, (i + 1) * hl * d
        ref = np.concatenate([full[:, c0:c1], full[:, h + c0:h + c1], full[:, 2 * h + c0:2 * h + c1]], axis=1)
        assert_close(out[i], ref, TOL_BF16, f"QKV shard {i}")


def test_tiny_fp32_mlp_forward_backward():
    """The tiny fp32 MLP (X 64x128, A 128x512, B 512x128, p = 2) against the
    unsharded definition, fwd + bwd, within 1e-4."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    inp = tp_synth.draw_tiny_fp32_mlp(0)
    m = TPMLP(128, 512, 2, "gelu", "f32", bias=True)
    m.load_weights(dev(inp.W1), dev(inp.W2), dev(inp.b1), dev(inp.b2))
    Y = m.forward(dev(inp.X))
    dX = m.backward(dev(inp.dY))
    X, W1, W2, b1, b2, dY = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.b1, inp.b2, inp.dY))
    ref = O.mlp_fwd(X, W1, b1, W2, b2, "gelu")
    g = O.mlp_bwd(X, W1, W2, ref["Z"], ref["H"], dY, "gelu")
    assert_close(Y, ref["Y"], TOL_F32, "Y")
    assert_close(dX, g["dX"], TOL_F32, "dX")
    assert_close(torch.cat(m.dW1, 0), g["dW1"], TOL_F32, "dW1")
    assert_close(torch.cat(m.dW2, 1), g["dW2"], TOL_F32, "dW2")
    assert_close(torch.cat(m.db1, 0)[None, :], g["db1"][None, :], TOL_F32, "db1")
    assert_close(m.db2[None, :], g["db2"][None, :], TOL_F32, "db2")


@pytest.mark.parametrize("fused", [False, True], ids=["partials", "fused"])
@pytest.mark.parametrize("act,bias", [("gelu", True), ("swiglu", False), ("none", True)])
def test_fp32_mlp_every_epilogue(act, bias, fused):
    """fp32 plans run the same fused epilogues as bf16 (bias + GELU, SwiGLU with
    paired gate/up accumulators, their derivatives) in one grouped FMA launch,
    and the shard sums fused into the row and dX GEMMs; ragged tiles (T = 200,
    ffn/p = 72)."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    T, h, f, p = 200, 96, 288, 4
    inp = tp_synth.draw_mlp(T, h, f, act, torch.float32, seed=17, bias=bias)
    m = TPMLP(h, f, p, act, "f32", bias=bias, fused=fused)
    m.load_weights(dev(inp.W1), dev(inp.W2), dev(inp.b1), dev(inp.b2))
    Y = m.forward(dev(inp.X))
    dX = m.backward(dev(inp.dY))
    X, W1, W2, dY = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    b1, b2 = (O.f64(inp.b1), O.f64(inp.b2)) if bias else (None, None)
    ref = O.mlp_fwd(X, W1, b1, W2, b2, act)
    g = O.mlp_bwd(X, W1, W2, ref["Z"], ref["H"], dY, act)
    assert_close(Y, ref["Y"], TOL_F32, "Y")
    assert_close(dX, g["dX"], TOL_F32, "dX")
    for i in range(p):
        assert_close(m.dW1[i], _shard_w1(g["dW1"], act, p, i), TOL_F32, f"dW1 shard {i}")
        assert_close(m.dW2[i], O.shard_cols(g["dW2"], p, i), TOL_F32, f"dW2 shard {i}")
        if act != "none":
            assert_close(m.Z[i], _shard_w1(ref["Z"].T, act, p, i).T, TOL_F32, f"Z shard {i}")


@pytest.mark.parametrize("act,bias", [("gelu", True), ("swiglu", False)])
def test_bf16_mlp_end_to_end_small(act, bias):
    """Whole sharded MLP (forward + backward through TPMLP) against the unsharded
    definition on a small multi-tile case."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    T, h, f, p = 384, 256, 1024, 4
    inp = tp_synth.draw_mlp(T, h, f, act, torch.bfloat16, seed=5, bias=bias)
    m = TPMLP(h, f, p, act, "bf16", bias=bias)
    m.load_weights(dev(inp.W1), dev(inp.W2), dev(inp.b1), dev(inp.b2))
    Y = m.forward(dev(inp.X))
    dX = m.backward(dev(inp.dY))
    X, W1, W2, dY = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    b1, b2 = (O.f64(inp.b1), O.f64(inp.b2)) if bias else (None, None)
    ref = O.mlp_fwd(X, W1, b1, W2, b2, act)
    g = O.mlp_bwd(X, W1, W2, ref["Z"], ref["H"], dY, act)
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, g["dX"], TOL_BF16, "dX")
    dW1 = torch.empty(W1.shape, dtype=torch.bfloat16, device="cuda")
    m.plan.unshard_column("mlp", m.dW1, dW1)
    assert_close(dW1, g["dW1"], TOL_BF16, "dW1")
    dW2 = torch.empty(W2.shape, dtype=torch.bfloat16, device="cuda")
    m.plan.unshard_row("mlp", m.dW2, dW2)
    assert_close(dW2, g["dW2"], TOL_BF16, "dW2")


@pytest.mark.parametrize("T,K,h,p", [(300, 264, 192, 2), (257, 1376, 512, 8), (64, 128, 256, 1),
                                     (512, 264, 192, 4), (320, 136, 280, 5)])
def test_row_forward_fused_reduce(T, K, h, p):
    """The row GEMM with the shard sum fused: sum_i H_i W2_i^T + b + residual."""
    tp = _tp()
    g = torch.Generator().manual_seed(T + 11)
    Hs = [torch.randn(T, K, generator=g).to(torch.bfloat16) for _ in range(p)]
    W2 = (torch.randn(h, K * p, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.rand(h, generator=g) * 0.2 - 0.1).to(torch.bfloat16)
    r = torch.randn(T, h, generator=g).to(torch.bfloat16)
    plan = tp.Plan(h, K * p, 0, p, "bf16", "gelu")
    W2s = [_empty(h, K) for _ in range(p)]
    plan.shard_row("mlp", dev(W2), W2s)
    Y = _empty(T, h)
    plan.row_fwd_reduce("mlp", T, [dev(x) for x in Hs], W2s, dev(b), dev(r), Y)
    P = [O.row_partial(O.f64(Hs[i]), O.shard_cols(O.f64(W2), p, i)) for i in range(p)]
    ref = O.reduce_partials(P, O.f64(b), O.f64(r))
    assert_close(Y, ref, TOL_BF16, "fused row fwd")
    if T % p == 0:
        t = T // p
        Ys = [_empty(t, h) for _ in range(p)]
        rs = [dev(r[j * t:(j + 1) * t]) for j in range(p)]
        plan.row_fwd_reduce_scatter_seq("mlp", T, [dev(x) for x in Hs], W2s, dev(b), rs, Ys)
        refs = O.reduce_scatter_seq(P, O.f64(b), [O.f64(r[j * t:(j + 1) * t]) for j in range(p)])
        for j in range(p):
            assert_close(Ys[j], refs[j], TOL_BF16, f"fused RS shard {j}")


@pytest.mark.parametrize("T,h,f,p,act", [(300, 192, 528, 2, "gelu"), (256, 256, 272, 2, "swiglu"),
                                        (384, 192, 528, 3, "gelu")])
def test_column_backward_fused_reduce(T, h, f, p, act):
    tp = _tp()
    g = torch.Generator().manual_seed(T + 12)
    n = (2 if act == "swiglu" else 1) * f // p
    Wfull = (torch.randn(n * p, h, generator=g) * 0.05).to(torch.bfloat16)
    X = torch.randn(T, h, generator=g).to(torch.bfloat16)
    dZs = [torch.randn(T, n, generator=g).to(torch.bfloat16) for _ in range(p)]
    plan = tp.Plan(h, f, 0, p, "bf16", act)
    Ws = [_empty(n, h) for _ in range(p)]
    plan.shard_column("mlp", dev(Wfull), Ws)
    dX = _empty(T, h)
    plan.column_bwd_reduce("mlp", T, dev(X), [dev(z) for z in dZs], Ws, None, None, dX)
    Wf = O.f64(Wfull)
    parts = [O.column_bwd_shard(O.f64(X), O.f64(dZs[i]), _shard_w1(Wf, act, p, i))[2] for i in range(p)]
    assert_close(dX, O.reduce_partials(parts), TOL_BF16, "fused dX")
    t = T // p
    dXs = [_empty(t, h) for _ in range(p)]
    plan.column_bwd_reduce_scatter_seq("mlp", T, dev(X), [dev(z) for z in dZs], Ws, None, None, dXs)
    refs = O.reduce_scatter_seq(parts)
    for j in range(p):
        assert_close(dXs[j], refs[j], TOL_BF16, f"fused dX RS shard {j}")


@pytest.mark.parametrize("act,bias", [("gelu", True), ("swiglu", False)])
def test_bf16_mlp_end_to_end_small_fused(act, bias):
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    T, h, f, p = 384, 256, 1024, 4
    inp = tp_synth.draw_mlp(T, h, f, act, torch.bfloat16, seed=6, bias=bias)
    m = TPMLP(h, f, p, act, "bf16", bias=bias, fused=True)
    m.load_weights(dev(inp.W1), dev(inp.W2), dev(inp.b1), dev(inp.b2))
    Y = m.forward(dev(inp.X))
    dX = m.backward(dev(inp.dY))
    X, W1, W2, dY = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    b1, b2 = (O.f64(inp.b1), O.f64(inp.b2)) if bias else (None, None)
    ref = O.mlp_fwd(X, W1, b1, W2, b2, act)
    gr = O.mlp_bwd(X, W1, W2, ref["Z"], ref["H"], dY, act)
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, gr["dX"], TOL_BF16, "dX")


def test_overlapped_reduce_matches_sequential_bit_for_bit():
    """Token blocks reduced on a side stream under the next block's GEMM give
    exactly the sequential partials result (same kernels, same sums)."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    T, h, f, p = 1000, 256, 1024, 4
    inp = tp_synth.draw_mlp(T, h, f, "swiglu", torch.bfloat16, seed=8)
    outs = []
    for chunks in (0, 3):
        m = TPMLP(h, f, p, "swiglu", "bf16", overlap_chunks=chunks)
        m.load_weights(dev(inp.W1), dev(inp.W2))
        Y = m.forward(dev(inp.X)).clone()
        dX = m.backward(dev(inp.dY)).clone()
        torch.cuda.synchronize()
        outs.append((Y, dX, torch.cat(m.dW1, 0).clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][2], outs[1][2])


@pytest.mark.parametrize("chunks", [2, 3])
@pytest.mark.parametrize("act,bias", [("gelu", True), ("swiglu", False)])
def test_overlap_chunks_vs_oracle(chunks, act, bias):
    """f2 (token blocks, each block's reduce on a side stream under the next
    block's GEMM) against the oracle. T = 1000 is not a multiple of the
    128-row blocks (2 chunks: 512 + 488 rows; 3 chunks: 384 + 384 + 232)."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    T, h, f, p = 1000, 256, 1024, 4
    inp = tp_synth.draw_mlp(T, h, f, act, torch.bfloat16, seed=21, bias=bias)
    m = TPMLP(h, f, p, act, "bf16", bias=bias, overlap_chunks=chunks)
    assert m.chunks == chunks
    m.load_weights(dev(inp.W1), dev(inp.W2), dev(inp.b1), dev(inp.b2))
    Y = m.forward(dev(inp.X))
    dX = m.backward(dev(inp.dY))
    X, W1, W2, dY = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    b1, b2 = (O.f64(inp.b1), O.f64(inp.b2)) if bias else (None, None)
    ref = O.mlp_fwd(X, W1, b1, W2, b2, act)
    gr = O.mlp_bwd(X, W1, W2, ref["Z"], ref["H"], dY, act)
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, gr["dX"], TOL_BF16, "dX")
    for i in range(p):
        assert_close(m.dW1[i], _shard_w1(gr["dW1"], act, p, i), TOL_BF16, f"dW1 shard {i}")
        assert_close(m.dW2[i], O.shard_cols(gr["dW2"], p, i), TOL_BF16, f"dW2 shard {i}")
    if bias:
        for i in range(p):
            assert_close(m.db1[i][None, :], O.shard_vec(gr["db1"], p, i)[None, :], TOL_BF16, f"db1 shard {i}")
        assert_close(m.db2[None, :], gr["db2"][None, :], 1e-4, "db2")


def test_host_step_pipeline_matches_direct_steps():
    """Three overlapped host-fed steps with different inputs give, bit for
    bit, the outputs of the same steps run directly on device tensors."""
    from megatron_tensor_transformer_gemm_b200.block import HostStepPipeline, TPMLP
    T, h, f, p = 512, 256, 768, 4
    w = tp_synth.draw_mlp(T, h, f, "swiglu", torch.bfloat16, seed=3)
    m = TPMLP(h, f, p, "swiglu", "bf16", fused=True)
    m.load_weights(dev(w.W1), dev(w.W2))
    ins = [tp_synth.draw_mlp(T, h, f, "swiglu", torch.bfloat16, seed=10 + k) for k in range(3)]
    ref = []
    for d in ins:
        Y = m.forward(dev(d.X)).clone()
        dX = m.backward(dev(d.dY)).clone()
        ref.append((Y.cpu(), dX.cpu()))
    pipe = HostStepPipeline(m, T)
    outs = [(torch.empty(T, h, dtype=torch.bfloat16).pin_memory(),
             torch.empty(T, h, dtype=torch.bfloat16).pin_memory()) for _ in ins]
    for d, (Yh, dXh) in zip(ins, outs):
        pipe.step(d.X.pin_memory(), d.dY.pin_memory(), Yh, dXh)
    pipe.finish()
    torch.cuda.synchronize()
    for (Yr, dXr), (Yh, dXh) in zip(ref, outs):
        assert torch.equal(Yr, Yh)
        assert torch.equal(dXr, dXh)


@pytest.mark.parametrize("splits", ["2", "3", "16"])
def test_weight_gradients_with_split_k(splits):
    """Weight gradients whose K (the token dim) is split over several tile
    passes writing fp32 partials, summed in order by the reduce kernel into
    each shard's dW: forced split counts, ragged K (T = 1000: 16 K blocks, the
    last one partial), GELU and SwiGLU, in a subprocess so the forced split is
    read by a fresh library."""
    import subprocess
    import sys
    code = f"""
import sys; sys.path.insert(0, {ROOT!r}); sys.path.insert(0, {os.path.join(ROOT, 'tests')!r})
import numpy as np, torch, oracle as O, tp_synth
from gpu_helpers import TOL_BF16, assert_close, dev
from megatron_tensor_transformer_gemm_b200.block import TPMLP
for act in ("gelu", "swiglu"):
    T, h, f, p = 1000, 256, 512, 4
    inp = tp_synth.draw_mlp(T, h, f, act, torch.bfloat16, seed=23)
    m = TPMLP(h, f, p, act, "bf16", fused=True)
    m.load_weights(dev(inp.W1), dev(inp.W2))
    m.forward(dev(inp.X)); m.backward(dev(inp.dY))
    X, W1, W2, dY = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    ref = O.mlp_fwd(X, W1, None, W2, None, act)
    g = O.mlp_bwd(X, W1, W2, ref["Z"], ref["H"], dY, act)
    for i in range(p):
        sh1 = O.shard_gate_up(g["dW1"], p, i) if act == "swiglu" else O.shard_rows(g["dW1"], p, i)
        assert_close(m.dW1[i], sh1, TOL_BF16, f"dW1 shard {{i}}")
        assert_close(m.dW2[i], O.shard_cols(g["dW2"], p, i), TOL_BF16, f"dW2 shard {{i}}")
print("ok")
"""
    env = dict(os.environ, TP_GEMM_SPLITK=splits)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


@pytest.mark.parametrize("fused,act,T", [(True, "swiglu", 520), (False, "gelu", 384), (True, "gelu", 256)])
def test_grouped_weight_gradients_match_separate(fused, act, T, monkeypatch):
    """tp_set_wgrad_grouping: the row backward's dW2 waits and runs in one
    grouped launch with the column backward's dW1; every gradient is bit for
    bit the one the separate launches give (same tiles, same K order). The
    backward calls are kept on one stream (at these small sizes they would
    otherwise put the activation gradient beside the weight gradient, which
    launches the weight gradient at once)."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    monkeypatch.setenv("TP_BWD_CONCURRENT", "0")
    h, f, p = 256, 1024, 4
    inp = tp_synth.draw_mlp(T, h, f, act, torch.bfloat16, seed=81)
    outs = []
    for grouped in (False, True):
        m = TPMLP(h, f, p, act, "bf16", fused=fused, group_wgrad=grouped)
        m.load_weights(dev(inp.W1), dev(inp.W2))
        m.forward(dev(inp.X))
        dX = m.backward(dev(inp.dY)).clone()
        torch.cuda.synchronize()
        outs.append((dX, [w.clone() for w in m.dW1], [w.clone() for w in m.dW2]))
    (dX0, dW10, dW20), (dX1, dW11, dW21) = outs
    assert torch.equal(dX0, dX1)
    for i in range(p):
        assert torch.equal(dW10[i], dW11[i]), f"dW1 shard {i}"
        assert torch.equal(dW20[i], dW21[i]), f"dW2 shard {i}"
    Xo, W1, W2, dYo = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    ref = O.mlp_fwd(Xo, W1, None, W2, None, act)
    gr = O.mlp_bwd(Xo, W1, W2, ref["Z"], ref["H"], dYo, act)
    for i in range(p):
        assert_close(dW21[i], O.shard_cols(gr["dW2"], p, i), TOL_BF16, f"dW2 {i}")


def test_pending_weight_gradient_flushes(monkeypatch):
    """A row backward's waiting weight gradient is written by tp_flush_wgrad
    alone, and by switching grouping off."""
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    monkeypatch.setenv("TP_BWD_CONCURRENT", "0")
    T, h, f, p = 256, 256, 1024, 2
    inp = tp_synth.draw_mlp(T, h, f, "gelu", torch.bfloat16, seed=82)
    m = TPMLP(h, f, p, "gelu", "bf16", fused=True, group_wgrad=False)
    m.load_weights(dev(inp.W1), dev(inp.W2))
    m.forward(dev(inp.X))
    dY = dev(inp.dY)
    m.plan.row_bwd("mlp", T, dY, m.H, m.W2, m.Z, m.dZ, m.dW2, None)
    ref = [w.clone() for w in m.dW2]
    for grouped_flush in ("flush", "off"):
        m.plan.set_wgrad_grouping(True)
        for w in m.dW2:
            w.zero_()
        m.plan.row_bwd("mlp", T, dY, m.H, m.W2, m.Z, m.dZ, m.dW2, None)
        torch.cuda.synchronize()
        assert all(float(w.abs().max()) == 0.0 for w in m.dW2), "dW2 written before the flush"
        if grouped_flush == "flush":
            m.plan.flush_wgrad()
        else:
            m.plan.set_wgrad_grouping(False)
        torch.cuda.synchronize()
        for i in range(p):
            assert torch.equal(m.dW2[i], ref[i])
    m.plan.set_wgrad_grouping(False)
