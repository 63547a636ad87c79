"""DistTPMLP (p shards split over the ranks of an NCCL group) on the one GPU
these tests have: a single-rank NCCL group, so every collective is the
identity and the result must equal the single-GPU fused path bit for bit,
and the oracle within the bf16 tolerance. The multi-rank exchange logic is
covered on CPU gloo ranks (test_dist_cpu.py)."""
import datetime
import os
import socket

import pytest
import torch

import oracle as O
import tp_synth
from gpu_helpers import TOL_BF16, assert_close, dev

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture(scope="module")
def nccl_group():
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


def test_dist_mlp_single_rank_equals_local_fused(nccl_group):
    from megatron_tensor_transformer_gemm_b200.block import TPMLP
    from megatron_tensor_transformer_gemm_b200.dist import DistTPMLP
    T, h, f, p = 768, 512, 2048, 8
    inp = tp_synth.draw_mlp(T, h, f, "swiglu", torch.bfloat16, seed=11)
    m = TPMLP(h, f, p, "swiglu", "bf16", fused=True)
    m.load_weights(dev(inp.W1), dev(inp.W2))
    d = DistTPMLP(h, f, p, "swiglu", group=nccl_group)
    d.load_weights(inp.W1, inp.W2)
    X, dY, res = dev(inp.X), dev(inp.dY), dev(inp.X) * 0.5
    Y_ref = m.forward(X, residual=res).clone()
    dX_ref = m.backward(dY).clone()
    Y = d.forward(X, residual=res)
    dX = d.backward(dY)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_ref)
    assert torch.equal(dX, dX_ref)
    for i in range(p):
        assert torch.equal(d.dW1[i], m.dW1[i])
        assert torch.equal(d.dW2[i], m.dW2[i])
    Xo, W1, W2, dYo = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    ref = O.mlp_fwd(Xo, W1, None, W2, None, "swiglu", residual=O.f64(res))
    gr = O.mlp_bwd(Xo, W1, W2, ref["Z"], ref["H"], dYo, "swiglu")
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, gr["dX"], TOL_BF16, "dX")


def test_dist_mlp_sequence_parallel_single_rank(nccl_group):
    """Megatron-SP through the distributed layer (LayerNorm on the rank's
    sequence shard, all-gather, column, row, reduce-scatter, and back)."""
    from megatron_tensor_transformer_gemm_b200.dist import DistTPMLP
    seq, h, f, p = 256, 512, 1536, 4
    X, g, b, W1, W2, dY = tp_synth.draw_sp_mlp(seq, h, f, p, torch.bfloat16, seed=12, ln_affine_random=True)
    d = DistTPMLP(h, f, p, "swiglu", group=nccl_group, sequence_parallel=True)
    d.load_weights(W1, W2)
    d.gamma.copy_(dev(g))
    d.beta.copy_(dev(b))
    Y = d.forward(dev(X))
    dX = d.backward(dev(dY))
    Xo, go, bo, W1o, W2o, dYo = (O.f64(t) for t in (X, g, b, W1, W2, dY))
    ref = O.sp_mlp_fwd(Xo, go, bo, W1o, W2o)
    rb = O.sp_mlp_bwd(Xo, go, W1o, W2o, ref, dYo)
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, rb["dX"], TOL_BF16, "dX")
    assert_close(d.dgamma[None, :], rb["dg"][None, :], TOL_BF16, "dgamma")
    assert_close(d.dbeta[None, :], rb["db"][None, :], TOL_BF16, "dbeta")


def test_dist_mlp_gelu_bias_single_rank(nccl_group):
    from megatron_tensor_transformer_gemm_b200.dist import DistTPMLP
    T, h, f, p = 384, 256, 1024, 4
    inp = tp_synth.draw_mlp(T, h, f, "gelu", torch.bfloat16, seed=13, bias=True)
    d = DistTPMLP(h, f, p, "gelu", group=nccl_group, bias=True)
    d.load_weights(inp.W1, inp.W2, inp.b1, dev(inp.b2))
    Y = d.forward(dev(inp.X))
    dX = d.backward(dev(inp.dY))
    Xo, W1, W2, dYo = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
    ref = O.mlp_fwd(Xo, W1, O.f64(inp.b1), W2, O.f64(inp.b2), "gelu")
    gr = O.mlp_bwd(Xo, W1, W2, ref["Z"], ref["H"], dYo, "gelu")
    assert_close(Y, ref["Y"], TOL_BF16, "Y")
    assert_close(dX, gr["dX"], TOL_BF16, "dX")
    assert_close(d.db2[None, :], gr["db2"][None, :], 1e-4, "db2")
    for j, i in enumerate(d.shards):
        assert_close(d.db1[j][None, :], O.shard_vec(gr["db1"], p, i)[None, :], TOL_BF16, f"db1 {i}")


@pytest.mark.parametrize("sp", [False, True])
def test_dist_mlp_peer_comm_single_rank(nccl_group, sp):
    """comm="peer": the all-reduces (SP: reduce-scatters) of Y and dX through
    the peer-memory steps (push from the GEMM epilogue, reduce, wait) on a
    one-rank group, against the oracle; a second step repeats the first."""
    from megatron_tensor_transformer_gemm_b200.dist import DistTPMLP
    if sp:
        seq, h, f, p = 256, 512, 1536, 4
        X, g, b, W1, W2, dY = tp_synth.draw_sp_mlp(seq, h, f, p, torch.bfloat16, seed=14, ln_affine_random=True)
        d = DistTPMLP(h, f, p, "swiglu", group=nccl_group, sequence_parallel=True, comm="peer")
        d.load_weights(W1, W2)
        d.gamma.copy_(dev(g))
        d.beta.copy_(dev(b))
        try:
            Y = d.forward(dev(X)).clone()
            dX = d.backward(dev(dY)).clone()
            Y2 = d.forward(dev(X)).clone()
            dX2 = d.backward(dev(dY)).clone()
            Xo, go, bo, W1o, W2o, dYo = (O.f64(t) for t in (X, g, b, W1, W2, dY))
            ref = O.sp_mlp_fwd(Xo, go, bo, W1o, W2o)
            rb = O.sp_mlp_bwd(Xo, go, W1o, W2o, ref, dYo)
            assert_close(Y, ref["Y"], TOL_BF16, "Y")
            assert_close(dX, rb["dX"], TOL_BF16, "dX")
            assert torch.equal(Y, Y2) and torch.equal(dX, dX2)
        finally:
            d.close_peer()
        return
    T, h, f, p = 384, 256, 1024, 4
    inp = tp_synth.draw_mlp(T, h, f, "gelu", torch.bfloat16, seed=15, bias=True)
    d = DistTPMLP(h, f, p, "gelu", group=nccl_group, bias=True, comm="peer")
    d.load_weights(inp.W1, inp.W2, inp.b1, dev(inp.b2))
    res = (dev(inp.X) * 0.5).contiguous()
    try:
        Y = d.forward(dev(inp.X), residual=res).clone()
        dX = d.backward(dev(inp.dY)).clone()
        Y2 = d.forward(dev(inp.X), residual=res).clone()
        dX2 = d.backward(dev(inp.dY)).clone()
        from megatron_tensor_transformer_gemm_b200 import tp
        torch.cuda.synchronize()
        assert tp.lib.tp_get_device_status(None, None) == 0
        Xo, W1, W2, dYo = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
        ref = O.mlp_fwd(Xo, W1, O.f64(inp.b1), W2, O.f64(inp.b2), "gelu", residual=O.f64(res))
        gr = O.mlp_bwd(Xo, W1, W2, ref["Z"], ref["H"], dYo, "gelu")
        assert_close(Y, ref["Y"], TOL_BF16, "Y")
        assert_close(dX, gr["dX"], TOL_BF16, "dX")
        assert torch.equal(Y, Y2) and torch.equal(dX, dX2)
    finally:
        d.close_peer()
