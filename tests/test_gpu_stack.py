"""The 12-layer block stack (hidden 512, MLP 2048, 8 heads of 64, tokens 8x512,
p in {1, 2, 4}), forward and backward on the GPU against the oracle.

(a) Every layer, forward and backward, from an independently drawn input and
    upstream gradient: the layer's output, input gradient and every parameter
    gradient within the bf16 bound (2e-2, row-normalised).
(b) The whole stack chained (each layer fed its predecessor's output) against
    the oracle's own chain from the same inputs. bf16 storage rounds the
    residual stream at two boundaries per layer (x1 and y), and the two chains
    do not share those roundings, so their difference grows with depth: the
    bound for layer l is 2e-2 + l * 2 * 2^-8 (one bf16 unit roundoff, 2^-8,
    at each of the two stored boundaries of every layer before it), and the
    same again per layer for the backward chain."""
import numpy as np
import pytest
import torch

import oracle as O
import tp_synth
from gpu_helpers import dev, host

pytestmark = pytest.mark.gpu

TOL = 2e-2
PER_BOUNDARY = 2.0 ** -8          # bf16 unit roundoff, once per stored boundary
L, BATCH, SEQ, H_, F_, HEADS = 12, 8, 512, 512, 2048, 8


def _params64(prm):
    return {k: O.f64(getattr(prm, k)) for k in prm.__dataclass_fields__}


def _gpu_layer(prm, p, fused=True):
    from megatron_tensor_transformer_gemm_b200.block import TPLayer
    lay = TPLayer(H_, F_, HEADS, p, fused=fused)
    lay.load(type(prm)(**{k: dev(getattr(prm, k)) for k in prm.__dataclass_fields__}))
    return lay


def _err(got, ref):
    g = host(got) if isinstance(got, torch.Tensor) else got
    return O.max_row_rel_err(g, ref)


def _grad_errors(lay, gr, p):
    h, f = H_, F_
    errs = {}
    W1 = torch.empty(f, h, dtype=torch.bfloat16, device="cuda")
    lay.mlp.plan.unshard_column("mlp", lay.mlp.dW1, W1)
    errs["dW1"] = _err(W1, gr["dW1"])
    W2 = torch.empty(h, f, dtype=torch.bfloat16, device="cuda")
    lay.mlp.plan.unshard_row("mlp", lay.mlp.dW2, W2)
    errs["dW2"] = _err(W2, gr["dW2"])
    Wq = torch.empty(3 * h, h, dtype=torch.bfloat16, device="cuda")
    lay.attn.plan.unshard_column("qkv", lay.attn.dWqkv, Wq)
    errs["dWqkv"] = _err(Wq, gr["dWqkv"])
    Wo = torch.empty(h, h, dtype=torch.bfloat16, device="cuda")
    lay.attn.plan.unshard_row("outproj", lay.attn.dWo, Wo)
    errs["dWo"] = _err(Wo, gr["dWo"])
    errs["db2"] = _err(lay.mlp.db2[None, :], gr["db2"][None, :])
    errs["dbo"] = _err(lay.attn.dbo[None, :], gr["dbo"][None, :])
    errs["db1"] = _err(torch.cat(lay.mlp.db1)[None, :], gr["db1"][None, :])
    hl_d = h // p
    dbq = np.concatenate([host(b) for b in lay.attn.dbqkv])
    ref = np.concatenate([np.concatenate([gr["dbqkv"][part * h + i * hl_d: part * h + (i + 1) * hl_d]
                                          for part in range(3)]) for i in range(p)])
    errs["dbqkv"] = _err(dbq[None, :], ref[None, :])
    for k in ("dln1_g", "dln1_b", "dln2_g", "dln2_b"):
        errs[k] = _err(getattr(lay, k)[None, :], gr[k][None, :])
    return errs


@pytest.mark.parametrize("p,fused", [(1, True), (2, True), (4, True), (2, False), (4, False)])
def test_every_layer_fwd_bwd_from_independent_inputs(p, fused):
    _, layers, _ = tp_synth.draw_block_stack(L, BATCH, SEQ, H_, F_, torch.bfloat16, seed=0,
                                             ln_affine_random=True)
    report, worst = [], 0.0
    for l_, prm in enumerate(layers):
        g = torch.Generator().manual_seed(1000 + l_)
        x = torch.randn(BATCH * SEQ, H_, generator=g).to(torch.bfloat16)
        dy = torch.randn(BATCH * SEQ, H_, generator=g).to(torch.bfloat16)
        lay = _gpu_layer(prm, p, fused)
        y = lay.forward(dev(x), BATCH, SEQ)
        dx = lay.backward(dev(dy), BATCH, SEQ)
        P = _params64(prm)
        c = O.layer_fwd(O.f64(x), P, BATCH, HEADS)
        gr = O.layer_bwd(c, P, O.f64(dy), BATCH, HEADS)
        errs = {"y": _err(y, c["y"]), "dx": _err(dx, gr["dx"]), **_grad_errors(lay, gr, p)}
        report.append((l_, errs))
        worst = max(worst, max(errs.values()))
    lines = "\n".join(f"layer {l_}: " + " ".join(f"{k}={v:.2e}" for k, v in e.items()) for l_, e in report)
    assert worst <= TOL, f"worst {worst:.3e} > {TOL}\n{lines}"


@pytest.mark.parametrize("p", [1, 4])
def test_twelve_layer_chain_fwd_bwd(p):
    X, layers, dY = tp_synth.draw_block_stack(L, BATCH, SEQ, H_, F_, torch.bfloat16, seed=0,
                                              ln_affine_random=True)
    gpu_layers = [_gpu_layer(prm, p) for prm in layers]
    x = dev(X)
    outs = []
    for lay in gpu_layers:
        x = lay.forward(x, BATCH, SEQ)
        outs.append(x)
    g = dev(dY)
    for lay in reversed(gpu_layers):
        g = lay.backward(g, BATCH, SEQ)
    P64 = [_params64(prm) for prm in layers]
    xo = O.f64(X)
    caches, fails, lines = [], [], []
    for l_, prm in enumerate(P64):
        c = O.layer_fwd(xo, prm, BATCH, HEADS)
        caches.append(c)
        xo = c["y"]
        e = _err(outs[l_], xo)
        bound = TOL + 2 * l_ * PER_BOUNDARY
        lines.append(f"layer {l_} y: {e:.3e} (bound {bound:.3e})")
        if e > bound:
            fails.append(lines[-1])
    go = O.f64(dY)
    for l_ in reversed(range(L)):
        go = O.layer_bwd(caches[l_], P64[l_], go, BATCH, HEADS)["dx"]
    e = _err(g, go)
    bound = TOL + 2 * (2 * L) * PER_BOUNDARY
    lines.append(f"stack dX: {e:.3e} (bound {bound:.3e})")
    if e > bound:
        fails.append(lines[-1])
    assert not fails, "\n".join(lines)


def test_stack_step_replayed_as_cuda_graph_matches_eager():
    """One fwd+bwd step of three layers captured into a CUDA graph and replayed
    gives bit-identical outputs and gradients to the eager calls."""
    from megatron_tensor_transformer_gemm_b200.block import CapturedStep
    X, layers, dY = tp_synth.draw_block_stack(3, BATCH, SEQ, H_, F_, torch.bfloat16, seed=5,
                                              ln_affine_random=True)
    lays = [_gpu_layer(prm, 2) for prm in layers]
    Xd, dYd = dev(X), dev(dY)
    out = {}

    def step():
        x = Xd
        for lay in lays:
            x = lay.forward(x, BATCH, SEQ)
        g = dYd
        for lay in reversed(lays):
            g = lay.backward(g, BATCH, SEQ)
        out["y"], out["dx"] = x, g

    from megatron_tensor_transformer_gemm_b200 import tp
    tp.launch_count(reset=True)
    step()
    torch.cuda.synchronize()
    eager_launches = tp.launch_count(reset=True)
    y_eager, dx_eager = out["y"].clone(), out["dx"].clone()
    w_eager = lays[0].mlp.dW1[0].clone()
    g = CapturedStep(step)
    assert g.launches == eager_launches > 0  # the graph holds every kernel of the step
    out["y"].zero_()
    lays[0].mlp.dW1[0].zero_()
    g()
    torch.cuda.synchronize()
    assert torch.equal(out["y"], y_eager)
    assert torch.equal(out["dx"], dx_eager)
    assert torch.equal(lays[0].mlp.dW1[0], w_eager)


def test_deferred_weight_gradients_joined_once():
    """TPLayer leaves its weight gradients and bias sums on the side stream
    (tp_set_backward_defer). Backpropagating three layers with one join at the
    end gives the gradients, bit for bit, of joining after every layer, and,
    within the bf16 tolerance, those of the plans with deferral off (every
    backward GEMM joined inside its call)."""
    from megatron_tensor_transformer_gemm_b200 import tp
    from gpu_helpers import TOL_BF16, assert_close
    X, layers, dY = tp_synth.draw_block_stack(3, BATCH, SEQ, H_, F_, torch.bfloat16, seed=9,
                                              ln_affine_random=True)
    lays = [_gpu_layer(prm, 2) for prm in layers]

    def run(join_each):
        x = dev(X)
        for lay in lays:
            x = lay.forward(x, BATCH, SEQ)
        g = dev(dY)
        for lay in reversed(lays):
            g = lay.backward(g, BATCH, SEQ, join=join_each)
        if not join_each:
            tp.backward_join()
        torch.cuda.synchronize()
        out = [g.clone()]
        for lay in lays:
            out += [t.clone() for t in (lay.mlp.dW1[0], lay.mlp.dW2[1], lay.attn.dWqkv[1], lay.attn.dWo[0])]
            out += [lay.mlp.db2.clone()[None, :], lay.attn.dbo.clone()[None, :], lay.mlp.db1[1].clone()[None, :]]
        return out

    each = run(True)
    once = run(False)
    for a, b in zip(each, once):
        assert torch.equal(a, b)
    for lay in lays:
        lay.attn.plan.set_backward_defer(False)
        lay.mlp.plan.set_backward_defer(False)
    immediate = run(True)
    for i, (a, b) in enumerate(zip(each, immediate)):
        assert_close(a, host(b).astype(np.float64), TOL_BF16, f"gradient {i}")
