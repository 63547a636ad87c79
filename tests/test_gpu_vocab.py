"""GPU parity of the vocab-parallel embedding and cross-entropy (the vocab is
padded so the p shards split it; padding excluded from the softmax)."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import TOL_BF16, TOL_F32, assert_bitexact, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _tp():
    from megatron_tensor_transformer_gemm_b200 import tp
    return tp


@pytest.mark.parametrize("p", [1, 2, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_embedding_fwd_bwd(p, dtype):
    tp = _tp()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    T, V, h = 1000, 1000, 256
    plan = tp.Plan(h, 0, 0, p, dtype, "none")
    Vp = plan.set_vocab(V)
    g = torch.Generator().manual_seed(p)
    E = torch.randn(Vp, h, generator=g).to(tdt)
    ids = torch.randint(0, V, (T,), generator=g, dtype=torch.int32)
    ids[:50] = 7                      # a heavily repeated id
    ids[-1] = V - 1
    Es = [torch.empty(Vp // p, h, dtype=tdt, device="cuda") for _ in range(p)]
    plan.shard_column("vocab", dev(E), Es)
    Y = torch.empty(T, h, dtype=tdt, device="cuda")
    idd = ids.cuda()
    plan.embedding_fwd(T, idd, Es, Y)
    assert_bitexact(Y, O.embedding_fwd(ids.numpy(), O.f64(E)), "lookup")
    # integer-valued gradients: every sum is exact, so the backward is bit for bit
    dY = torch.randint(-2, 3, (T, h), generator=g).to(tdt)
    dE = [torch.full((Vp // p, h), 9.0, dtype=tdt, device="cuda") for _ in range(p)]
    plan.embedding_bwd(T, idd, dev(dY), dE)
    ref = O.embedding_bwd(ids.numpy(), O.f64(dY), Vp)
    assert_bitexact(torch.cat(dE, 0), ref, "embedding grad")
    dY = torch.randn(T, h, generator=g).to(tdt)
    plan.embedding_bwd(T, idd, dev(dY), dE)
    ref = O.embedding_bwd(ids.numpy(), O.f64(dY), Vp)
    used = np.unique(ids.numpy())
    assert_close(host(torch.cat(dE, 0))[used], ref[used], TOL_BF16 if dtype == "bf16" else TOL_F32, "dE")
    assert _tp().device_status() == "TP_OK"


@pytest.mark.parametrize("p,V,dtype", [(1, 1000, "bf16"), (4, 1001, "bf16"), (8, 32000, "bf16"),
                                       (4, 50000, "bf16"), (8, 128000, "bf16"), (3, 997, "f32"),
                                       (8, 32000, "f32")])
def test_vocab_parallel_cross_entropy(p, V, dtype):
    """Rows staged three or two deep in shared memory (up to 66 KB / 100 KB)
    and wider rows (the streaming kernel), padded and unpadded vocabularies,
    bf16 and fp32; 1000 rows so every persistent CTA recycles its stages."""
    tp = _tp()
    T, h = (1000, 64) if V <= 50000 else (40, 64)
    plan = tp.Plan(h if h % p == 0 else 3 * h, 0, 0, p, dtype, "none")
    Vp = plan.set_vocab(V)
    g = torch.Generator().manual_seed(V)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    z = (torch.randn(T, Vp, generator=g) * 3).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    labels = torch.randint(0, V, (T,), generator=g, dtype=torch.int32)
    labels[0] = V - 1
    labels[5] = -1                    # ignored token
    Vs = Vp // p
    L = [dev(z[:, i * Vs:(i + 1) * Vs]) for i in range(p)]
    G = [torch.empty_like(x) for x in L]
    loss = torch.empty(T, dtype=torch.float32, device="cuda")
    lse = torch.empty(T, dtype=torch.float32, device="cuda")
    plan.vocab_cross_entropy(T, L, labels.cuda(), 1.0 / T, loss, lse, G)
    lab = labels.numpy().copy()
    keep = lab >= 0
    z64 = O.f64(z)
    rl, rg = O.cross_entropy(z64[keep], lab[keep], V)
    gl = host(loss)
    np.testing.assert_allclose(gl[keep], rl, rtol=1e-4, atol=1e-4)
    assert gl[5] == 0.0
    gg = np.concatenate([host(x) for x in G], axis=1)
    assert np.all(gg[5] == 0) and np.all(gg[:, V:] == 0)
    # oracle gradient of the mean over the kept tokens, rescaled to 1/T
    assert_close(gg[keep] * T, rg * keep.sum(), tol, "dlogits")
    # in place (dlogits aliasing the logits)
    plan.vocab_cross_entropy(T, L, labels.cuda(), 1.0 / T, loss, None, L)
    assert_close(np.concatenate([host(x) for x in L], axis=1)[keep] * T, rg * keep.sum(), tol, "in place")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_embedding_bwd_many_blocks_heavy_id_and_ignored_ids(dtype):
    """Tokens spanning several 1024-token blocks, one id repeated 2000 times (a
    token list longer than one chunk), ids outside [0, vocab) ignored, a hidden
    size with a ragged 512-column tile; integer-valued dY makes every sum exact,
    so the result is bit for bit, and two calls agree bit for bit."""
    tp = _tp()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    T, V, h, p = 5000, 3000, 1032, 4
    plan = tp.Plan(h, 0, 0, p, dtype, "none")
    Vp = plan.set_vocab(V)
    g = torch.Generator().manual_seed(5)
    ids = torch.randint(0, V, (T,), generator=g, dtype=torch.int32)
    heavy = torch.randperm(T, generator=g)[:2000]
    ids[heavy] = V - 1
    ids[17] = -1
    ids[4000] = -5
    dY = torch.randint(-1, 2, (T, h), generator=g).to(tdt)
    dE = [torch.full((Vp // p, h), 7.0, dtype=tdt, device="cuda") for _ in range(p)]
    idd = ids.cuda()
    plan.embedding_bwd(T, idd, dev(dY), dE)
    keep = (ids >= 0).numpy()
    ref = O.embedding_bwd(ids.numpy()[keep], O.f64(dY)[keep], Vp)
    assert np.abs(ref).max() <= 256      # every sum is an integer that bf16 holds exactly
    assert_bitexact(torch.cat(dE, 0), ref, "embedding grad")
    dY = torch.randn(T, h, generator=g).to(tdt)
    first = [torch.empty_like(x) for x in dE]
    plan.embedding_bwd(T, idd, dev(dY), first)
    plan.embedding_bwd(T, idd, dev(dY), dE)
    for a, b in zip(first, dE):
        assert torch.equal(a, b)
    ref = O.embedding_bwd(ids.numpy()[keep], O.f64(dY)[keep], Vp)
    used = np.unique(ids.numpy()[keep])
    assert_close(host(torch.cat(dE, 0))[used], ref[used], TOL_BF16 if dtype == "bf16" else TOL_F32, "dE")
    assert tp.device_status() == "TP_OK"


def test_output_head_logits_loss_and_gradients():
    """Output head end to end: logits = X W^T by vocab shards (column GEMM),
    vocab-parallel loss, then dX (shard sum fused) and dW from the loss gradient."""
    tp = _tp()
    T, h, V, p = 512, 512, 32000, 8
    plan = tp.Plan(h, 0, 0, p, "bf16", "none")
    Vp = plan.set_vocab(V)
    g = torch.Generator().manual_seed(1)
    X = torch.randn(T, h, generator=g).to(torch.bfloat16)
    W = (torch.randn(Vp, h, generator=g) * 0.02).to(torch.bfloat16)
    labels = torch.randint(0, V, (T,), generator=g, dtype=torch.int32)
    Vs = Vp // p
    Ws = [torch.empty(Vs, h, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    plan.shard_column("vocab", dev(W), Ws)
    L = [torch.empty(T, Vs, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    Xd = dev(X)
    plan.column_fwd("vocab", T, Xd, Ws, None, None, L)
    loss = torch.empty(T, dtype=torch.float32, device="cuda")
    plan.vocab_cross_entropy(T, L, labels.cuda(), 1.0 / T, loss, None, L)
    dX = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    dW = [torch.empty_like(w) for w in Ws]
    plan.column_bwd_reduce("vocab", T, Xd, L, Ws, dW, None, dX)
    X64, W64 = O.f64(X), O.f64(W)
    z = O.linear(X64, W64)
    rl, rg = O.cross_entropy(z, labels.numpy(), V)
    np.testing.assert_allclose(host(loss), rl, rtol=2e-3, atol=2e-3)
    assert_close(dX, rg @ W64, TOL_BF16, "dX")
    assert_close(torch.cat(dW, 0)[:V], (rg.T @ X64)[:V], TOL_BF16, "dW")
