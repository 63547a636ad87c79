"""GPU parity of the attention core on local heads and of the attention
sublayer (QKV by whole heads -> attention -> out-projection partials -> reduce)."""
import numpy as np
import pytest
import torch

import oracle as O
import tp_synth
from gpu_helpers import TOL_BF16, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _tp():
    from megatron_tensor_transformer_gemm_b200 import tp
    return tp


@pytest.mark.parametrize("batch,seq,heads,d,p", [
    (2, 300, 4, 64, 2),     # 3 query tiles, ragged last tile and key block
    (1, 256, 2, 128, 1),
    (3, 129, 8, 64, 4),
    (2, 512, 4, 128, 2),
])
def test_attention_fwd_local_heads(batch, seq, heads, d, p):
    tp = _tp()
    h = heads * d
    Q, K, V, _ = tp_synth.draw_qkv_activations(batch, seq, heads, d, torch.bfloat16, seed=seq, dy=False)
    hl = heads // p
    plan = tp.Plan(h, 0, heads, p, "bf16", "none")
    qkv, outs, lses = [], [], []
    for i in range(p):
        sl = slice(i * hl * d, (i + 1) * hl * d)
        qkv.append(dev(torch.cat([Q[:, :, sl], K[:, :, sl], V[:, :, sl]], dim=2).reshape(seq * batch, 3 * hl * d)))
        outs.append(torch.empty(seq * batch, hl * d, dtype=torch.bfloat16, device="cuda"))
        lses.append(torch.empty(batch, hl, seq, dtype=torch.float32, device="cuda"))
    plan.attention_fwd(batch, seq, qkv, outs, lses)
    ref, ref_lse = O.attention_fwd(O.f64(Q), O.f64(K), O.f64(V), batch, heads, True)
    got = np.concatenate([host(o).reshape(seq, batch, hl * d) for o in outs], axis=2)
    assert_close(got.reshape(seq * batch, h), ref.reshape(seq * batch, h), TOL_BF16, "O")
    got_lse = np.concatenate([host(l_) for l_ in lses], axis=1)
    np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=2e-2)


@pytest.mark.parametrize("d", [64, 128])
def test_attention_fwd_growing_scores_rescale(d):
    """Keys scaled up along the sequence so that every row's max grows by far
    more than 2^8 from one key block to the next: exercises the in-place
    rescale of O (and l) in TMEM."""
    tp = _tp()
    batch, seq, heads, p = 1, 1024, 2, 1
    h = heads * d
    Q, K, V, _ = tp_synth.draw_qkv_activations(batch, seq, heads, d, torch.bfloat16, seed=d, dy=False)
    ramp = (1.0 + torch.arange(seq, dtype=torch.float32) / 16.0).view(seq, 1, 1)
    Q = (Q.float() * 2.0).to(torch.bfloat16)
    K = (K.float() * ramp).to(torch.bfloat16)
    plan = tp.Plan(h, 0, heads, p, "bf16", "none")
    qkv = dev(torch.cat([Q, K, V], dim=2).reshape(seq * batch, 3 * h))
    out = torch.empty(seq * batch, h, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(batch, heads, seq, dtype=torch.float32, device="cuda")
    plan.attention_fwd(batch, seq, [qkv], [out], [lse])
    ref, ref_lse = O.attention_fwd(O.f64(Q), O.f64(K), O.f64(V), batch, heads, True)
    assert_close(out, ref.reshape(seq * batch, h), TOL_BF16, "O")
    np.testing.assert_allclose(host(lse), ref_lse, rtol=1e-4, atol=5e-2)
    assert tp.device_status() == "TP_OK"


@pytest.mark.parametrize("fused", [False, True])
def test_attention_block_full_size_sampled(fused):
    """hidden 4096, 32 heads x 128, seq 4096, batch 2, p 8 (4 heads per shard),
    causal; QKV -> attention -> out-projection partials -> reduce + residual
    (fused: the out-projection sums the shards in its accumulator)."""
    from megatron_tensor_transformer_gemm_b200.block import TPAttention
    batch, seq, h, H, p = 2, 4096, 4096, 32, 8
    a = tp_synth.draw_attn_block(batch, seq, h, torch.bfloat16, seed=0)
    blk = TPAttention(h, H, p, fused=fused)
    blk.load_weights(dev(a.Wqkv), dev(a.Wo))
    X = dev(a.X)
    Y = blk.forward(X, batch, seq, residual=X)
    rows_s = tp_synth.sample_rows(seq, 16, seed=5).numpy()
    X64 = O.f64(a.X)
    QKV = O.linear(X64, O.f64(a.Wqkv))
    Qf = QKV[:, :h].reshape(seq, batch, h)
    Kf = QKV[:, h:2 * h].reshape(seq, batch, h)
    Vf = QKV[:, 2 * h:].reshape(seq, batch, h)
    Osub, _ = O.attention_fwd_rows(Qf, Kf, Vf, batch, H, rows_s, True)
    Yref = O.linear(Osub.reshape(-1, h), O.f64(a.Wo)) + X64.reshape(seq, batch, h)[rows_s].reshape(-1, h)
    got = host(Y).reshape(seq, batch, h)[rows_s].reshape(-1, h)
    assert_close(got, Yref, TOL_BF16, "Y sampled rows")
    assert _tp().device_status() == "TP_OK"


@pytest.mark.parametrize("ds", ["1", "0"])
@pytest.mark.parametrize("batch,seq,heads,d,p", [
    (2, 300, 4, 64, 2),
    (1, 256, 2, 128, 1),
    (3, 129, 8, 64, 4),
    (1, 520, 2, 128, 2),
])
def test_attention_bwd_local_heads(batch, seq, heads, d, p, ds, monkeypatch):
    """dQ, dK, dV of each shard's heads from independent Q, K, V, dO; O and LSE
    come from the GPU forward of those inputs (the oracle computes its own).
    ds = "1": dQ as a GEMM over the dS^T the dK/dV kernel stores; "0": dQ
    recomputing S and dP (TP_ATTN_BWD_DS=0, read at each call)."""
    monkeypatch.setenv("TP_ATTN_BWD_DS", ds)
    tp = _tp()
    h = heads * d
    Q, K, V, dO = tp_synth.draw_qkv_activations(batch, seq, heads, d, torch.bfloat16, seed=seq + 7)
    hl = heads // p
    plan = tp.Plan(h, 0, heads, p, "bf16", "none")
    qkv, outs, lses, dos, dqkv = [], [], [], [], []
    for i in range(p):
        sl = slice(i * hl * d, (i + 1) * hl * d)
        qkv.append(dev(torch.cat([Q[:, :, sl], K[:, :, sl], V[:, :, sl]], dim=2).reshape(seq * batch, 3 * hl * d)))
        outs.append(torch.empty(seq * batch, hl * d, dtype=torch.bfloat16, device="cuda"))
        lses.append(torch.empty(batch, hl, seq, dtype=torch.float32, device="cuda"))
        dos.append(dev(dO[:, :, sl].reshape(seq * batch, hl * d)))
        dqkv.append(torch.empty(seq * batch, 3 * hl * d, dtype=torch.bfloat16, device="cuda"))
    plan.attention_fwd(batch, seq, qkv, outs, lses)
    plan.attention_bwd(batch, seq, qkv, outs, dos, lses, dqkv)
    rq, rk, rv = O.attention_bwd(O.f64(Q), O.f64(K), O.f64(V), O.f64(dO), batch, heads, True)
    got = [host(x).reshape(seq, batch, 3, hl * d) for x in dqkv]
    for name, idx, ref in (("dQ", 0, rq), ("dK", 1, rk), ("dV", 2, rv)):
        g = np.concatenate([x[:, :, idx, :] for x in got], axis=2)
        assert_close(g.reshape(seq * batch, h), ref.reshape(seq * batch, h), TOL_BF16, name)


def test_attention_fwd_p_in_shared_memory():
    """The forward's earlier form (TP_ATTN_P_SMEM=1: P through shared memory
    instead of TMEM) on the same forward cases, in a subprocess so the choice
    is made before the library's first launch."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(root, "tests", "test_gpu_attention.py"), "-k",
                        "fwd_local_heads or growing_scores"],
                       cwd=root, env=dict(os.environ, TP_ATTN_P_SMEM="1"), capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
