"""Pins for the CPU oracle: checks against things other than the oracle itself.

Closed forms, library routines for special cases, hand-worked integer values,
central finite differences (fp64) for every backward, algebraic invariants of
the sharded method the pages state, and brute force in pure-Python loops on
tiny shapes. The mutation tests at the end plant plausible mistakes in copies
of oracle functions and check that some pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit
from scipy.stats import norm

import oracle as O
import tp_synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(7)


def randn(*shape, std=1.0):
    return rng.standard_normal(shape) * std


# ---------------------------------------------------------------- closed forms

def test_gelu_is_z_times_normal_cdf():
    z = np.linspace(-8, 8, 4001)
    np.testing.assert_allclose(O.gelu(z), z * norm.cdf(z), rtol=1e-13, atol=1e-15)
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu(np.array([30.0]))[0] - 30.0) < 1e-12
    assert abs(O.gelu(np.array([-30.0]))[0]) < 1e-12


def test_silu_is_z_times_logistic():
    z = np.linspace(-30, 30, 4001)
    np.testing.assert_allclose(O.silu(z), z * expit(z), rtol=1e-13, atol=1e-15)
    assert O.silu(np.array([0.0]))[0] == 0.0


def _fd_scalar(f, z, eps=1e-6):
    return (f(z + eps) - f(z - eps)) / (2 * eps)


def test_activation_derivatives_by_finite_differences():
    z = np.linspace(-6, 6, 241)
    np.testing.assert_allclose(O.gelu_grad(z), _fd_scalar(O.gelu, z), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(O.silu_grad(z), _fd_scalar(O.silu, z), rtol=1e-7, atol=1e-9)
    assert abs(O.gelu_grad(np.array([0.0]))[0] - 0.5) < 1e-15
    assert abs(O.silu_grad(np.array([0.0]))[0] - 0.5) < 1e-15


# ------------------------------------------------------- hand-worked golden

def test_golden_column_and_row_split():
    g = json.load(open(os.path.join(GOLDEN, "split_2x2_hand.json")))
    X, A, B = (np.array(g[k], dtype=np.float64) for k in ("X", "A", "B"))
    assert np.array_equal(O.linear(X, A), np.array(g["XAt"]))
    for i in range(2):
        assert np.array_equal(O.linear(X, O.shard_rows(A, 2, i)), np.array(g["XAt_shards_p2"][i]))
    assert np.array_equal(O.linear(X, B), np.array(g["XBt"]))
    Xs = [X[:, :2], X[:, 2:]]
    P = [O.row_partial(Xs[i], O.shard_cols(B, 2, i)) for i in range(2)]
    for i in range(2):
        assert np.array_equal(P[i], np.array(g["XBt_partials_p2"][i]))
    assert np.array_equal(O.reduce_partials(P), np.array(g["XBt"]))


# --------------------------------------------------------- brute force (loops)

def _bf_linear(X, W, b=None):
    T, n_in = len(X), len(X[0])
    n_out = len(W)
    Y = [[0.0] * n_out for _ in range(T)]
    for t in range(T):
        for o in range(n_out):
            acc = 0.0
            for k in range(n_in):
                acc += X[t][k] * W[o][k]
            Y[t][o] = acc + (b[o] if b is not None else 0.0)
    return np.array(Y)


def _bf_gelu(z):
    return z * 0.5 * (1.0 + math.erf(z / math.sqrt(2.0)))


def _bf_silu(z):
    return z / (1.0 + math.exp(-z))


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_brute_force_mlp_tiny(act):
    T, h, f = 5, 8, 12
    X = randn(T, h)
    W1 = randn(f if act == "gelu" else 2 * f, h, std=0.3)
    W2 = randn(h, f, std=0.3)
    b1 = randn(W1.shape[0]) if act == "gelu" else None
    b2 = randn(h)
    Z = _bf_linear(X.tolist(), W1.tolist(), None if b1 is None else b1.tolist())
    if act == "gelu":
        H = np.vectorize(_bf_gelu)(Z)
    else:
        H = np.vectorize(_bf_silu)(Z[:, :f]) * Z[:, f:]
    Y = _bf_linear(H.tolist(), W2.tolist(), b2.tolist())
    out = O.mlp_fwd(X, W1, b1, W2, b2, act)
    np.testing.assert_allclose(out["Z"], Z, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out["H"], H, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out["Y"], Y, rtol=1e-12, atol=1e-13)


def _bf_attention(q, k, v, causal):
    """q, k, v: lists [s][d] for one (batch, head)."""
    s, d = len(q), len(q[0])
    out = []
    for i in range(s):
        scores = []
        for j in range(s):
            if causal and j > i:
                continue
            scores.append((j, sum(q[i][x] * k[j][x] for x in range(d)) / math.sqrt(d)))
        m = max(sc for _, sc in scores)
        w = [(j, math.exp(sc - m)) for j, sc in scores]
        z = sum(e for _, e in w)
        out.append([sum(e * v[j][x] for j, e in w) / z for x in range(d)])
    return out


@pytest.mark.parametrize("causal", [True, False])
def test_brute_force_attention_tiny(causal):
    s, b, H, d = 5, 2, 3, 4
    Q, K, V = randn(s, b, H * d), randn(s, b, H * d), randn(s, b, H * d)
    got, _ = O.attention_fwd(Q, K, V, b, H, causal)
    for bi in range(b):
        for hh in range(H):
            sl = slice(hh * d, (hh + 1) * d)
            ref = _bf_attention(Q[:, bi, sl].tolist(), K[:, bi, sl].tolist(), V[:, bi, sl].tolist(), causal)
            np.testing.assert_allclose(got[:, bi, sl], np.array(ref), rtol=1e-12, atol=1e-13)


def test_brute_force_layernorm_tiny():
    x = randn(4, 10)
    g, b = randn(10), randn(10)
    y, mean, rstd = O.layernorm_fwd(x, g, b)
    for r in range(4):
        row = x[r].tolist()
        mu = sum(row) / len(row)
        var = sum((v - mu) ** 2 for v in row) / len(row)
        ref = [(v - mu) / math.sqrt(var + 1e-5) * g[c] + b[c] for c, v in enumerate(row)]
        np.testing.assert_allclose(y[r], ref, rtol=1e-12, atol=1e-13)
        assert abs(mean[r] - mu) < 1e-14


# ------------------------------------------------- invariants of the method

@pytest.mark.parametrize("p", [1, 2, 4])
@pytest.mark.parametrize("act", ["none", "gelu"])
def test_column_split_concat_equals_full(p, act):
    """XA = [XA_1, ..., XA_p] (wiki 两种切法; walkthrough §2.1)."""
    X, A, a = randn(6, 16), randn(32, 16), randn(32)
    Z, H = O.column_fwd_shard(X, A, a, act)
    parts = [O.column_fwd_shard(X, O.shard_rows(A, p, i), O.shard_vec(a, p, i), act) for i in range(p)]
    np.testing.assert_allclose(np.concatenate([z for z, _ in parts], axis=1), Z, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(np.concatenate([hh for _, hh in parts], axis=1), H, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("p", [1, 2, 4])
def test_swiglu_gate_up_pairing(p):
    """Each shard must pair gate units i with up units i (walkthrough §3.2):
    concat of the shards' H equals the unsharded H; a naive p-way split of the
    stacked [G; U] rows does not (for p > 1)."""
    T, h, f = 6, 16, 24
    X, W1 = randn(T, h), randn(2 * f, h)
    H = O.mlp_fwd(X, W1, None, randn(h, f), None, "swiglu")["H"]
    Hs = [O.column_fwd_shard(X, O.shard_gate_up(W1, p, i), None, "swiglu")[1] for i in range(p)]
    np.testing.assert_allclose(np.concatenate(Hs, axis=1), H, rtol=1e-13, atol=1e-14)
    if p > 1:
        naive = [O.column_fwd_shard(X, O.shard_rows(W1, p, i), None, "swiglu")[1] for i in range(p)]
        assert not np.allclose(np.concatenate(naive, axis=1), H)


@pytest.mark.parametrize("p", [1, 2, 4, 8])
def test_row_partials_sum_to_full(p):
    """XB = X_1B_1 + ... + X_pB_p (wiki 两种切法; walkthrough §2.2)."""
    H, B = randn(7, 32), randn(16, 32)
    P = [O.row_partial(O.shard_cols(H, p, i), O.shard_cols(B, p, i)) for i in range(p)]
    for Pi in P:
        assert Pi.shape == (7, 16)
    full = H @ B.T
    assert np.abs(O.reduce_partials(P) - full).max() <= 1e-12 * np.abs(full).max()


@pytest.mark.parametrize("p", [2, 4, 8])
def test_bias_added_once(p):
    """The row bias enters once, after the sum (bjdmk 实现细节). Integer values
    make every sum exact: a per-shard bias would differ by exactly (p-1)*b."""
    P, b, _ = tp_synth.draw_partials(p, 5, 6, torch.float32, integer_valued=True)
    P, b = [O.f64(x) for x in P], O.f64(b)
    once = O.reduce_partials(P, bias=b)
    pfold = O.reduce_partials([Pi + b[None, :] for Pi in P])
    assert np.array_equal(pfold - once, np.broadcast_to((p - 1) * b, once.shape))
    assert np.array_equal(once, sum(P) + b[None, :])


def test_reduce_p1_is_copy_plus_bias():
    P, b, r = tp_synth.draw_partials(1, 4, 8, torch.float32, residual=True)
    P, b, r = [O.f64(x) for x in P], O.f64(b), O.f64(r)
    assert np.array_equal(O.reduce_partials(P, b, r), (P[0] + b[None, :]) + r)


@pytest.mark.parametrize("p", [1, 2, 4])
def test_head_split_attention_equals_unsplit(p):
    """Attention on each shard's whole heads, concatenated, equals attention on
    all heads (walkthrough §3.1): the per-head computation is identical."""
    s, b, H, d = 6, 2, 4, 3
    Q, K, V = randn(s, b, H * d), randn(s, b, H * d), randn(s, b, H * d)
    full, lse = O.attention_fwd(Q, K, V, b, H, True)
    hl = H // p
    outs, lses = [], []
    for i in range(p):
        sl = slice(i * hl * d, (i + 1) * hl * d)
        o, l_ = O.attention_fwd(Q[:, :, sl], K[:, :, sl], V[:, :, sl], b, hl, True)
        outs.append(o)
        lses.append(l_)
    assert np.array_equal(np.concatenate(outs, axis=2), full)
    assert np.array_equal(np.concatenate(lses, axis=1), lse)


@pytest.mark.parametrize("p", [1, 2, 4])
def test_qkv_head_shard_feeds_local_attention(p):
    """QKV weight sharded by whole heads gives each shard exactly its heads' Q, K, V."""
    T, h, H = 6, 12, 4
    u, W, bq = randn(T, h), randn(3 * h, h), randn(3 * h)
    full = O.linear(u, W, bq)
    d, hl = h // H, H // p
    for i in range(p):
        part = O.linear(u, O.shard_qkv(W, H, p, i), O.shard_qkv_vec(bq, H, p, i))
        c0, c1 = i * hl * d, (i + 1) * hl * d
        ref = np.concatenate([full[:, c0:c1], full[:, h + c0:h + c1], full[:, 2 * h + c0:2 * h + c1]], axis=1)
        np.testing.assert_allclose(part, ref, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("p", [1, 2, 4, 8])
def test_reduce_scatter_then_all_gather_is_all_reduce(p):
    """AG(RS(P)) == AR(P) bit for bit (walkthrough §4.3, wiki Megatron-SP)."""
    P, b, _ = tp_synth.draw_partials(p, 8 * p, 12, torch.float32)
    P, b = [O.f64(x) for x in P], O.f64(b)
    assert np.array_equal(O.all_gather_seq(O.reduce_scatter_seq(P, b)), O.reduce_partials(P, b))


def test_layernorm_commutes_with_all_gather():
    X = randn(16, 10)
    g, b = randn(10), randn(10)
    shards = [X[i * 4:(i + 1) * 4] for i in range(4)]
    a = O.all_gather_seq([O.layernorm_fwd(s_, g, b)[0] for s_ in shards])
    assert np.array_equal(a, O.layernorm_fwd(O.all_gather_seq(shards), g, b)[0])


def test_layernorm_rows_standardised():
    y, _, _ = O.layernorm_fwd(randn(8, 64, std=3.0) + 5.0, np.ones(64), np.zeros(64))
    np.testing.assert_allclose(y.mean(axis=1), 0.0, atol=1e-13)
    np.testing.assert_allclose(y.var(axis=1), 1.0, rtol=1e-4)


def test_softmax_rows_sum_to_one_and_causal_row0():
    s, d = 6, 6
    Q, K = randn(s, 1, d), randn(s, 1, d)
    V = np.eye(s).reshape(s, 1, s)  # O = P itself when V is the identity
    Pm, _ = O.attention_fwd(Q, K, V, 1, 1, True)
    Pm = Pm[:, 0, :]
    np.testing.assert_allclose(Pm.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(np.triu(Pm, k=1) == 0.0)
    V2 = randn(s, 1, d)
    out, _ = O.attention_fwd(Q, K, V2, 1, 1, True)
    assert np.array_equal(out[0, 0], V2[0, 0])


# ------------------------------------------- backward: finite differences

def _fd_grad(fun, x, eps=1e-6, idx=None):
    """Central differences of scalar fun() with respect to entries of x (in place)."""
    flat = x.reshape(-1)
    if idx is None:
        idx = range(flat.size)
    g = []
    for i in idx:
        old = flat[i]
        flat[i] = old + eps
        fp = fun()
        flat[i] = old - eps
        fm = fun()
        flat[i] = old
        g.append((fp - fm) / (2 * eps))
    return np.array(g)


def _check_fd(analytic, fun, x, n=12, rtol=1e-6):
    idx = rng.choice(x.size, size=min(n, x.size), replace=False)
    num = _fd_grad(fun, x, idx=idx)
    ana = analytic.reshape(-1)[idx]
    scale = max(np.abs(ana).max(), 1e-3)
    assert np.abs(num - ana).max() <= rtol * scale, (num, ana)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_mlp_bwd_finite_differences(act):
    T, h, f = 4, 6, 8
    X = randn(T, h)
    W1 = randn(f if act == "gelu" else 2 * f, h, std=0.5)
    W2 = randn(h, f, std=0.5)
    b1 = randn(W1.shape[0]) if act == "gelu" else None
    b2 = randn(h)
    C = randn(T, h)  # loss = sum(C * Y), so dY = C

    def loss():
        return float((O.mlp_fwd(X, W1, b1, W2, b2, act)["Y"] * C).sum())

    fwd = O.mlp_fwd(X, W1, b1, W2, b2, act)
    g = O.mlp_bwd(X, W1, W2, fwd["Z"], fwd["H"], C, act)
    _check_fd(g["dX"], loss, X)
    _check_fd(g["dW1"], loss, W1)
    _check_fd(g["dW2"], loss, W2)
    _check_fd(g["db2"], loss, b2)
    if b1 is not None:
        _check_fd(g["db1"], loss, b1)


def test_layernorm_bwd_finite_differences():
    x, g, b = randn(5, 7), randn(7), randn(7)
    C = randn(5, 7)

    def loss():
        return float((O.layernorm_fwd(x, g, b)[0] * C).sum())

    _, mean, rstd = O.layernorm_fwd(x, g, b)
    dx, dg, db = O.layernorm_bwd(x, g, C, mean, rstd)
    _check_fd(dx, loss, x, n=20)
    _check_fd(dg, loss, g, n=7)
    _check_fd(db, loss, b, n=7)


@pytest.mark.parametrize("causal", [True, False])
def test_attention_bwd_finite_differences(causal):
    s, b, H, d = 5, 2, 2, 3
    Q, K, V = randn(s, b, H * d), randn(s, b, H * d), randn(s, b, H * d)
    C = randn(s, b, H * d)

    def loss():
        return float((O.attention_fwd(Q, K, V, b, H, causal)[0] * C).sum())

    dQ, dK, dV = O.attention_bwd(Q, K, V, C, b, H, causal)
    _check_fd(dQ, loss, Q, n=20)
    _check_fd(dK, loss, K, n=20)
    _check_fd(dV, loss, V, n=20)


def test_attention_rows_matches_full():
    s, b, H, d = 9, 2, 2, 3
    Q, K, V = randn(s, b, H * d), randn(s, b, H * d), randn(s, b, H * d)
    full, lse = O.attention_fwd(Q, K, V, b, H, True)
    rows = np.array([0, 4, 8])
    part, lse_r = O.attention_fwd_rows(Q, K, V, b, H, rows, True)
    np.testing.assert_allclose(part, full[rows], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse_r, lse[:, :, rows], rtol=1e-13, atol=1e-14)


def test_attention_lse_definition():
    s, b, H, d = 4, 1, 1, 2
    Q, K, V = randn(s, b, d), randn(s, b, d), randn(s, b, d)
    _, lse = O.attention_fwd(Q, K, V, b, H, True)
    for i in range(s):
        sc = [float(Q[i, 0] @ K[j, 0]) / math.sqrt(d) for j in range(i + 1)]
        assert abs(lse[0, 0, i] - math.log(sum(math.exp(x) for x in sc))) < 1e-12


def _layer_params(h, f, H):
    P = {"ln1_g": 1 + 0.1 * randn(h), "ln1_b": 0.1 * randn(h), "Wqkv": randn(3 * h, h, std=0.4),
         "bqkv": 0.1 * randn(3 * h), "Wo": randn(h, h, std=0.4), "bo": 0.1 * randn(h),
         "ln2_g": 1 + 0.1 * randn(h), "ln2_b": 0.1 * randn(h), "W1": randn(f, h, std=0.4),
         "b1": 0.1 * randn(f), "W2": randn(h, f, std=0.4), "b2": 0.1 * randn(h)}
    return P


def test_layer_bwd_finite_differences():
    batch, s, h, f, H = 2, 3, 4, 8, 2
    x = randn(batch * s, h)
    P = _layer_params(h, f, H)
    C = randn(batch * s, h)

    def loss():
        return float((O.layer_fwd(x, P, batch, H)["y"] * C).sum())

    cache = O.layer_fwd(x, P, batch, H)
    g = O.layer_bwd(cache, P, C, batch, H)
    _check_fd(g["dx"], loss, x, n=10)
    for name, gname in [("Wqkv", "dWqkv"), ("bqkv", "dbqkv"), ("Wo", "dWo"), ("bo", "dbo"),
                        ("W1", "dW1"), ("b1", "db1"), ("W2", "dW2"), ("b2", "db2"),
                        ("ln1_g", "dln1_g"), ("ln1_b", "dln1_b"), ("ln2_g", "dln2_g"), ("ln2_b", "dln2_b")]:
        _check_fd(g[gname], loss, P[name], n=6)


def test_sp_mlp_bwd_finite_differences():
    s, h, f = 6, 6, 8
    X, g, b = randn(s, h), 1 + 0.1 * randn(h), 0.1 * randn(h)
    W1, W2 = randn(2 * f, h, std=0.5), randn(h, f, std=0.5)
    C = randn(s, h)

    def loss():
        return float((O.sp_mlp_fwd(X, g, b, W1, W2)["Y"] * C).sum())

    fwd = O.sp_mlp_fwd(X, g, b, W1, W2)
    gr = O.sp_mlp_bwd(X, g, W1, W2, fwd, C)
    _check_fd(gr["dX"], loss, X)
    _check_fd(gr["dg"], loss, g, n=6)
    _check_fd(gr["db"], loss, b, n=6)
    _check_fd(gr["dW1"], loss, W1)


# ----------------------------------- sharded backward equals the unsharded one

@pytest.mark.parametrize("p", [1, 2, 4])
@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_sharded_backward_matches_unsharded(p, act):
    """Row bwd needs no sum (dY replicated); column bwd dX partials sum to dX
    (从零实现 Tensor Parallel §四)."""
    T, h, f = 6, 8, 16
    X = randn(T, h)
    W1 = randn(f if act == "gelu" else 2 * f, h, std=0.5)
    W2 = randn(h, f, std=0.5)
    b1 = randn(W1.shape[0]) if act == "gelu" else None
    dY = randn(T, h)
    fwd = O.mlp_fwd(X, W1, b1, W2, None, act)
    ref = O.mlp_bwd(X, W1, W2, fwd["Z"], fwd["H"], dY, act)
    shard = (lambda W, i: O.shard_rows(W, p, i)) if act == "gelu" else (lambda W, i: O.shard_gate_up(W, p, i))
    dXp, dW1s, dW2s, db1s = [], [], [], []
    for i in range(p):
        Wi = shard(W1, i)
        bi = None if b1 is None else O.shard_vec(b1, p, i)
        Zi, Hi = O.column_fwd_shard(X, Wi, bi, act)
        dZi, dW2i = O.row_bwd_shard(dY, Hi, O.shard_cols(W2, p, i), Zi, act)
        dWi, dbi, dXi = O.column_bwd_shard(X, dZi, Wi)
        dXp.append(dXi)
        dW1s.append(dWi)
        dW2s.append(dW2i)
        db1s.append(dbi)
    np.testing.assert_allclose(O.reduce_partials(dXp), ref["dX"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(dW2s, axis=1), ref["dW2"], rtol=1e-12, atol=1e-12)
    for i in range(p):
        np.testing.assert_allclose(dW1s[i], shard(ref["dW1"], i), rtol=1e-12, atol=1e-12)
        if b1 is not None:
            np.testing.assert_allclose(db1s[i], O.shard_vec(ref["db1"], p, i), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("p", [1, 2, 4])
def test_sp_pipeline_equals_unsharded(p):
    """LN on sequence shards -> AG -> column -> row partials -> RS equals the
    unsharded LN -> MLP, and the backward (AG of dY, RS of dX partials, LN bwd
    per shard, dgamma/dbeta summed over shards) equals the unsharded backward."""
    s, h, f = 8, 8, 16
    X, g, b = randn(s, h), 1 + 0.1 * randn(h), 0.1 * randn(h)
    W1, W2 = randn(2 * f, h, std=0.5), randn(h, f, std=0.5)
    dY = randn(s, h)
    ref = O.sp_mlp_fwd(X, g, b, W1, W2)
    refb = O.sp_mlp_bwd(X, g, W1, W2, ref, dY)
    t = s // p
    Xs = [X[j * t:(j + 1) * t] for j in range(p)]
    lns = [O.layernorm_fwd(x, g, b) for x in Xs]
    u = O.all_gather_seq([l_[0] for l_ in lns])
    Zs, Hs, P = [], [], []
    for i in range(p):
        Zi, Hi = O.column_fwd_shard(u, O.shard_gate_up(W1, p, i), None, "swiglu")
        Zs.append(Zi)
        Hs.append(Hi)
        P.append(O.row_partial(Hi, O.shard_cols(W2, p, i)))
    Ys = O.reduce_scatter_seq(P)
    np.testing.assert_allclose(O.all_gather_seq(Ys), ref["Y"], rtol=1e-12, atol=1e-12)
    dYfull = O.all_gather_seq([dY[j * t:(j + 1) * t] for j in range(p)])
    dXp = []
    for i in range(p):
        dZi, _ = O.row_bwd_shard(dYfull, Hs[i], O.shard_cols(W2, p, i), Zs[i], "swiglu")
        dXp.append(O.column_bwd_shard(u, dZi, O.shard_gate_up(W1, p, i))[2])
    du_seq = O.reduce_scatter_seq(dXp)
    dXs, dgs, dbs = [], [], []
    for j in range(p):
        dx, dg_, db_ = O.layernorm_bwd(Xs[j], g, du_seq[j], lns[j][1], lns[j][2])
        dXs.append(dx)
        dgs.append(dg_)
        dbs.append(db_)
    np.testing.assert_allclose(O.all_gather_seq(dXs), refb["dX"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(sum(dgs), refb["dg"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(sum(dbs), refb["db"], rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_sampled_backward_matches_full(act):
    T, h, f = 20, 8, 12
    X = randn(T, h)
    W1 = randn(f if act == "gelu" else 2 * f, h, std=0.5)
    b1 = randn(W1.shape[0]) if act == "gelu" else None
    W2, dY = randn(h, f, std=0.5), randn(T, h)
    fwd = O.mlp_fwd(X, W1, b1, W2, None, act)
    ref = O.mlp_bwd(X, W1, W2, fwd["Z"], fwd["H"], dY, act)
    rows, fcols = np.array([0, 3, 19]), np.array([1, 5, 11])
    smp = O.mlp_bwd_sampled(X, W1, b1, W2, dY, act, rows, fcols)
    np.testing.assert_allclose(smp["dX_rows"], ref["dX"][rows], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(smp["dW2_cols"], ref["dW2"][:, fcols], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(smp["dW1_rows"], ref["dW1"][smp["W1_rows_index"]], rtol=1e-12, atol=1e-12)
    if act == "gelu":
        np.testing.assert_allclose(smp["db1"], ref["db1"][fcols], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(
        O.mlp_fwd_rows(X, W1, b1, W2, None, act, rows)["Y"], fwd["Y"][rows], rtol=1e-12, atol=1e-12)


def test_max_row_rel_err():
    ref = np.array([[1.0, -4.0], [0.0, 0.0], [2.0, 1.0]])
    got = ref + np.array([[0.0, 0.04], [0.0, 0.0], [0.02, 0.0]])
    assert abs(O.max_row_rel_err(got, ref) - 0.01) < 1e-15
    assert O.max_row_rel_err(got * np.nan, ref) == float("inf")


def test_divisibility_is_checked():
    with pytest.raises(ValueError):
        O.shard_rows(np.zeros((10, 4)), 4, 0)
    with pytest.raises(ValueError):
        O.shard_qkv(np.zeros((3 * 12, 12)), 3, 2, 0)


# ------------------------------- bias gradient, gate/up bias shard, RS residual

def test_bias_grad_hand_worked():
    """A bias added to every token row receives the column sums of dY over the
    tokens (chain rule through Y = ... + 1 b^T); integers worked by hand."""
    dY = np.array([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0], [-2.0, 0.0, 7.0]])
    assert np.array_equal(O.bias_grad(dY), np.array([3.0, 7.0, 16.0]))


def test_bias_grad_brute_force_and_fd():
    T, n = 9, 5
    dY, X, b = randn(T, n), randn(T, n), randn(1, n)
    got = O.bias_grad(dY)
    assert got.shape == (n,)
    loops = [sum(dY[t, c] for t in range(T)) for c in range(n)]
    np.testing.assert_allclose(got, loops, rtol=1e-14, atol=1e-14)
    # d/db of sum(dY * (X + 1 b^T)) by central differences
    _check_fd(got, lambda: float((dY * (X + b)).sum()), b, n=n)


def test_mutant_bias_grad_mean_or_wrong_axis_fails():
    dY = np.array([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0], [-2.0, 0.0, 7.0]])
    ref = np.array([3.0, 7.0, 16.0])
    assert not np.array_equal(dY.mean(axis=0), ref)
    assert not np.array_equal(dY.sum(axis=1), ref)


def test_shard_gate_up_vec_hand_worked_and_matches_weight_rows():
    """The bias of a SwiGLU column shard pairs gate entries i*f/p.. with the
    same up entries, exactly like the weight rows of [G_i; U_i] (walkthrough §3.2)."""
    b1 = np.array([10.0, 11.0, 12.0, 13.0, 20.0, 21.0, 22.0, 23.0])  # gate 10.., up 20..
    assert np.array_equal(O.shard_gate_up_vec(b1, 2, 0), [10.0, 11.0, 20.0, 21.0])
    assert np.array_equal(O.shard_gate_up_vec(b1, 2, 1), [12.0, 13.0, 22.0, 23.0])
    for p in (1, 2, 4):
        b = randn(2 * 8)
        for i in range(p):
            as_rows = O.shard_gate_up(b[:, None], p, i)[:, 0]
            assert np.array_equal(O.shard_gate_up_vec(b, p, i), as_rows)
    with pytest.raises(ValueError):
        O.shard_gate_up_vec(np.zeros(2 * 6), 4, 0)


@pytest.mark.parametrize("p", [1, 2, 4])
def test_gate_up_bias_shards_give_the_full_swiglu(p):
    """Column shards of W1 and of its bias, each paired gate/up, reproduce the
    full SwiGLU activation's columns i*f/p.. of shard i."""
    T, h, f = 5, 6, 8
    X, W1, b1 = randn(T, h), randn(2 * f, h), randn(2 * f)
    Z = X @ W1.T + b1[None, :]
    H_full = O.silu(Z[:, :f]) * Z[:, f:]
    k = f // p
    for i in range(p):
        _, H_i = O.column_fwd_shard(X, O.shard_gate_up(W1, p, i), O.shard_gate_up_vec(b1, p, i), "swiglu")
        np.testing.assert_allclose(H_i, H_full[:, i * k:(i + 1) * k], rtol=1e-13, atol=1e-14)


def test_reduce_scatter_residual_hand_worked():
    """Each sequence shard j adds ITS residual rows after the sum and the bias
    (walkthrough §4.3); integers worked by hand, T = 4 rows over n = 2 shards."""
    P0 = np.array([[1.0, 2.0], [3.0, 4.0], [5.0, 6.0], [7.0, 8.0]])
    P1 = np.array([[10.0, 20.0], [30.0, 40.0], [50.0, 60.0], [70.0, 80.0]])
    b = np.array([100.0, 200.0])
    r = [np.array([[1000.0, 2000.0], [3000.0, 4000.0]]),
         np.array([[5000.0, 6000.0], [7000.0, 8000.0]])]
    out = O.reduce_scatter_seq([P0, P1], b, r)
    assert np.array_equal(out[0], [[1111.0, 2222.0], [3133.0, 4244.0]])
    assert np.array_equal(out[1], [[5155.0, 6266.0], [7177.0, 8288.0]])


@pytest.mark.parametrize("p", [1, 2, 4, 8])
def test_reduce_scatter_residual_brute_force(p):
    """Integer-valued partials, bias and residual shards: element by element in
    pure Python, shard j row r = sum_i P_i[j*t + r] + b + R_j[r]."""
    t, h = 3, 4
    P, b, _ = tp_synth.draw_partials(p, p * t, h, torch.float32, integer_valued=True)
    P, b = [O.f64(x) for x in P], O.f64(b)
    R = [rng.integers(-8, 9, (t, h)).astype(np.float64) for _ in range(p)]
    out = O.reduce_scatter_seq(P, b, R)
    for j in range(p):
        for r in range(t):
            for c in range(h):
                want = sum(P[i][j * t + r, c] for i in range(p)) + b[c] + R[j][r, c]
                assert out[j][r, c] == want
    if p > 1:  # a residual taken from the wrong shard gives a different result
        bad = O.reduce_scatter_seq(P, b, R[::-1])
        assert any(not np.array_equal(x, y) for x, y in zip(bad, out))


# ------------------------------------------------ mutation checks (plant bugs)

def _mut_gelu_tanh(z):
    return 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))


def test_mutant_tanh_gelu_fails_the_cdf_pin():
    z = np.linspace(-8, 8, 4001)
    assert not np.allclose(_mut_gelu_tanh(z), z * norm.cdf(z), rtol=1e-13, atol=1e-15)


def test_mutant_layernorm_bwd_dropped_term_fails_fd():
    x, g, b = randn(5, 7), randn(7), randn(7)
    C = randn(5, 7)
    _, mean, rstd = O.layernorm_fwd(x, g, b)
    xhat = (x - mean[:, None]) * rstd[:, None]
    gy = C * g[None, :]
    bad_dx = rstd[:, None] * (gy - gy.mean(axis=1, keepdims=True))  # dropped the xhat term
    with pytest.raises(AssertionError):
        _check_fd(bad_dx, lambda: float((O.layernorm_fwd(x, g, b)[0] * C).sum()), x, n=20)


def test_mutant_attention_missing_scale_fails_brute_force():
    s, b, H, d = 4, 1, 1, 4
    Q, K, V = randn(s, b, d), randn(s, b, d), randn(s, b, d)
    bad, _ = O.attention_fwd(Q * math.sqrt(d), K, V, b, H, True)  # scale dropped
    ref = _bf_attention(Q[:, 0].tolist(), K[:, 0].tolist(), V[:, 0].tolist(), True)
    assert not np.allclose(bad[:, 0], np.array(ref), rtol=1e-6)


def test_mutant_transposed_row_shard_fails_the_sum_pin():
    H, B = randn(7, 32), randn(16, 32)
    p = 4
    bad = [O.shard_cols(H, p, i) @ O.shard_cols(B, p, p - 1 - i).T for i in range(p)]  # wrong shard index
    assert not np.allclose(O.reduce_partials(bad), H @ B.T)


def test_mutant_silu_grad_sign_fails_fd():
    z = np.linspace(-6, 6, 241)
    s = 1 / (1 + np.exp(-z))
    bad = s * (1 - z * (1 - s))
    assert not np.allclose(bad, _fd_scalar(O.silu, z), rtol=1e-7, atol=1e-9)


# --------------------------------------------- hidden-sharded norm statistics

def test_rmsnorm_brute_force_and_fd():
    x, g = randn(4, 9), randn(9)
    y, rstd = O.rmsnorm_fwd(x, g)
    for r in range(4):
        ms = sum(v * v for v in x[r].tolist()) / 9
        ref = [v / math.sqrt(ms + 1e-5) * g[c] for c, v in enumerate(x[r].tolist())]
        np.testing.assert_allclose(y[r], ref, rtol=1e-12, atol=1e-13)
    C = randn(4, 9)
    dx, dg = O.rmsnorm_bwd(x, g, C, rstd)
    _check_fd(dx, lambda: float((O.rmsnorm_fwd(x, g)[0] * C).sum()), x, n=20)
    _check_fd(dg, lambda: float((O.rmsnorm_fwd(x, g)[0] * C).sum()), g, n=9)


def test_rmsnorm_rows_have_unit_rms():
    y, _ = O.rmsnorm_fwd(randn(6, 64, std=4.0), np.ones(64))
    np.testing.assert_allclose(np.sqrt((y * y).mean(axis=1)), 1.0, rtol=1e-5)


@pytest.mark.parametrize("kind", ["rms", "ln"])
@pytest.mark.parametrize("p", [1, 2, 4])
def test_hidden_sharded_norm_equals_full_norm(kind, p):
    """Local sums reduced over shards give the full-row statistics (walkthrough §3.3)."""
    T, h = 5, 16
    x, g, b, dy = randn(T, h, std=2.0) + 0.3, 1 + 0.1 * randn(h), 0.1 * randn(h), randn(T, h)
    xs, gs, bs, dys = ([O.shard_cols(a, p, i) for i in range(p)] for a in (x, g[None, :], b[None, :], dy))
    gs, bs = [a[0] for a in gs], [a[0] for a in bs]
    ys, stats = O.norm_sharded_fwd(xs, gs, bs, kind)
    dxs, dgs, dbs = O.norm_sharded_bwd(xs, gs, dys, stats, kind)
    if kind == "rms":
        y, rstd = O.rmsnorm_fwd(x, g)
        dx, dg = O.rmsnorm_bwd(x, g, dy, rstd)
    else:
        y, mean, rstd = O.layernorm_fwd(x, g, b)
        dx, dg, db = O.layernorm_bwd(x, g, dy, mean, rstd)
        np.testing.assert_allclose(np.concatenate(dbs), db, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(ys, axis=1), y, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(dxs, axis=1), dx, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(dgs), dg, rtol=1e-10, atol=1e-12)


def test_mutant_local_only_statistics_fail_the_sharded_norm_pin():
    """Normalising each shard by its own statistics (the mistake the walkthrough
    §3.3 warns about) does not reproduce the full-row norm."""
    x, g = randn(5, 16, std=2.0) + 1.0, np.ones(16)
    y, _ = O.rmsnorm_fwd(x, g)
    bad = np.concatenate([O.rmsnorm_fwd(O.shard_cols(x, 2, i), g[:8])[0] for i in range(2)], axis=1)
    assert not np.allclose(bad, y, rtol=1e-6)


# ------------------------------------------ vocab-parallel embedding and loss

def test_vocab_padding():
    assert O.vocab_padded(32000, 8) == 32000
    assert O.vocab_padded(32001, 8) == 32064
    assert O.vocab_padded(50257, 4) == 50272
    assert O.vocab_padded(10, 3, align=1) == 12


@pytest.mark.parametrize("p", [1, 2, 4])
def test_vocab_parallel_embedding_equals_lookup(p):
    V, h, T = 40, 6, 25
    E = randn(V, h)
    ids = rng.integers(0, V, size=T)
    shards = [E[i * V // p:(i + 1) * V // p] for i in range(p)]
    assert np.array_equal(O.embedding_fwd_sharded(ids, shards), O.embedding_fwd(ids, E))
    assert np.array_equal(O.embedding_fwd(ids, E)[3], E[ids[3]])


def test_embedding_bwd_by_finite_differences_and_counting():
    V, h, T = 7, 3, 12
    E, C = randn(V, h), randn(T, h)
    ids = rng.integers(0, V, size=T)
    dE = O.embedding_bwd(ids, C, V)
    _check_fd(dE, lambda: float((O.embedding_fwd(ids, E) * C).sum()), E, n=21)
    ones = O.embedding_bwd(ids, np.ones((T, 1)), V)[:, 0]
    assert np.array_equal(ones, np.bincount(ids, minlength=V).astype(float))


def test_cross_entropy_brute_force_and_closed_forms():
    T, V = 4, 5
    z = randn(T, V + 3)   # 3 padding columns
    labels = rng.integers(0, V, size=T)
    loss, g = O.cross_entropy(z, labels, V)
    for t in range(T):
        row = z[t, :V].tolist()
        ref = math.log(sum(math.exp(v) for v in row)) - row[labels[t]]
        assert abs(loss[t] - ref) < 1e-12
    assert np.all(loss >= 0)
    assert np.all(g[:, V:] == 0)
    np.testing.assert_allclose(g.sum(axis=1), 0.0, atol=1e-15)
    u, _ = O.cross_entropy(np.zeros((2, V)), [0, 3], V)
    np.testing.assert_allclose(u, math.log(V), rtol=1e-15)
    _check_fd(g, lambda: float(O.cross_entropy(z, labels, V)[0].mean()), z, n=20)


@pytest.mark.parametrize("p", [1, 2, 4])
def test_vocab_parallel_cross_entropy_equals_full(p):
    """Local max / sum / target per shard, reduced over shards, equals the
    cross-entropy on the full logits (walkthrough §6.2), padding excluded."""
    T, V = 9, 37
    Vp = O.vocab_padded(V, p, align=2)
    z = randn(T, Vp, std=3.0)
    labels = rng.integers(0, V, size=T)
    labels[0] = V - 1                      # a label in the last, padded shard
    Vs = Vp // p
    shards = [z[:, i * Vs:(i + 1) * Vs] for i in range(p)]
    loss, grads = O.cross_entropy_vocab_parallel(shards, labels, V)
    rl, rg = O.cross_entropy(z, labels, V)
    np.testing.assert_allclose(loss, rl, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(grads, axis=1), rg, rtol=1e-12, atol=1e-14)


def test_mutant_padding_included_fails_the_ce_pin():
    T, V = 6, 10
    z = randn(T, 16)
    labels = rng.integers(0, V, size=T)
    bad, _ = O.cross_entropy(z, labels, 16)   # padding columns wrongly in the softmax
    good, _ = O.cross_entropy(z, labels, V)
    assert not np.allclose(bad, good)


# ---- the attention sublayer and the pre-LN layer, by their special cases

def _attn_params(h):
    return randn(3 * h, h, std=0.5), 0.1 * randn(3 * h), randn(h, h, std=0.5), 0.1 * randn(h)


def test_attn_sublayer_one_position_passes_v_through():
    # One position per sequence: the causal softmax runs over a single score
    # and equals 1, so the attention output is V itself and the sublayer is
    # (u Wv^T + bv) Wo^T + bo, with Wv the last h rows of Wqkv.
    batch, h, H = 3, 4, 2
    u = randn(batch, h)
    Wqkv, bqkv, Wo, bo = _attn_params(h)
    a = O.attn_sublayer_fwd(u, Wqkv, bqkv, Wo, bo, batch, H)
    V = u @ Wqkv[2 * h:].T + bqkv[2 * h:]
    np.testing.assert_allclose(a["Y"], V @ Wo.T + bo, rtol=1e-12, atol=1e-12)


def test_attn_sublayer_equal_scores_average_the_values_so_far():
    # Wq = 0, bq = 0: every score is 0, so causal attention at position i is the
    # plain mean of V over positions 0..i (the diagonal included).
    batch, s, h, H = 2, 5, 4, 2
    u = randn(s * batch, h)
    Wqkv, bqkv, Wo, bo = _attn_params(h)
    Wqkv[:h] = 0.0
    bqkv[:h] = 0.0
    a = O.attn_sublayer_fwd(u, Wqkv, bqkv, Wo, bo, batch, H)
    V = (u @ Wqkv[2 * h:].T + bqkv[2 * h:]).reshape(s, batch, h)
    want = np.stack([V[:i + 1].mean(axis=0) for i in range(s)]).reshape(s * batch, h)
    np.testing.assert_allclose(a["O"], want, rtol=1e-12, atol=1e-12)


def test_attn_sublayer_is_causal():
    # Changing the tokens of the last position leaves every earlier row as it
    # was and changes the last one (rows are position-major: row = pos * batch + b).
    batch, s, h, H = 2, 4, 4, 2
    u = randn(s * batch, h)
    Wqkv, bqkv, Wo, bo = _attn_params(h)
    y0 = O.attn_sublayer_fwd(u, Wqkv, bqkv, Wo, bo, batch, H)["Y"]
    u2 = u.copy()
    u2[(s - 1) * batch:] += randn(batch, h)
    y1 = O.attn_sublayer_fwd(u2, Wqkv, bqkv, Wo, bo, batch, H)["Y"]
    np.testing.assert_allclose(y1[:(s - 1) * batch], y0[:(s - 1) * batch], rtol=0, atol=1e-14)
    assert np.abs(y1[(s - 1) * batch:] - y0[(s - 1) * batch:]).max() > 1e-3


def test_layer_fwd_zero_sublayers_are_residual_identities():
    batch, s, h, f, H = 2, 3, 4, 8, 2
    x = randn(batch * s, h)
    P = _layer_params(h, f, H)
    # both sublayers' output projections zero: each adds nothing
    Z = dict(P, Wo=np.zeros_like(P["Wo"]), bo=np.zeros_like(P["bo"]),
             W2=np.zeros_like(P["W2"]), b2=np.zeros_like(P["b2"]))
    assert np.array_equal(O.layer_fwd(x, Z, batch, H)["y"], x)
    # only the MLP zero: y = x + Attn(LN1(x))
    A = dict(P, W2=np.zeros_like(P["W2"]), b2=np.zeros_like(P["b2"]))
    u1 = O.layernorm_fwd(x, P["ln1_g"], P["ln1_b"])[0]
    att = O.attn_sublayer_fwd(u1, P["Wqkv"], P["bqkv"], P["Wo"], P["bo"], batch, H)["Y"]
    np.testing.assert_allclose(O.layer_fwd(x, A, batch, H)["y"], x + att, rtol=1e-13, atol=1e-13)
    # both on: the MLP reads LN2 of the attention's residual sum, not of x
    full = O.layer_fwd(x, P, batch, H)
    x1 = x + att
    u2 = O.layernorm_fwd(x1, P["ln2_g"], P["ln2_b"])[0]
    mlp = O.mlp_fwd(u2, P["W1"], P["b1"], P["W2"], P["b2"], "gelu")["Y"]
    np.testing.assert_allclose(full["y"], x1 + mlp, rtol=1e-13, atol=1e-13)
    wrong = O.mlp_fwd(O.layernorm_fwd(x, P["ln2_g"], P["ln2_b"])[0], P["W1"], P["b1"], P["W2"], P["b2"],
                      "gelu")["Y"]
    assert np.abs(full["y"] - (x1 + wrong)).max() > 1e-3
