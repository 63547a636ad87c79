"""Plain, slow, fp64 CPU oracle for the Megatron tensor-parallel block.

TEST INFRASTRUCTURE ONLY: ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py`` use it; the CUDA path shares no code with it.

Everything here is fp64 numpy. Inputs arrive already rounded to their storage
dtype (bf16 or fp32) and are widened exactly; nothing is rounded in between,
so each function is the exact definition of what the sharded method computes
(the pages state that the split reaches the unsplit result).

Sources (web pages on tensor parallelism; cited by title and section):
  [TP-blog]  "企业官网建设流程全解析" (2kiu.com/news/5653011), a long TP walkthrough:
             §2.1 column parallel, §2.2 row parallel, §2.3 pairing,
             §3.1 attention by heads, §3.2 MLP / gate+up, §3.3 normalisation,
             §4.1 collectives, §4.3 sequence parallelism, §6.1 divisibility.
  [TP-wiki]  "张量并行" (ai-infra-wiki), sections 两种切法 (MLP equations
             Y = GELU(XA)B, XA = [XA_1, XA_2], XB = X_1B_1 + X_2B_2) and
             序列维度的补充：Megatron-SP.
  [TP-scratch] "大模型分布式训练篇——从零实现 Tensor Parallel" (makesence),
             §四 (f/g conjugates: identity forward / all-reduce backward).
  [TP-basics] "Tensor Parallelism基础：模型切分原理" (bjdmk), 实现细节 section:
             F.linear weight layout [out, in], row bias added once after the sum.

Readings where the pages are silent (each also listed in the design notes):
  * GELU is the exact erf form; SwiGLU is H = SiLU(gate) * up with the shard
    buffer [G_i; U_i] (gate rows first).
  * Weights are stored [out, in] (F.linear layout) and the layer computes X W^T.
  * Column bias is sharded with its columns; row bias is added once after the sum.
  * Tokens are rows of [T, h] in sequence-major order (row = s*batch + b), so a
    sequence shard is a contiguous block of rows.
  * LayerNorm: biased variance over the full hidden dim, eps = 1e-5, affine.
  * Attention: scale 1/sqrt(d), causal mask j <= i, softmax per row, no dropout.
  * Layers are pre-LN: x += Attn(LN1(x)); x += MLP(LN2(x)).
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "f64", "gelu", "gelu_grad", "silu", "silu_grad", "linear",
    "mlp_fwd", "mlp_bwd", "mlp_fwd_rows", "mlp_bwd_sampled",
    "shard_rows", "shard_cols", "shard_vec", "shard_gate_up", "shard_gate_up_vec",
    "shard_qkv", "shard_qkv_vec",
    "column_fwd_shard", "row_partial", "reduce_partials", "reduce_scatter_seq",
    "all_gather_seq", "row_bwd_shard", "column_bwd_shard", "bias_grad",
    "attention_fwd", "attention_fwd_rows", "attention_bwd", "layernorm_fwd", "layernorm_bwd",
    "attn_sublayer_fwd", "attn_sublayer_bwd", "layer_fwd", "layer_bwd",
    "sp_mlp_fwd", "sp_mlp_bwd", "max_row_rel_err", "LN_EPS",
    "rmsnorm_fwd", "rmsnorm_bwd", "norm_sharded_fwd", "norm_sharded_bwd",
    "vocab_padded", "embedding_fwd", "embedding_fwd_sharded", "embedding_bwd",
    "cross_entropy", "cross_entropy_vocab_parallel",
]

LN_EPS = 1e-5


def f64(t) -> np.ndarray:
    """Widen a torch tensor (any float dtype) or array to an fp64 numpy array."""
    if t is None:
        return None
    if hasattr(t, "detach"):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


# ---------------------------------------------------------------------------
# Element-wise activations. [TP-wiki] 两种切法: Y = GELU(XA)B; [TP-blog] §3.2
# names the SwiGLU gate/up two-branch MLP.
# ---------------------------------------------------------------------------

def gelu(z):
    """GELU(z) = z * Phi(z) with Phi the standard normal CDF (exact erf form)."""
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def gelu_grad(z):
    """d/dz GELU(z) = Phi(z) + z * phi(z)."""
    return 0.5 * (1.0 + _erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def silu(z):
    """SiLU(z) = z * sigmoid(z)."""
    return z / (1.0 + np.exp(-z))


def silu_grad(z):
    """d/dz SiLU(z) = s(z) * (1 + z * (1 - s(z))), s the logistic sigmoid."""
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def linear(X, W, b=None):
    """F.linear: X [T, in] times W [out, in] transposed, plus b [out] if given.

    [TP-basics] 实现细节: the weight chunk is stored [out, in] and the layer
    computes x @ w^T; [TP-blog] §2 writes the same product as X W with W [in, out].
    """
    Y = X @ W.T
    if b is not None:
        Y = Y + b[None, :]
    return Y


# ---------------------------------------------------------------------------
# Unsharded MLP: the plain definition the sharded method reaches.
# [TP-wiki] 两种切法: Y = GELU(X A) B; [TP-blog] §3.2 (gate/up SwiGLU variant).
# ---------------------------------------------------------------------------

def mlp_fwd(X, W1, b1, W2, b2, act, residual=None):
    """Z = X W1^T + b1; H = act(Z); Y = H W2^T + b2 (+ residual).

    For act == "swiglu", W1 = [G; U] ([2f, h], gate rows first), b1 must be
    None, Z = [Zg | Zu] ([T, 2f]) and H = SiLU(Zg) * Zu.
    """
    Z = linear(X, W1, b1)
    if act == "gelu":
        H = gelu(Z)
    elif act == "swiglu":
        f = W1.shape[0] // 2
        H = silu(Z[:, :f]) * Z[:, f:]
    elif act == "none":
        H = Z
    else:
        raise ValueError(act)
    Y = linear(H, W2, b2)
    if residual is not None:
        Y = Y + residual
    return {"Z": Z, "H": H, "Y": Y}


def mlp_bwd(X, W1, W2, Z, H, dY, act):
    """Chain rule through mlp_fwd. Returns dH, dZ, dX, dW1, db1, dW2, db2.

    dH = dY W2; GELU: dZ = dH * GELU'(Z); SwiGLU: dZg = dH * Zu * SiLU'(Zg),
    dZu = dH * SiLU(Zg); dW1 = dZ^T X; db1 = sum_t dZ; dX = dZ W1;
    dW2 = dY^T H; db2 = sum_t dY. [TP-scratch] §四 gives the backward
    communication that pairs with this (dX is the sum over shards).
    """
    dH = dY @ W2
    if act == "gelu":
        dZ = dH * gelu_grad(Z)
    elif act == "swiglu":
        f = W1.shape[0] // 2
        Zg, Zu = Z[:, :f], Z[:, f:]
        dZ = np.concatenate([dH * Zu * silu_grad(Zg), dH * silu(Zg)], axis=1)
    elif act == "none":
        dZ = dH
    else:
        raise ValueError(act)
    return {
        "dH": dH, "dZ": dZ, "dX": dZ @ W1, "dW1": dZ.T @ X, "db1": dZ.sum(axis=0),
        "dW2": dY.T @ H, "db2": dY.sum(axis=0),
    }


def mlp_fwd_rows(X, W1, b1, W2, b2, act, rows):
    """mlp_fwd restricted to token rows ``rows`` (every output row is row-local)."""
    return mlp_fwd(X[rows], W1, b1, W2, b2, act)


def mlp_bwd_sampled(X, W1, b1, W2, dY, act, rows, fcols):
    """Exact samples of the MLP gradients, computed from their definitions.

    dX[rows] (row-local); for the sampled hidden-unit indices ``fcols`` of the
    intermediate dim: dW2[:, fcols], dW1 rows of those units (for SwiGLU both
    the gate row j and the up row f + j), db1 of those units (GELU only).
    Each sampled column needs the intermediate activations of that unit over
    all T tokens, which are computed here from X, W1, W2 and dY.
    """
    out = {}
    fwd = mlp_fwd(X[rows], W1, b1, W2, None, act)
    out["dX_rows"] = mlp_bwd(X[rows], W1, W2, fwd["Z"], fwd["H"], dY[rows], act)["dX"]
    f = W2.shape[1]
    fcols = np.asarray(fcols)
    dHc = dY @ W2[:, fcols]                       # [T, k]
    if act == "gelu":
        Zc = linear(X, W1[fcols], None if b1 is None else b1[fcols])
        Hc = gelu(Zc)
        dZc = dHc * gelu_grad(Zc)
        out["dW1_rows"] = dZc.T @ X               # rows fcols of dW1
        out["db1"] = dZc.sum(axis=0)
        out["W1_rows_index"] = fcols
    else:
        Zg = linear(X, W1[fcols])
        Zu = linear(X, W1[f + fcols])
        Hc = silu(Zg) * Zu
        dZg = dHc * Zu * silu_grad(Zg)
        dZu = dHc * silu(Zg)
        out["dW1_rows"] = np.concatenate([dZg.T @ X, dZu.T @ X], axis=0)
        out["W1_rows_index"] = np.concatenate([fcols, f + fcols])
    out["dW2_cols"] = dY.T @ Hc                   # columns fcols of dW2
    out["db2"] = dY.sum(axis=0)
    return out


# ---------------------------------------------------------------------------
# Sharding. [TP-blog] §2.1 (column: output-dim blocks), §2.2 (row: input-dim
# blocks), §3.1 (QKV by whole heads), §3.2 (gate and up share one column
# shard; the intermediate dim must divide by p), §6.1 (divisibility).
# ---------------------------------------------------------------------------

def _check_div(n, p, what):
    if n % p:
        raise ValueError(f"{what}={n} is not divisible by p={p}")


def shard_rows(W, p, i):
    """Column-parallel shard i of an [out, in] weight: rows [i*out/p, (i+1)*out/p)."""
    _check_div(W.shape[0], p, "out")
    n = W.shape[0] // p
    return W[i * n:(i + 1) * n, :]


def shard_cols(W, p, i):
    """Row-parallel shard i of an [out, in] weight: columns [i*in/p, (i+1)*in/p)."""
    _check_div(W.shape[1], p, "in")
    k = W.shape[1] // p
    return W[:, i * k:(i + 1) * k]


def shard_vec(b, p, i):
    """Shard i of a column bias: entries [i*n/p, (i+1)*n/p)."""
    _check_div(b.shape[0], p, "len")
    n = b.shape[0] // p
    return b[i * n:(i + 1) * n]


def shard_gate_up(W1, p, i):
    """[G_i; U_i] for W1 = [G; U] ([2f, h]): gate rows i*f/p.. and the same up rows.

    [TP-blog] §3.2: gate and up are concatenated into one larger projection, and
    every shard must hold an equal, matching piece of the intermediate dim.
    """
    f = W1.shape[0] // 2
    _check_div(f, p, "ffn")
    k = f // p
    return np.concatenate([W1[i * k:(i + 1) * k], W1[f + i * k:f + (i + 1) * k]], axis=0)


def shard_gate_up_vec(b1, p, i):
    """The column bias of shard i of a SwiGLU MLP, paired like its weight rows:
    [b_gate entries i*f/p.., b_up entries i*f/p..] for b1 = [b_gate; b_up] ([2f])."""
    f = b1.shape[0] // 2
    _check_div(f, p, "ffn")
    k = f // p
    return np.concatenate([b1[i * k:(i + 1) * k], b1[f + i * k:f + (i + 1) * k]])


def shard_qkv(Wqkv, heads, p, i):
    """[Q_i; K_i; V_i] rows of whole heads i*H/p..(i+1)*H/p from each of Wq, Wk, Wv.

    [TP-blog] §3.1: the QKV projection is split along the attention heads; each
    shard owns heads/p complete heads (heads must divide by p).
    """
    h = Wqkv.shape[0] // 3
    _check_div(heads, p, "heads")
    _check_div(h, heads, "hidden/heads")
    d = h // heads
    hl = heads // p
    r0, r1 = i * hl * d, (i + 1) * hl * d
    return np.concatenate([Wqkv[r0:r1], Wqkv[h + r0:h + r1], Wqkv[2 * h + r0:2 * h + r1]], axis=0)


def shard_qkv_vec(bqkv, heads, p, i):
    h = bqkv.shape[0] // 3
    d = h // heads
    hl = heads // p
    r0, r1 = i * hl * d, (i + 1) * hl * d
    return np.concatenate([bqkv[r0:r1], bqkv[h + r0:h + r1], bqkv[2 * h + r0:2 * h + r1]])


# ---------------------------------------------------------------------------
# The sharded path, step by step, as the pages describe it.
# ---------------------------------------------------------------------------

def column_fwd_shard(X, W_i, b_i, act):
    """Shard i of the column-parallel GEMM with its activation.

    [TP-blog] §2.1 / [TP-wiki] 两种切法 (XA = [XA_1, XA_2], no communication):
    Z_i = X W_i^T + b_i; H_i = act(Z_i). For SwiGLU W_i = [G_i; U_i] and
    Z_i = [Zg_i | Zu_i], H_i = SiLU(Zg_i) * Zu_i.
    """
    Z = linear(X, W_i, b_i)
    if act == "gelu":
        H = gelu(Z)
    elif act == "swiglu":
        k = W_i.shape[0] // 2
        H = silu(Z[:, :k]) * Z[:, k:]
    elif act == "none":
        H = Z
    else:
        raise ValueError(act)
    return Z, H


def row_partial(H_i, W2_i):
    """Shard i of the row-parallel GEMM: the full-shape partial H_i W2_i^T, no bias.

    [TP-blog] §2.2 / [TP-wiki] 两种切法 (XB = X_1B_1 + X_2B_2): every shard
    holds a partial of the complete output shape.
    """
    return H_i @ W2_i.T


def reduce_partials(P, bias=None, residual=None):
    """Sum of the p partials in order 0..p-1, then the bias once, then the residual.

    [TP-blog] §2.2 (element-wise sum of the partials, all-reduce SUM);
    [TP-basics] 实现细节 (the row bias is added once, after the sum).
    """
    Y = np.zeros_like(P[0])
    for Pi in P:
        Y = Y + Pi
    if bias is not None:
        Y = Y + bias[None, :]
    if residual is not None:
        Y = Y + residual
    return Y


def reduce_scatter_seq(P, bias=None, residual_shards=None):
    """Reduce-scatter along the sequence: shard j gets rows [j*T/p, (j+1)*T/p) of the sum.

    [TP-blog] §4.3 / [TP-wiki] Megatron-SP: the row-parallel all-reduce becomes a
    reduce-scatter over the sequence dim. n = len(P) output shards.
    """
    n = len(P)
    T = P[0].shape[0]
    _check_div(T, n, "T")
    t = T // n
    Y = reduce_partials(P, bias)
    out = []
    for j in range(n):
        Yj = Y[j * t:(j + 1) * t]
        if residual_shards is not None:
            Yj = Yj + residual_shards[j]
        out.append(Yj)
    return out


def all_gather_seq(X_seq):
    """All-gather along the sequence: concatenate the p row blocks in order.

    [TP-blog] §4.3 (all-gather before the next column GEMM), [TP-wiki] Megatron-SP.
    """
    return np.concatenate(list(X_seq), axis=0)


def row_bwd_shard(dY, H_i, W2_i, Z_i, act):
    """Backward of shard i of the row-parallel layer (input grad needs no sum).

    [TP-scratch] §四: the row layer's forward sums, so its backward is the
    identity on dY (replicated); each shard computes dH_i = dY W2_i, then the
    activation's derivative gives dZ_i, and dW2_i = dY^T H_i.
    """
    dH = dY @ W2_i
    if act == "gelu":
        dZ = dH * gelu_grad(Z_i)
    elif act == "swiglu":
        k = Z_i.shape[1] // 2
        Zg, Zu = Z_i[:, :k], Z_i[:, k:]
        dZ = np.concatenate([dH * Zu * silu_grad(Zg), dH * silu(Zg)], axis=1)
    elif act == "none":
        dZ = dH
    else:
        raise ValueError(act)
    return dZ, dY.T @ H_i


def column_bwd_shard(X, dZ_i, W_i):
    """Backward of shard i of the column-parallel layer.

    [TP-scratch] §四: the column layer's forward is the identity on X, so its
    backward sums the input gradient over shards: this returns shard i's
    partial dX_i = dZ_i W_i (to be reduced), dW_i = dZ_i^T X, db_i = sum_t dZ_i.
    """
    return dZ_i.T @ X, dZ_i.sum(axis=0), dZ_i @ W_i


def bias_grad(dY):
    """Column sums over tokens (the gradient of a bias added to every row)."""
    return dY.sum(axis=0)


# ---------------------------------------------------------------------------
# Attention core on local heads. [TP-blog] §3.1: each shard runs full-sequence
# attention on its own heads with no cross-shard step.
# ---------------------------------------------------------------------------

def _split_heads(A, batch, heads):
    """[s, b, H*d] (or [s*b, H*d]) -> [b, H, s, d]."""
    A = np.asarray(A)
    s = A.shape[0] if A.ndim == 3 else A.shape[0] // batch
    A = A.reshape(s, batch, heads, -1)
    return A.transpose(1, 2, 0, 3)


def _merge_heads(A):
    """[b, H, s, d] -> [s, b, H*d]."""
    b, H, s, d = A.shape
    return A.transpose(2, 0, 1, 3).reshape(s, b, H * d)


def attention_fwd(Q, K, V, batch, heads, causal=True):
    """O = softmax(Q K^T / sqrt(d) + mask) V per (batch, head).

    Inputs [s, batch, heads*d] (sequence-major tokens). Returns O [s, batch,
    heads*d] and the row log-sum-exp of the scaled, masked scores [batch, heads, s].
    """
    q, k, v = (_split_heads(a, batch, heads) for a in (Q, K, V))
    d = q.shape[-1]
    S = np.matmul(q, k.swapaxes(-1, -2)) / math.sqrt(d)
    s = S.shape[-1]
    if causal:
        mask = np.triu(np.ones((s, s), dtype=bool), k=1)
        S = np.where(mask[None, None], -np.inf, S)
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    L = E.sum(axis=-1, keepdims=True)
    P = E / L
    O = np.matmul(P, v)
    lse = (m + np.log(L))[..., 0]
    return _merge_heads(O), lse


def attention_fwd_rows(Q, K, V, batch, heads, rows, causal=True):
    """attention_fwd restricted to the query positions ``rows`` (each output row
    depends only on its own query and the keys it may see).

    Returns O [len(rows), batch, heads*d] and lse [batch, heads, len(rows)].
    """
    q, k, v = (_split_heads(a, batch, heads) for a in (Q, K, V))
    d = q.shape[-1]
    rows = np.asarray(rows)
    S = np.matmul(q[:, :, rows], k.swapaxes(-1, -2)) / math.sqrt(d)
    if causal:
        mask = np.arange(k.shape[2])[None, :] > rows[:, None]
        S = np.where(mask[None, None], -np.inf, S)
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    L = E.sum(axis=-1, keepdims=True)
    O = np.matmul(E / L, v)
    return _merge_heads(O), (m + np.log(L))[..., 0]


def attention_bwd(Q, K, V, dO, batch, heads, causal=True):
    """Gradients of attention_fwd: dQ, dK, dV (each [s, batch, heads*d]).

    dV = P^T dO; dP = dO V^T; dS = P * (dP - rowsum(dO * O)); dQ = dS K / sqrt(d);
    dK = dS^T Q / sqrt(d).
    """
    q, k, v, do = (_split_heads(a, batch, heads) for a in (Q, K, V, dO))
    d = q.shape[-1]
    S = np.matmul(q, k.swapaxes(-1, -2)) / math.sqrt(d)
    s = S.shape[-1]
    if causal:
        mask = np.triu(np.ones((s, s), dtype=bool), k=1)
        S = np.where(mask[None, None], -np.inf, S)
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    P = E / E.sum(axis=-1, keepdims=True)
    O = np.matmul(P, v)
    dV = np.matmul(P.swapaxes(-1, -2), do)
    dP = np.matmul(do, v.swapaxes(-1, -2))
    Dr = (do * O).sum(axis=-1, keepdims=True)
    dS = P * (dP - Dr)
    dQ = np.matmul(dS, k) / math.sqrt(d)
    dK = np.matmul(dS.swapaxes(-1, -2), q) / math.sqrt(d)
    return _merge_heads(dQ), _merge_heads(dK), _merge_heads(dV)


# ---------------------------------------------------------------------------
# LayerNorm on the full hidden dim. [TP-blog] §3.3: the statistics must span
# the whole hidden dim; with sequence parallelism it runs per sequence shard
# ([TP-blog] §4.3, [TP-wiki] Megatron-SP).
# ---------------------------------------------------------------------------

def layernorm_fwd(x, g, b, eps=LN_EPS):
    """y = (x - mean) / sqrt(var + eps) * g + b per row; biased variance."""
    mean = x.mean(axis=1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (x - mean) * rstd
    return xhat * g[None, :] + b[None, :], mean[:, 0], rstd[:, 0]


def layernorm_bwd(x, g, dy, mean, rstd):
    """dx, dg, db of layernorm_fwd.

    With xhat = (x - mean) * rstd and gy = dy * g:
    dx = rstd * (gy - mean_row(gy) - xhat * mean_row(gy * xhat));
    dg = sum_rows dy * xhat; db = sum_rows dy.
    """
    xhat = (x - mean[:, None]) * rstd[:, None]
    gy = dy * g[None, :]
    dx = rstd[:, None] * (gy - gy.mean(axis=1, keepdims=True)
                          - xhat * (gy * xhat).mean(axis=1, keepdims=True))
    return dx, (dy * xhat).sum(axis=0), dy.sum(axis=0)


def rmsnorm_fwd(x, g, eps=LN_EPS):
    """y = x / sqrt(mean(x^2) + eps) * g per row (RMSNorm over the full hidden dim)."""
    rstd = 1.0 / np.sqrt((x * x).mean(axis=1, keepdims=True) + eps)
    return x * rstd * g[None, :], rstd[:, 0]


def rmsnorm_bwd(x, g, dy, rstd):
    """dx, dg of rmsnorm_fwd: with xhat = x * rstd and gy = dy * g,
    dx = rstd * (gy - xhat * mean_row(gy * xhat)); dg = sum_rows dy * xhat."""
    xhat = x * rstd[:, None]
    gy = dy * g[None, :]
    dx = rstd[:, None] * (gy - xhat * (gy * xhat).mean(axis=1, keepdims=True))
    return dx, (dy * xhat).sum(axis=0)


def norm_sharded_fwd(x_shards, g_shards, b_shards, kind):
    """LayerNorm / RMSNorm whose input is split over the hidden dim, the way
    [TP-blog] §3.3 describes: every shard forms its local sums (sum x and
    sum x^2 for LayerNorm, sum x^2 for RMSNorm), the per-row scalars are summed
    over shards, and the resulting statistics normalise each shard's slice.
    Returns the output shards and (mean, rstd) (mean is None for RMSNorm)."""
    h = sum(xs.shape[1] for xs in x_shards)
    s2 = sum((xs * xs).sum(axis=1) for xs in x_shards)
    if kind == "rms":
        rstd = 1.0 / np.sqrt(s2 / h + LN_EPS)
        return [xs * rstd[:, None] * gs[None, :] for xs, gs in zip(x_shards, g_shards)], (None, rstd)
    s1 = sum(xs.sum(axis=1) for xs in x_shards)
    mean = s1 / h
    var = s2 / h - mean * mean
    rstd = 1.0 / np.sqrt(var + LN_EPS)
    return ([(xs - mean[:, None]) * rstd[:, None] * gs[None, :] + bs[None, :]
             for xs, gs, bs in zip(x_shards, g_shards, b_shards)], (mean, rstd))


def norm_sharded_bwd(x_shards, g_shards, dy_shards, stats, kind):
    """Backward of norm_sharded_fwd: the two per-row means of the backward
    (of gy and of gy * xhat) are again local sums reduced over shards.
    Returns dx shards and dg (and db for LayerNorm) shards."""
    mean, rstd = stats
    h = sum(xs.shape[1] for xs in x_shards)
    xh = [(xs if mean is None else xs - mean[:, None]) * rstd[:, None] for xs in x_shards]
    gy = [dys * gs[None, :] for dys, gs in zip(dy_shards, g_shards)]
    m2 = sum((a * b).sum(axis=1) for a, b in zip(gy, xh)) / h
    if kind == "rms":
        dx = [rstd[:, None] * (a - b * m2[:, None]) for a, b in zip(gy, xh)]
        return dx, [(d * b).sum(axis=0) for d, b in zip(dy_shards, xh)], None
    m1 = sum(a.sum(axis=1) for a in gy) / h
    dx = [rstd[:, None] * (a - m1[:, None] - b * m2[:, None]) for a, b in zip(gy, xh)]
    return (dx, [(d * b).sum(axis=0) for d, b in zip(dy_shards, xh)],
            [d.sum(axis=0) for d in dy_shards])


# ---------------------------------------------------------------------------
# Vocab-parallel embedding and cross-entropy. [TP-blog] §6.2: the vocab dim is
# split over shards, padded up to a size the split divides; the output head
# computes only its own vocab slice of the logits and its partial loss, and the
# partials are reduced instead of gathering the full logits. [TP-wiki] 工程实践
# (vocab-parallel embedding).
# ---------------------------------------------------------------------------

def vocab_padded(vocab, p, align=8):
    """Smallest padded vocab >= vocab whose p shards each hold a multiple of
    `align` rows (the split must divide it; the alignment keeps shard rows at
    16-byte multiples for bf16)."""
    unit = p * align
    return ((vocab + unit - 1) // unit) * unit


def embedding_fwd(ids, E):
    """Y[t] = E[ids[t]]: the plain definition of the lookup."""
    return E[np.asarray(ids)]


def embedding_fwd_sharded(ids, E_shards):
    """The vocab-parallel lookup: shard i holds rows [i*Vs, (i+1)*Vs) and
    returns the row for tokens in its range and zeros otherwise; the sum over
    shards (the all-reduce) gives the lookup."""
    ids = np.asarray(ids)
    Vs = E_shards[0].shape[0]
    parts = []
    for i, Ei in enumerate(E_shards):
        loc = ids - i * Vs
        own = (loc >= 0) & (loc < Vs)
        part = np.zeros((len(ids), Ei.shape[1]))
        part[own] = Ei[loc[own]]
        parts.append(part)
    return reduce_partials(parts)


def embedding_bwd(ids, dY, vocab_rows):
    """dE[v] = sum over tokens t with ids[t] == v of dY[t]."""
    dE = np.zeros((vocab_rows, dY.shape[1]))
    for t, v in enumerate(np.asarray(ids)):
        dE[v] += dY[t]
    return dE


def cross_entropy(logits, labels, vocab):
    """Per-token loss log(sum_v exp(z_v)) - z_label over the first `vocab`
    columns (padding columns excluded), and d(mean loss)/d logits =
    (softmax - onehot) / T (zero on padding columns)."""
    z = logits[:, :vocab]
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    S = e.sum(axis=1, keepdims=True)
    labels = np.asarray(labels)
    T = z.shape[0]
    loss = (np.log(S) + m)[:, 0] - z[np.arange(T), labels]
    g = np.zeros_like(logits)
    g[:, :vocab] = e / S
    g[np.arange(T), labels] -= 1.0
    return loss, g / T


def cross_entropy_vocab_parallel(logit_shards, labels, vocab):
    """The pages' way: every shard forms its local row max, its local sum of
    exp(z - local max) over its real (non-padding) columns and, if it owns the
    label, the target logit; the per-row scalars are reduced over shards
    (max, rescaled sum, target). Returns per-token loss and per-shard gradients
    of the mean loss."""
    labels = np.asarray(labels)
    Vs = logit_shards[0].shape[1]
    T = logit_shards[0].shape[0]
    ms, ss, zt = [], [], np.zeros(T)
    for i, Li in enumerate(logit_shards):
        real = max(0, min(Vs, vocab - i * Vs))
        zi = Li[:, :real]
        mi = zi.max(axis=1) if real > 0 else np.full(T, -np.inf)
        si = np.exp(zi - mi[:, None]).sum(axis=1) if real > 0 else np.zeros(T)
        ms.append(mi)
        ss.append(si)
        loc = labels - i * Vs
        own = (loc >= 0) & (loc < real)
        zt[own] = Li[np.arange(T)[own], loc[own]]
    m = np.max(np.stack(ms), axis=0)
    S = sum(si * np.exp(mi - m) for mi, si in zip(ms, ss))
    lse = np.log(S) + m
    loss = lse - zt
    grads = []
    for i, Li in enumerate(logit_shards):
        real = max(0, min(Vs, vocab - i * Vs))
        g = np.zeros_like(Li)
        g[:, :real] = np.exp(Li[:, :real] - lse[:, None])
        loc = labels - i * Vs
        own = (loc >= 0) & (loc < real)
        g[np.arange(T)[own], loc[own]] -= 1.0
        grads.append(g / T)
    return loss, grads


# ---------------------------------------------------------------------------
# Attention sublayer and a pre-LN layer (the 12-layer stack), unsharded.
# [TP-blog] §3.1 (QKV column-parallel by heads, local attention, out-projection
# row-parallel followed by the sum), §3.2 (MLP), §3.3 (LayerNorm).
# ---------------------------------------------------------------------------

def attn_sublayer_fwd(u, Wqkv, bqkv, Wo, bo, batch, heads, causal=True):
    """QKV = u Wqkv^T + bqkv; O = attention(Q, K, V); Y = O Wo^T + bo."""
    h = Wqkv.shape[1]
    QKV = linear(u, Wqkv, bqkv)
    T = u.shape[0]
    s = T // batch
    Q = QKV[:, :h].reshape(s, batch, h)
    K = QKV[:, h:2 * h].reshape(s, batch, h)
    V = QKV[:, 2 * h:].reshape(s, batch, h)
    O, lse = attention_fwd(Q, K, V, batch, heads, causal)
    O2 = O.reshape(T, h)
    return {"QKV": QKV, "O": O2, "lse": lse, "Y": linear(O2, Wo, bo)}


def attn_sublayer_bwd(u, Wqkv, Wo, fwd, dY, batch, heads, causal=True):
    h = Wqkv.shape[1]
    T = u.shape[0]
    s = T // batch
    QKV = fwd["QKV"]
    dO = (dY @ Wo).reshape(s, batch, h)
    dWo = dY.T @ fwd["O"]
    dbo = dY.sum(axis=0)
    Q = QKV[:, :h].reshape(s, batch, h)
    K = QKV[:, h:2 * h].reshape(s, batch, h)
    V = QKV[:, 2 * h:].reshape(s, batch, h)
    dQ, dK, dV = attention_bwd(Q, K, V, dO, batch, heads, causal)
    dQKV = np.concatenate([dQ.reshape(T, h), dK.reshape(T, h), dV.reshape(T, h)], axis=1)
    return {"du": dQKV @ Wqkv, "dWqkv": dQKV.T @ u, "dbqkv": dQKV.sum(axis=0),
            "dWo": dWo, "dbo": dbo, "dQKV": dQKV, "dO": dO.reshape(T, h)}


def layer_fwd(x, P, batch, heads, causal=True):
    """Pre-LN layer: x1 = x + Attn(LN1(x)); y = x1 + MLP_gelu(LN2(x1)).

    ``P`` maps field names of a LayerParams to fp64 arrays.
    """
    u1, m1, r1 = layernorm_fwd(x, P["ln1_g"], P["ln1_b"])
    a = attn_sublayer_fwd(u1, P["Wqkv"], P["bqkv"], P["Wo"], P["bo"], batch, heads, causal)
    x1 = x + a["Y"]
    u2, m2, r2 = layernorm_fwd(x1, P["ln2_g"], P["ln2_b"])
    m = mlp_fwd(u2, P["W1"], P["b1"], P["W2"], P["b2"], "gelu")
    y = x1 + m["Y"]
    return {"x": x, "u1": u1, "m1": m1, "r1": r1, "attn": a, "x1": x1,
            "u2": u2, "m2": m2, "r2": r2, "mlp": m, "y": y}


def layer_bwd(cache, P, dy, batch, heads, causal=True):
    """Gradients of layer_fwd with respect to x and every parameter."""
    g = {}
    mb = mlp_bwd(cache["u2"], P["W1"], P["W2"], cache["mlp"]["Z"], cache["mlp"]["H"], dy, "gelu")
    g.update(dW1=mb["dW1"], db1=mb["db1"], dW2=mb["dW2"], db2=mb["db2"])
    du2 = mb["dX"]
    dx1_ln, g["dln2_g"], g["dln2_b"] = layernorm_bwd(cache["x1"], P["ln2_g"], du2, cache["m2"], cache["r2"])
    dx1 = dy + dx1_ln
    ab = attn_sublayer_bwd(cache["u1"], P["Wqkv"], P["Wo"], cache["attn"], dx1, batch, heads, causal)
    g.update(dWqkv=ab["dWqkv"], dbqkv=ab["dbqkv"], dWo=ab["dWo"], dbo=ab["dbo"])
    dx_ln, g["dln1_g"], g["dln1_b"] = layernorm_bwd(cache["x"], P["ln1_g"], ab["du"], cache["m1"], cache["r1"])
    g["dx"] = dx1 + dx_ln
    return g


# ---------------------------------------------------------------------------
# Sequence-parallel SwiGLU MLP. [TP-blog] §4.3, [TP-wiki] Megatron-SP:
# LN on sequence shards -> all-gather(seq) -> column GEMM -> row GEMM ->
# reduce-scatter(seq). The result equals the unsharded LN -> MLP.
# ---------------------------------------------------------------------------

def sp_mlp_fwd(X, g, b, W1, W2):
    """Unsharded definition of the SP sublayer: Y = MLP_swiglu(LN(X)) (no biases)."""
    u, mean, rstd = layernorm_fwd(X, g, b)
    m = mlp_fwd(u, W1, None, W2, None, "swiglu")
    return {"u": u, "mean": mean, "rstd": rstd, **m}


def sp_mlp_bwd(X, g, W1, W2, fwd, dY):
    mb = mlp_bwd(fwd["u"], W1, W2, fwd["Z"], fwd["H"], dY, "swiglu")
    dX, dg, db = layernorm_bwd(X, g, mb["dX"], fwd["mean"], fwd["rstd"])
    return {**mb, "du": mb["dX"], "dX": dX, "dg": dg, "db": db}


# ---------------------------------------------------------------------------
# The comparison metric used by the parity tests.
# ---------------------------------------------------------------------------

def max_row_rel_err(got, ref):
    """max over rows of (max_j |got - ref|) / (max_j |ref|): the error of each row
    normalised by that row's largest magnitude. Rows of ref that are all zero
    compare absolutely."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.shape != ref.shape:
        raise ValueError(f"shape mismatch {got.shape} vs {ref.shape}")
    if got.ndim == 1:
        got, ref = got[None, :], ref[None, :]
    got = got.reshape(got.shape[0], -1)
    ref = ref.reshape(ref.shape[0], -1)
    if not np.all(np.isfinite(got)):
        return float("inf")
    num = np.abs(got - ref).max(axis=1)
    den = np.abs(ref).max(axis=1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max()) if num.size else 0.0
