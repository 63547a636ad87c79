"""Seeded synthetic inputs for the tensor-parallel MLP / attention block.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it without sharing any computation.

Every tensor is drawn on the CPU from one ``torch.Generator`` seeded with
``seed``, in the fixed order the ``draw_*`` functions list, then rounded to the
storage dtype. Callers that need the values in fp64 widen the rounded tensor,
so both sides see bit-identical inputs.

Distributions follow the workloads the pages describe (hidden/ffn/head sizes,
token counts): activations ~ N(0, 1) (the tiny fp32 MLP uses N(0, 0.02)),
weights ~ N(0, 0.02), biases ~ U(-0.1, 0.1), upstream gradients ~ N(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


def _normal(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std


def _uniform(gen: torch.Generator, shape, lo: float, hi: float) -> torch.Tensor:
    return torch.rand(*shape, generator=gen, dtype=torch.float32) * (hi - lo) + lo


@dataclass
class MLPInputs:
    """Full (unsharded) tensors of one MLP sublayer.

    Weights use the ``[out, in]`` row-major layout of ``F.linear``:
    ``W1`` is ``[f, h]`` for GELU and ``[2f, h]`` = ``[G; U]`` (gate rows
    first) for SwiGLU; ``W2`` is ``[h, f]``.
    """

    X: torch.Tensor
    W1: torch.Tensor
    W2: torch.Tensor
    b1: torch.Tensor | None
    b2: torch.Tensor | None
    dY: torch.Tensor
    act: str
    extra: dict = field(default_factory=dict)


def draw_mlp(T: int, h: int, f: int, act: str, dtype: torch.dtype, seed: int = 0,
             x_std: float = 1.0, w_std: float = 0.02, bias: bool = False,
             dy: bool = True) -> MLPInputs:
    """Draw X, W1, W2, b1, b2, dY in that order from one seeded generator."""
    if act not in ("gelu", "swiglu", "none"):
        raise ValueError(f"unknown activation {act!r}")
    gen = torch.Generator().manual_seed(seed)
    X = _normal(gen, (T, h), x_std)
    n1 = 2 * f if act == "swiglu" else f
    W1 = _normal(gen, (n1, h), w_std)
    W2 = _normal(gen, (h, f), w_std)
    b1 = _uniform(gen, (n1,), -0.1, 0.1) if bias else None
    b2 = _uniform(gen, (h,), -0.1, 0.1) if bias else None
    dY = _normal(gen, (T, h), 1.0) if dy else None
    cast = lambda t: None if t is None else t.to(dtype).contiguous()
    return MLPInputs(cast(X), cast(W1), cast(W2), cast(b1), cast(b2), cast(dY), act)


def draw_tiny_fp32_mlp(seed: int = 0) -> MLPInputs:
    """The tiny fp32 GELU MLP: X 64x128, A 128x512, B 512x128, p = 2.

    X, A, B ~ N(0, 0.02); biases ~ U(-0.1, 0.1); dY ~ N(0, 1).
    """
    return draw_mlp(64, 128, 512, "gelu", torch.float32, seed=seed, x_std=0.02,
                    w_std=0.02, bias=True)


@dataclass
class AttnBlockInputs:
    """Tensors of one attention sublayer (QKV projection, core, out-projection).

    ``Wqkv`` is ``[3h, h]`` with rows ``[Wq; Wk; Wv]``; inside each of the
    three blocks the rows of head ``j`` are ``[j*d, (j+1)*d)``. ``Wo`` is
    ``[h, h]``. Tokens are rows of ``[T, h]`` in sequence-major order:
    row ``s*batch + b``.
    """

    X: torch.Tensor
    Wqkv: torch.Tensor
    Wo: torch.Tensor
    bqkv: torch.Tensor | None
    bo: torch.Tensor | None
    dY: torch.Tensor | None


def draw_attn_block(batch: int, seq: int, h: int, dtype: torch.dtype, seed: int = 0,
                    bias: bool = False, dy: bool = False) -> AttnBlockInputs:
    """Draw X, Wqkv, Wo, bqkv, bo, dY in that order."""
    gen = torch.Generator().manual_seed(seed)
    T = batch * seq
    X = _normal(gen, (T, h), 1.0)
    Wqkv = _normal(gen, (3 * h, h), 0.02)
    Wo = _normal(gen, (h, h), 0.02)
    bqkv = _uniform(gen, (3 * h,), -0.1, 0.1) if bias else None
    bo = _uniform(gen, (h,), -0.1, 0.1) if bias else None
    dY = _normal(gen, (T, h), 1.0) if dy else None
    cast = lambda t: None if t is None else t.to(dtype).contiguous()
    return AttnBlockInputs(cast(X), cast(Wqkv), cast(Wo), cast(bqkv), cast(bo), cast(dY))


def draw_qkv_activations(batch: int, seq: int, heads: int, d: int, dtype: torch.dtype,
                         seed: int = 0, std: float = 1.0, dy: bool = True):
    """Q, K, V (and dO) for the attention core alone, each ``[seq, batch, heads*d]``."""
    gen = torch.Generator().manual_seed(seed)
    shape = (seq, batch, heads * d)
    Q = _normal(gen, shape, std)
    K = _normal(gen, shape, std)
    V = _normal(gen, shape, std)
    dO = _normal(gen, shape, 1.0) if dy else None
    cast = lambda t: None if t is None else t.to(dtype).contiguous()
    return cast(Q), cast(K), cast(V), cast(dO)


@dataclass
class LayerParams:
    """Parameters of one pre-LN transformer layer (attention + GELU MLP)."""

    ln1_g: torch.Tensor
    ln1_b: torch.Tensor
    Wqkv: torch.Tensor
    bqkv: torch.Tensor
    Wo: torch.Tensor
    bo: torch.Tensor
    ln2_g: torch.Tensor
    ln2_b: torch.Tensor
    W1: torch.Tensor
    b1: torch.Tensor
    W2: torch.Tensor
    b2: torch.Tensor


def draw_block_stack(layers: int, batch: int, seq: int, h: int, f: int, dtype: torch.dtype,
                     seed: int = 0, ln_affine_random: bool = False):
    """A stack of pre-LN layers: returns (X, [LayerParams], dY).

    LayerNorm gamma = 1 and beta = 0 unless ``ln_affine_random`` (then
    gamma ~ 1 + U(-0.1, 0.1), beta ~ U(-0.1, 0.1)), drawn per layer in
    the field order of ``LayerParams``.
    """
    gen = torch.Generator().manual_seed(seed)
    T = batch * seq
    X = _normal(gen, (T, h), 1.0)
    cast = lambda t: t.to(dtype).contiguous()
    out = []
    for _ in range(layers):
        def ln_pair():
            if ln_affine_random:
                return (cast(1.0 + _uniform(gen, (h,), -0.1, 0.1)),
                        cast(_uniform(gen, (h,), -0.1, 0.1)))
            return cast(torch.ones(h)), cast(torch.zeros(h))
        g1, be1 = ln_pair()
        Wqkv = cast(_normal(gen, (3 * h, h), 0.02))
        bqkv = cast(_uniform(gen, (3 * h,), -0.1, 0.1))
        Wo = cast(_normal(gen, (h, h), 0.02))
        bo = cast(_uniform(gen, (h,), -0.1, 0.1))
        g2, be2 = ln_pair()
        W1 = cast(_normal(gen, (f, h), 0.02))
        b1 = cast(_uniform(gen, (f,), -0.1, 0.1))
        W2 = cast(_normal(gen, (h, f), 0.02))
        b2 = cast(_uniform(gen, (h,), -0.1, 0.1))
        out.append(LayerParams(g1, be1, Wqkv, bqkv, Wo, bo, g2, be2, W1, b1, W2, b2))
    dY = cast(_normal(gen, (T, h), 1.0))
    return cast(X), out, dY


def draw_sp_mlp(seq: int, h: int, f: int, p: int, dtype: torch.dtype, seed: int = 0,
                ln_affine_random: bool = False):
    """The sequence-parallel SwiGLU MLP: X as p sequence shards, LN gamma/beta,
    W1 = [G; U], W2, dY as p sequence shards. Drawn in that order.
    """
    if seq % p:
        raise ValueError("seq must be divisible by p")
    gen = torch.Generator().manual_seed(seed)
    cast = lambda t: t.to(dtype).contiguous()
    X = _normal(gen, (seq, h), 1.0)
    if ln_affine_random:
        g = 1.0 + _uniform(gen, (h,), -0.1, 0.1)
        b = _uniform(gen, (h,), -0.1, 0.1)
    else:
        g, b = torch.ones(h), torch.zeros(h)
    W1 = _normal(gen, (2 * f, h), 0.02)
    W2 = _normal(gen, (h, f), 0.02)
    dY = _normal(gen, (seq, h), 1.0)
    return cast(X), cast(g), cast(b), cast(W1), cast(W2), cast(dY)


def draw_partials(p: int, T: int, h: int, dtype: torch.dtype, seed: int = 0,
                  integer_valued: bool = False, bias: bool = True, residual: bool = False):
    """p full-shape partials [T, h], a bias [h] and an optional residual [T, h].

    With ``integer_valued`` every value is a small integer, so every partial
    sum is exact in fp32 and bf16 and a reduction can be checked bit for bit.
    """
    gen = torch.Generator().manual_seed(seed)
    if integer_valued:
        P = [torch.randint(-8, 9, (T, h), generator=gen).float() for _ in range(p)]
        b = torch.randint(-8, 9, (h,), generator=gen).float() if bias else None
        r = torch.randint(-8, 9, (T, h), generator=gen).float() if residual else None
    else:
        P = [_normal(gen, (T, h), 1.0) for _ in range(p)]
        b = _uniform(gen, (h,), -0.1, 0.1) if bias else None
        r = _normal(gen, (T, h), 1.0) if residual else None
    cast = lambda t: None if t is None else t.to(dtype).contiguous()
    return [cast(x) for x in P], cast(b), cast(r)


def sample_rows(n_total: int, n_sample: int, seed: int = 1234) -> torch.Tensor:
    """A fixed, sorted, seeded sample of row indices (always includes the last row)."""
    gen = torch.Generator().manual_seed(seed)
    if n_sample >= n_total:
        return torch.arange(n_total)
    idx = torch.randperm(n_total, generator=gen)[: n_sample - 1]
    idx = torch.cat([idx, torch.tensor([n_total - 1])])
    return torch.sort(torch.unique(idx)).values
