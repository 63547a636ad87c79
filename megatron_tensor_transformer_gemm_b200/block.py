"""Call sequences of the tensor-parallel sublayers on one GPU.

Buffers are torch CUDA tensors (device memory only); every step is one or
more libtp.so calls. Shard i of every layer is a separate buffer, as it would
be a separate rank's memory; the "collectives" are the library's local
reduce / reduce-scatter / all-gather kernels.

  TPMLP      column GEMM (+bias, GELU or SwiGLU) -> row GEMM partials ->
             reduce (+bias once); backward: row bwd (act' fused) -> column bwd
             -> reduce of the dX partials.       (TP walkthrough §2-§3.2, §四 of
             "从零实现 Tensor Parallel" for the backward pairing)
  TPAttention  QKV column GEMM (by whole heads) -> causal attention on local
             heads -> out-projection partials -> reduce (+bias, +residual), and
             its backward.                         (TP walkthrough §3.1)
  TPLayer    pre-LN layer: x1 = x + Attn(LN1(x)); y = x1 + MLP(LN2(x1)).
  SPMLP      Megatron-SP: LN on sequence shards fused with the all-gather ->
             column -> row -> reduce-scatter; backward: all-gather of dY ->
             row bwd -> column bwd -> reduce-scatter of dX partials -> LN bwd
             per shard.                            (TP walkthrough §4.3, wiki Megatron-SP)
"""
from __future__ import annotations

import torch

from .tp import Plan, backward_join


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


class TPMLP:
    """One MLP sublayer split over p shards that all live on ``device``."""

    def __init__(self, hidden: int, ffn: int, p: int, act: str = "gelu", dtype: str = "bf16",
                 device="cuda", bias: bool = False, fused: bool = False, overlap_chunks: int = 0,
                 group_wgrad: bool = False):
        """fused: sum the shards inside the row GEMM and the column-backward dX
        GEMM (tp_row_fwd_reduce / tp_column_bwd_reduce) instead of writing p
        partials and reducing them (tp_row_fwd_partial + tp_reduce_partials).
        overlap_chunks > 1 (partials only): split the tokens into that many
        blocks and reduce block c on a second stream while the GEMM of block
        c + 1 runs (the compute / communication overlap of "从零实现 Tensor
        Parallel" §三, with the local reduce in place of the collective).
        group_wgrad: the row and column backward's weight gradients run as one
        grouped launch (tp_set_wgrad_grouping; backward() issues both). Off by
        default: on the 7B step it measured slower than two launches."""
        self.h, self.f, self.p, self.act = hidden, ffn, p, act
        self.fused = fused
        self.chunks = overlap_chunks if (overlap_chunks > 1 and not fused) else 0
        self._side = None
        self.plan = Plan(hidden, ffn, 0, p, dtype, act)
        if group_wgrad:
            self.plan.set_wgrad_grouping(True)
        self.dt = self.plan.torch_dtype
        self.device = torch.device(device)
        self.bias = bias
        fp = ffn // p
        self.n1 = 2 * fp if act == "swiglu" else fp
        self.fp = fp
        dev, dt = self.device, self.dt
        self.W1 = [_empty((self.n1, hidden), dt, dev) for _ in range(p)]
        self.W2 = [_empty((hidden, fp), dt, dev) for _ in range(p)]
        self.b1 = [_empty((self.n1,), dt, dev) for _ in range(p)] if bias else None
        self.b2 = _empty((hidden,), dt, dev) if bias else None
        self._T = None

    # --------------------------------------------------------------- weights
    def load_weights(self, W1_full: torch.Tensor, W2_full: torch.Tensor, b1_full=None, b2_full=None):
        """Shard full weights (already on the device) into the per-shard buffers."""
        self.plan.shard_column("mlp", W1_full.contiguous(), self.W1)
        self.plan.shard_row("mlp", W2_full.contiguous(), self.W2)
        if self.bias:
            self.plan.shard_column_bias("mlp", b1_full.contiguous(), self.b1)
            self.b2.copy_(b2_full)

    # ------------------------------------------------------------ activations
    def alloc(self, T: int, backward: bool = True):
        if self._T == T and (not backward or hasattr(self, "dZ")):
            return
        dev, dt, p = self.device, self.dt, self.p
        self._T = T
        self.Z = [_empty((T, self.n1), dt, dev) for _ in range(p)]
        self.H = [_empty((T, self.fp), dt, dev) for _ in range(p)]
        self.P = None if self.fused else [_empty((T, self.h), dt, dev) for _ in range(p)]
        self.Y = _empty((T, self.h), dt, dev)
        if backward:
            self.dZ = [_empty((T, self.n1), dt, dev) for _ in range(p)]
            self.dXp = None if self.fused else [_empty((T, self.h), dt, dev) for _ in range(p)]
            self.dX = _empty((T, self.h), dt, dev)
            self.dW1 = [torch.empty_like(w) for w in self.W1]
            self.dW2 = [torch.empty_like(w) for w in self.W2]
            self.db1 = [_empty((self.n1,), torch.float32, dev) for _ in range(p)] if self.bias else None
            self.db2 = _empty((self.h,), torch.float32, dev) if self.bias else None

    # ---------------------------------------------------------------- passes
    def forward(self, X: torch.Tensor, residual=None, out=None):
        T = X.shape[0]
        self.alloc(T, backward=hasattr(self, "dZ") or True)
        self.X = X
        pl = self.plan
        pl.column_fwd("mlp", T, X, self.W1, self.b1, self.Z if self.act != "none" else None, self.H)
        Y = self.Y if out is None else out
        if self.fused:
            pl.row_fwd_reduce("mlp", T, self.H, self.W2, self.b2, residual, Y)
        elif self.chunks:
            self._overlapped(T, lambda r0, r1: pl.row_fwd_partial(
                                 "mlp", r1 - r0, [h[r0:r1] for h in self.H], self.W2,
                                 [q[r0:r1] for q in self.P]),
                             lambda r0, r1: pl.reduce_partials(
                                 r1 - r0, [q[r0:r1] for q in self.P], self.b2,
                                 None if residual is None else residual[r0:r1], Y[r0:r1]))
        else:
            pl.row_fwd_partial("mlp", T, self.H, self.W2, self.P)
            pl.reduce_partials(T, self.P, self.b2, residual, Y)
        return Y

    def _overlapped(self, T, gemm, reduce, tail=None):
        """gemm(r0, r1) on the current stream for token block after block; each
        block's reduce(r0, r1) on a side stream as soon as its GEMM is done, so
        it runs under the next block's GEMM (and under tail(), if given, after
        the last block). The current stream waits for the last reduce before
        returning."""
        main = torch.cuda.current_stream()
        if self._side is None:
            self._side = torch.cuda.Stream(device=self.device)
        side = self._side
        step = -(-T // self.chunks)
        step = -(-step // 128) * 128           # whole 128-row tiles per block
        r0 = 0
        side.wait_stream(main)
        while r0 < T:
            r1 = min(T, r0 + step)
            gemm(r0, r1)
            ev = torch.cuda.Event()
            ev.record(main)
            side.wait_event(ev)
            with torch.cuda.stream(side):
                reduce(r0, r1)
            r0 = r1
        if tail is not None:
            tail()
        main.wait_stream(side)

    def backward(self, dY: torch.Tensor, out=None):
        T = dY.shape[0]
        pl = self.plan
        pl.row_bwd("mlp", T, dY, self.H, self.W2, self.Z if self.act != "none" else None, self.dZ,
                   self.dW2, self.db2)
        dX = self.dX if out is None else out
        if self.fused:
            pl.column_bwd_reduce("mlp", T, self.X, self.dZ, self.W1, self.dW1, self.db1, dX)
        elif self.chunks:
            # dX block by block with the reduces overlapped; the weight gradient
            # last, so the final block's reduce runs under it too.
            self._overlapped(T, lambda r0, r1: pl.column_bwd(
                                 "mlp", r1 - r0, None, [z[r0:r1] for z in self.dZ], self.W1, None,
                                 None, [q[r0:r1] for q in self.dXp]),
                             lambda r0, r1: pl.reduce_partials(
                                 r1 - r0, [q[r0:r1] for q in self.dXp], None, None, dX[r0:r1]),
                             tail=lambda: pl.column_bwd("mlp", T, self.X, self.dZ, self.W1,
                                                        self.dW1, self.db1, None))
        else:
            pl.column_bwd("mlp", T, self.X, self.dZ, self.W1, self.dW1, self.db1, self.dXp)
            pl.reduce_partials(T, self.dXp, None, None, dX)
        return dX

    # Number of useful FLOPs in one forward + backward (three GEMMs of each layer).
    def flops(self, T: int) -> float:
        n1_total = self.n1 * self.p
        fwd = 2.0 * T * self.h * n1_total + 2.0 * T * self.f * self.h
        return 3.0 * fwd


class HostStepPipeline:
    """Training steps of a TPMLP fed from and drained to pinned host memory,
    with the transfers overlapped with the compute: step(X_h, dY_h, Y_h, dX_h)
    enqueues the host-to-device copies of X and dY on one stream, the
    forward and backward on the current stream and the device-to-host copies
    of Y and dX on another, with two device buffer sets so the copies of one
    step run under the GEMMs of its neighbours. Every call returns at once;
    finish() makes the current stream wait for all outstanding copies."""

    def __init__(self, mlp: "TPMLP", T: int):
        dev, dt, h = mlp.device, mlp.dt, mlp.h
        self.m = mlp
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        self.X = [_empty((T, h), dt, dev) for _ in range(2)]
        self.dY = [_empty((T, h), dt, dev) for _ in range(2)]
        self.Y = [_empty((T, h), dt, dev) for _ in range(2)]
        self.dX = [_empty((T, h), dt, dev) for _ in range(2)]
        self.in_free = [None, None]   # compute done with input slot s
        self.out_free = [None, None]  # copy-out done with output slot s
        self.i = 0

    def step(self, X_h, dY_h, Y_h, dX_h):
        s = self.i % 2
        self.i += 1
        main = torch.cuda.current_stream()
        with torch.cuda.stream(self.h2d):
            if self.in_free[s] is not None:
                self.h2d.wait_event(self.in_free[s])
            self.X[s].copy_(X_h, non_blocking=True)
            x_in = torch.cuda.Event()
            x_in.record(self.h2d)
            self.dY[s].copy_(dY_h, non_blocking=True)
            dy_in = torch.cuda.Event()
            dy_in.record(self.h2d)
        main.wait_event(x_in)
        if self.out_free[s] is not None:
            main.wait_event(self.out_free[s])
        self.m.forward(self.X[s], out=self.Y[s])
        y_done = torch.cuda.Event()
        y_done.record(main)
        main.wait_event(dy_in)
        self.m.backward(self.dY[s], out=self.dX[s])
        dx_done = torch.cuda.Event()
        dx_done.record(main)
        self.in_free[s] = dx_done  # the backward reads X (weight gradient) and dY
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(y_done)
            Y_h.copy_(self.Y[s], non_blocking=True)
            self.d2h.wait_event(dx_done)
            dX_h.copy_(self.dX[s], non_blocking=True)
            out = torch.cuda.Event()
            out.record(self.d2h)
        self.out_free[s] = out

    def finish(self):
        main = torch.cuda.current_stream()
        main.wait_stream(self.h2d)
        main.wait_stream(self.d2h)


class SPMLP:
    """Megatron-SP SwiGLU MLP: LayerNorm on sequence shards, all-gather, column,
    row, reduce-scatter (and the mirrored backward)."""

    def __init__(self, hidden: int, ffn: int, p: int, act: str = "swiglu", device="cuda",
                 fused: bool = False):
        self.fused = fused
        self.mlp = TPMLP(hidden, ffn, p, act, "bf16", device, bias=False, fused=fused)
        self.plan = self.mlp.plan
        self.h, self.p = hidden, p
        self.gamma = torch.ones(hidden, dtype=torch.bfloat16, device=device)
        self.beta = torch.zeros(hidden, dtype=torch.bfloat16, device=device)
        self.device = torch.device(device)
        self._T = None

    def alloc(self, T: int):
        if self._T == T:
            return
        self._T = T
        dev, p, h = self.device, self.p, self.h
        t = T // p
        self.U = _empty((T, h), torch.bfloat16, dev)          # LN output, gathered
        self.mean = _empty((T,), torch.float32, dev)
        self.rstd = _empty((T,), torch.float32, dev)
        self.Y_seq = [_empty((t, h), torch.bfloat16, dev) for _ in range(p)]
        self.dY_full = _empty((T, h), torch.bfloat16, dev)
        self.dU_seq = [_empty((t, h), torch.bfloat16, dev) for _ in range(p)]
        self.dX_seq = [_empty((t, h), torch.bfloat16, dev) for _ in range(p)]
        self.dgamma = _empty((h,), torch.float32, dev)
        self.dbeta = _empty((h,), torch.float32, dev)
        self.mlp.alloc(T)

    def forward(self, X_seq):
        p = self.p
        T = X_seq[0].shape[0] * p
        self.alloc(T)
        self.X_seq = X_seq
        pl, m = self.plan, self.mlp
        pl.layernorm_all_gather_seq(T, X_seq, self.gamma, self.beta, self.U, self.mean, self.rstd)
        m.X = self.U
        pl.column_fwd("mlp", T, self.U, m.W1, None, m.Z, m.H)
        if self.fused:
            pl.row_fwd_reduce_scatter_seq("mlp", T, m.H, m.W2, None, None, self.Y_seq)
        else:
            pl.row_fwd_partial("mlp", T, m.H, m.W2, m.P)
            pl.reduce_scatter_seq(T, m.P, None, None, self.Y_seq)
        return self.Y_seq

    def backward(self, dY_seq):
        p = self.p
        T = dY_seq[0].shape[0] * p
        t = T // p
        pl, m = self.plan, self.mlp
        pl.reduce_scatter_seq_bwd(T, dY_seq, self.dY_full)
        pl.row_bwd("mlp", T, self.dY_full, m.H, m.W2, m.Z, m.dZ, m.dW2, None)
        if self.fused:
            pl.column_bwd_reduce_scatter_seq("mlp", T, self.U, m.dZ, m.W1, m.dW1, None, self.dU_seq)
        else:
            pl.column_bwd("mlp", T, self.U, m.dZ, m.W1, m.dW1, None, m.dXp)
            pl.all_gather_seq_bwd(T, m.dXp, self.dU_seq)
        for j in range(p):
            pl.layernorm_bwd(t, self.X_seq[j], self.gamma, self.dU_seq[j], self.mean[j * t:(j + 1) * t],
                             self.rstd[j * t:(j + 1) * t], self.dX_seq[j], self.dgamma, self.dbeta,
                             accumulate=j > 0)
        return self.dX_seq

    def flops(self, T: int) -> float:
        return self.mlp.flops(T)


class TPAttention:
    """Attention sublayer split by whole heads over p shards on one GPU:
    QKV column GEMM -> causal attention on local heads -> out-projection row
    GEMM partials -> reduce (+bias once, +residual).   (TP walkthrough §3.1)
    fused: the out-projection (forward) and the QKV dX (backward) sum the
    shards in the GEMM accumulator (tp_row_fwd_reduce / tp_column_bwd_reduce)
    instead of writing p partials and reducing them."""

    def __init__(self, hidden: int, heads: int, p: int, device="cuda", bias: bool = False,
                 fused: bool = False):
        self.fused = fused
        self.h, self.H, self.p = hidden, heads, p
        self.plan = Plan(hidden, 0, heads, p, "bf16", "none")
        self.device = torch.device(device)
        self.d = hidden // heads
        self.hl = heads // p
        n = 3 * hidden // p
        dev = self.device
        self.Wqkv = [_empty((n, hidden), torch.bfloat16, dev) for _ in range(p)]
        self.Wo = [_empty((hidden, hidden // p), torch.bfloat16, dev) for _ in range(p)]
        self.bias = bias
        self.bqkv = [_empty((n,), torch.bfloat16, dev) for _ in range(p)] if bias else None
        self.bo = _empty((hidden,), torch.bfloat16, dev) if bias else None
        self._key = None

    def load_weights(self, Wqkv_full, Wo_full, bqkv_full=None, bo_full=None):
        self.plan.shard_column("qkv", Wqkv_full.contiguous(), self.Wqkv)
        self.plan.shard_row("outproj", Wo_full.contiguous(), self.Wo)
        if self.bias:
            self.plan.shard_column_bias("qkv", bqkv_full.contiguous(), self.bqkv)
            self.bo.copy_(bo_full)

    def alloc(self, batch: int, seq: int):
        if self._key == (batch, seq):
            return
        self._key = (batch, seq)
        T, p, dev = batch * seq, self.p, self.device
        n = 3 * self.h // p
        self.QKV = [_empty((T, n), torch.bfloat16, dev) for _ in range(p)]
        self.O = [_empty((T, self.h // p), torch.bfloat16, dev) for _ in range(p)]
        self.LSE = [_empty((batch, self.hl, seq), torch.float32, dev) for _ in range(p)]
        self.P = None if self.fused else [_empty((T, self.h), torch.bfloat16, dev) for _ in range(p)]
        self.Y = _empty((T, self.h), torch.bfloat16, dev)

    def forward(self, X: torch.Tensor, batch: int, seq: int, residual=None, out=None):
        self.alloc(batch, seq)
        T = batch * seq
        pl = self.plan
        self.X = X
        pl.column_fwd("qkv", T, X, self.Wqkv, self.bqkv, None, self.QKV)
        pl.attention_fwd(batch, seq, self.QKV, self.O, self.LSE)
        Y = self.Y if out is None else out
        if self.fused:
            pl.row_fwd_reduce("outproj", T, self.O, self.Wo, self.bo, residual, Y)
        else:
            pl.row_fwd_partial("outproj", T, self.O, self.Wo, self.P)
            pl.reduce_partials(T, self.P, self.bo, residual, Y)
        return Y

    def alloc_bwd(self):
        if hasattr(self, "dQKV") and self.dQKV[0].shape == self.QKV[0].shape:
            return
        T, p, dev = self.QKV[0].shape[0], self.p, self.device
        self.dO = [_empty((T, self.h // p), torch.bfloat16, dev) for _ in range(p)]
        self.dQKV = [torch.empty_like(x) for x in self.QKV]
        self.dXp = None if self.fused else [_empty((T, self.h), torch.bfloat16, dev) for _ in range(p)]
        self.dX = _empty((T, self.h), torch.bfloat16, dev)
        self.dWqkv = [torch.empty_like(w) for w in self.Wqkv]
        self.dWo = [torch.empty_like(w) for w in self.Wo]
        self.dbqkv = [_empty((w.shape[0],), torch.float32, dev) for w in self.Wqkv] if self.bias else None
        self.dbo = _empty((self.h,), torch.float32, dev) if self.bias else None

    def backward(self, dY: torch.Tensor, batch: int, seq: int, out=None):
        """dY -> (out-proj row bwd) dO_i, dWo_i, dbo -> (attention bwd) dQKV_i ->
        (QKV column bwd) dWqkv_i, dbqkv_i, dX partials -> reduce."""
        self.alloc_bwd()
        T = batch * seq
        pl = self.plan
        pl.row_bwd("outproj", T, dY, self.O, self.Wo, None, self.dO, self.dWo, self.dbo)
        pl.attention_bwd(batch, seq, self.QKV, self.O, self.dO, self.LSE, self.dQKV)
        dX = self.dX if out is None else out
        if self.fused:
            pl.column_bwd_reduce("qkv", T, self.X, self.dQKV, self.Wqkv, self.dWqkv, self.dbqkv, dX)
        else:
            pl.column_bwd("qkv", T, self.X, self.dQKV, self.Wqkv, self.dWqkv, self.dbqkv, self.dXp)
            pl.reduce_partials(T, self.dXp, None, None, dX)
        return dX

    def flops_fwd(self, batch: int, seq: int, causal: bool = True) -> float:
        T = batch * seq
        proj = 2.0 * T * self.h * 3 * self.h + 2.0 * T * self.h * self.h
        pairs = seq * (seq + 1) / 2 if causal else seq * seq
        att = 4.0 * batch * self.H * pairs * self.d
        return proj + att


class TPLayer:
    """Pre-LN transformer layer with a GELU MLP, every sublayer split over p
    shards on one GPU: x1 = x + Attn(LN1(x)); y = x1 + MLP(LN2(x1)).
    Biases on every projection (TP-basics' row bias enters once, in the reduce)."""

    def __init__(self, hidden: int, ffn: int, heads: int, p: int, device="cuda", fused: bool = True):
        """fused: both sublayers sum their shards inside the GEMMs (no partials)."""
        self.h = hidden
        self.attn = TPAttention(hidden, heads, p, device, bias=True, fused=fused)
        self.mlp = TPMLP(hidden, ffn, p, "gelu", "bf16", device, bias=True, fused=fused)
        # weight gradients and bias sums off the critical path (joined in backward)
        self.attn.plan.set_backward_defer(True)
        self.mlp.plan.set_backward_defer(True)
        self.ln = Plan(hidden, 0, 0, 1, "bf16", "none")  # LayerNorm / elementwise calls
        self.device = torch.device(device)
        dev = self.device
        self.ln1_g = torch.ones(hidden, dtype=torch.bfloat16, device=dev)
        self.ln1_b = torch.zeros(hidden, dtype=torch.bfloat16, device=dev)
        self.ln2_g = torch.ones(hidden, dtype=torch.bfloat16, device=dev)
        self.ln2_b = torch.zeros(hidden, dtype=torch.bfloat16, device=dev)
        self._T = None

    def load(self, prm):
        """prm: a tp_synth.LayerParams with tensors already on the device."""
        self.ln1_g.copy_(prm.ln1_g)
        self.ln1_b.copy_(prm.ln1_b)
        self.ln2_g.copy_(prm.ln2_g)
        self.ln2_b.copy_(prm.ln2_b)
        self.attn.load_weights(prm.Wqkv, prm.Wo, prm.bqkv, prm.bo)
        self.mlp.load_weights(prm.W1, prm.W2, prm.b1, prm.b2)

    def alloc(self, T: int):
        if self._T == T:
            return
        self._T = T
        dev, h = self.device, self.h
        bf, f32 = torch.bfloat16, torch.float32
        self.u1, self.u2 = _empty((T, h), bf, dev), _empty((T, h), bf, dev)
        self.x1, self.y = _empty((T, h), bf, dev), _empty((T, h), bf, dev)
        self.m1, self.r1 = _empty((T,), f32, dev), _empty((T,), f32, dev)
        self.m2, self.r2 = _empty((T,), f32, dev), _empty((T,), f32, dev)
        self.dx1, self.dx = _empty((T, h), bf, dev), _empty((T, h), bf, dev)
        self.dln1_g, self.dln1_b = _empty((h,), f32, dev), _empty((h,), f32, dev)
        self.dln2_g, self.dln2_b = _empty((h,), f32, dev), _empty((h,), f32, dev)

    def forward(self, x: torch.Tensor, batch: int, seq: int):
        T = batch * seq
        self.alloc(T)
        self.x = x
        ln = self.ln
        ln.layernorm_fwd(T, x, self.ln1_g, self.ln1_b, self.u1, self.m1, self.r1)
        self.attn.forward(self.u1, batch, seq, residual=x, out=self.x1)
        ln.layernorm_fwd(T, self.x1, self.ln2_g, self.ln2_b, self.u2, self.m2, self.r2)
        self.mlp.forward(self.u2, residual=self.x1, out=self.y)
        return self.y

    def backward(self, dy: torch.Tensor, batch: int, seq: int, join: bool = True):
        """join=False leaves this layer's weight gradients and bias sums
        running on the side stream (a caller that backpropagates several
        layers joins once, with tp.backward_join(), before reading them)."""
        T = batch * seq
        ln = self.ln
        du2 = self.mlp.backward(dy)
        # dx1 = dy (residual branch) + LN2 backward, in one launch
        ln.layernorm_bwd(T, self.x1, self.ln2_g, du2, self.m2, self.r2, self.dx1,
                         self.dln2_g, self.dln2_b, dres=dy)
        du1 = self.attn.backward(self.dx1, batch, seq)
        ln.layernorm_bwd(T, self.x, self.ln1_g, du1, self.m1, self.r1, self.dx,
                         self.dln1_g, self.dln1_b, dres=self.dx1)
        if join:
            backward_join()
        return self.dx


class CapturedStep:
    """A step (a callable that only issues libtp.so launches on the current
    stream) captured once into a CUDA graph and replayed: one graph launch
    instead of one host call per kernel. The step runs eagerly `warmup` times
    first, on the capture stream, so every workspace the library allocates on
    first use exists before capture starts."""

    def __init__(self, fn, warmup: int = 2):
        from .tp import launch_count
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        before = launch_count()
        with torch.cuda.graph(self.graph):
            fn()
        self.launches = launch_count() - before  # kernel launches per replay

    def __call__(self):
        self.graph.replay()
