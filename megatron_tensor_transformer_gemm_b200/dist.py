"""Tensor parallelism across GPUs: the p shards of a layer split over N ranks
(one process per GPU, torch.distributed over NCCL), each rank holding p/N
shards as separate buffers in its own libtp plan.

Inside a rank everything is the single-GPU path: the column GEMM over the
local shards, and the row GEMM with the local shards' sum in its accumulator
(tp_row_fwd_reduce). Between ranks the method's exchange steps become NCCL
collectives:

  forward   Y   = all-reduce over ranks of each rank's local shard sum
            (Megatron-SP: reduce-scatter along the sequence instead, after an
            all-gather of the LayerNorm output)       TP walkthrough §2.2, §4.1, §4.3
  backward  dX  = all-reduce of each rank's local dX sum (SP: reduce-scatter,
            after an all-gather of dY)               从零实现 Tensor Parallel §四

The row bias and the residual enter the sum exactly once: rank 0 adds them in
its local GEMM epilogue, every other rank contributes its bare partial sum
(Tensor Parallelism基础, 实现细节: the row bias is added once, after the sum).

The collective steps (sum_over_ranks, scatter_seq_sum, gather_seq) and the
weight slicing are plain torch.distributed / tensor code, independent of the
device, so they run unchanged on CPU gloo ranks.

comm="peer" replaces the all-reduces (and the Megatron-SP reduce-scatters) of
Y and dX by libtp's peer-memory steps: the row GEMM (and the column
backward's dX GEMM) stores each row block of its local sum straight into the
owning rank's receive buffer from its epilogue, the owner sums the world
slots once and pushes its block to every rank's output (non-SP) or keeps it
(SP), and a device-side wait closes the exchange ("张量并行", Megatron-SP:
all-reduce = reduce-scatter + all-gather). Under SP the all-gathers go the same
way: the LayerNorm kernel pushes each normalised row into every rank's
gathered input, and dY's shard is pushed likewise. The buffers are mapped between the
processes with CUDA IPC (PeerMemory); bias and residual are added once, in
the owner's reduce.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import tp
from .tp import Plan


# ----------------------------------------------------------------- host logic

def rank_shards(p: int, world: int, rank: int) -> range:
    """Global shard indices owned by `rank`: a contiguous block of p/world."""
    if world < 1 or p % world:
        raise ValueError(f"p = {p} shards do not split over {world} ranks")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    k = p // world
    return range(rank * k, (rank + 1) * k)


def local_mlp_weights(W1: torch.Tensor, W2: torch.Tensor, p: int, world: int, rank: int, act: str):
    """The rows of W1 [n1, h] and the columns of W2 [h, f] that rank `rank`
    holds, arranged so that the local plan's own p/world-way split of them
    gives exactly the global shards rank_shards(p, world, rank).

    GELU / none: W1 rows [lo*f/p, hi*f/p). SwiGLU (W1 = [G; U]): the gate rows
    and the matching up rows of those units, stacked [G_r; U_r], so each local
    shard is [G_i; U_i] of its global index i (TP walkthrough §3.2)."""
    sh = rank_shards(p, world, rank)
    f = W2.shape[1]
    fp = f // p
    c0, c1 = sh.start * fp, sh.stop * fp
    if act == "swiglu":
        if W1.shape[0] != 2 * f:
            raise ValueError("SwiGLU W1 must be [2*ffn, hidden] = [G; U]")
        W1r = torch.cat([W1[c0:c1], W1[f + c0:f + c1]], 0)
    else:
        W1r = W1[c0:c1]
    return W1r.contiguous(), W2[:, c0:c1].contiguous()


def once_on_rank0(t, rank: int):
    """A term that must enter an all-reduced sum exactly once (the row bias,
    the residual): rank 0 contributes it, the others contribute nothing."""
    return t if rank == 0 else None


def sum_over_ranks(t: torch.Tensor, group=None) -> torch.Tensor:
    """The all-reduce of the row layer across ranks, in place (SUM)."""
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def scatter_seq_sum(full: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """Megatron-SP reduce-scatter: out (rows [r*T/N, (r+1)*T/N) of the sum of
    every rank's full-shape `full`) on rank r."""
    dist.reduce_scatter_tensor(out, full, op=dist.ReduceOp.SUM, group=group)
    return out


def gather_seq(shard: torch.Tensor, out: torch.Tensor, group=None) -> torch.Tensor:
    """Megatron-SP all-gather along the sequence: out = concat of every
    rank's shard in rank order."""
    dist.all_gather_into_tensor(out, shard, group=group)
    return out


# ------------------------------------------------------------- peer memory

class _DevView:
    """A raw device range as a __cuda_array_interface__ of int16 (bf16 bits)."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes // 2,), "typestr": "<i2", "data": (ptr, False),
                                         "version": 3, "strides": None}


def bf16_view(ptr: int, shape, device) -> torch.Tensor:
    """A bf16 tensor over the device range at `ptr` (not owned: the memory
    must outlive the tensor)."""
    n = 1
    for x in shape:
        n *= x
    t = torch.as_tensor(_DevView(ptr, 2 * n), device=device)
    return t.view(torch.bfloat16).view(*shape)


class PeerMemory:
    """`nbytes` of device memory on every rank of `group`, each rank's block
    mapped into every other rank's process (tp_peer_alloc, the IPC handles
    all-gathered, tp_peer_open). ptrs[d] is rank d's block as seen here;
    ptrs[rank] is this rank's own. close() unmaps and frees; tensors made by
    bf16() do not own the memory and must not outlive it."""

    def __init__(self, nbytes: int, group=None, device=None):
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.nbytes = nbytes
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.local, handle = tp.peer_alloc(nbytes)
        handles = [None] * self.world
        if self.world > 1:
            dist.all_gather_object(handles, handle, group=group)
        else:
            handles[0] = handle
        self.ptrs, self._opened = [], []
        try:
            for d, h in enumerate(handles):
                if d == self.rank:
                    self.ptrs.append(self.local)
                else:
                    ptr = tp.peer_open(h)
                    self._opened.append(ptr)
                    self.ptrs.append(ptr)
        except Exception:
            self.close()
            raise

    def bf16(self, offset: int, shape) -> torch.Tensor:
        """A bf16 tensor over this rank's block at byte `offset`."""
        n = 1
        for x in shape:
            n *= x
        if offset % 16 or offset + 2 * n > self.nbytes:
            raise ValueError("view outside the peer block or not 16-byte aligned")
        return bf16_view(self.local + offset, shape, self.device)

    def close(self):
        for ptr in self._opened:
            tp.peer_close(ptr)
        self._opened = []
        if self.local:
            tp.peer_free(self.local)
            self.local = 0


class PeerGroup:
    """The flag words and receive buffers of one exchange between the ranks
    of `group` (tp_peer_group), for up to recv_elems elements per rank, and
    the epoch counter every rank advances in step."""

    def __init__(self, recv_elems: int, group=None, device=None):
        self.mem = PeerMemory(tp.PEER_FLAG_BYTES + 2 * recv_elems, group, device)
        self.world, self.rank = self.mem.world, self.mem.rank
        self.recv_elems = recv_elems
        self.c = tp.peer_group(self.world, self.rank, recv_elems, self.mem.ptrs,
                               [q + tp.PEER_FLAG_BYTES for q in self.mem.ptrs])
        self.epoch = 0

    def next_epoch(self) -> int:
        self.epoch = (self.epoch + 1) & 0xFFFFFFFF
        return self.epoch

    def reduce(self, T: int, hidden: int, bias, residual, out, epoch: int):
        """tp_peer_reduce then tp_peer_wait: this rank's row block of the sum
        over ranks (+ bias + residual) into every pointer of `out`."""
        tp.peer_reduce(self.c, T, hidden, bias, residual, out, epoch)
        tp.peer_wait(self.c, epoch)

    def close(self):
        self.mem.close()


# ------------------------------------------------------------------- the layer

class DistTPMLP:
    """An MLP sublayer whose p shards are split over the ranks of `group`,
    p/N per GPU. sequence_parallel=False: replicated input X [T, h], output
    Y [T, h] on every rank. sequence_parallel=True (Megatron-SP): each rank
    holds the sequence shard X_r [T/N, h], LayerNorm runs on it, and the
    output is the rank's sequence shard of Y."""

    def __init__(self, hidden: int, ffn: int, p: int, act: str = "swiglu", group=None,
                 device="cuda", bias: bool = False, sequence_parallel: bool = False,
                 comm: str = "nccl"):
        if comm not in ("nccl", "peer"):
            raise ValueError(f"comm must be 'nccl' or 'peer', not {comm!r}")
        self.comm = comm
        self.peer = self.Ymem = self.dXmem = self.Umem = self.dYmem = None
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.shards = rank_shards(p, self.world, self.rank)
        self.p, self.pl = p, p // self.world
        self.h, self.f, self.act = hidden, ffn, act
        self.fl = ffn // self.world               # this rank's slice of the intermediate dim
        self.sp = sequence_parallel
        self.device = torch.device(device)
        self.plan = Plan(hidden, self.fl, 0, self.pl, "bf16", act)
        self.ln = Plan(hidden, 0, 0, 1, "bf16", "none")
        fp = ffn // p
        self.n1 = 2 * fp if act == "swiglu" else fp
        self.fp = fp
        dev, bf = self.device, torch.bfloat16
        self.W1 = [torch.empty(self.n1, hidden, dtype=bf, device=dev) for _ in range(self.pl)]
        self.W2 = [torch.empty(hidden, fp, dtype=bf, device=dev) for _ in range(self.pl)]
        self.bias = bias
        self.b1 = [torch.empty(self.n1, dtype=bf, device=dev) for _ in range(self.pl)] if bias else None
        self.b2 = torch.empty(hidden, dtype=bf, device=dev) if bias else None
        self.gamma = torch.ones(hidden, dtype=bf, device=dev)
        self.beta = torch.zeros(hidden, dtype=bf, device=dev)
        self._T = None

    def load_weights(self, W1_full, W2_full, b1_full=None, b2_full=None):
        """Full weights (any device, [out, in]) -> this rank's shards."""
        W1r, W2r = local_mlp_weights(W1_full, W2_full, self.p, self.world, self.rank, self.act)
        self.plan.shard_column("mlp", W1r.to(self.device), self.W1)
        self.plan.shard_row("mlp", W2r.to(self.device), self.W2)
        if self.bias:
            sh, fp = self.shards, self.fp
            b1r = b1_full[sh.start * fp:sh.stop * fp]
            if self.act == "swiglu":
                raise ValueError("a column bias is not supported with SwiGLU")
            self.plan.shard_column_bias("mlp", b1r.contiguous().to(self.device), self.b1)
            self.b2.copy_(b2_full)

    def alloc(self, T: int):
        if self._T == T:
            return
        if T % self.world:
            raise ValueError(f"T = {T} does not split over {self.world} ranks")
        self._T = T
        dev, bf, h, pl = self.device, torch.bfloat16, self.h, self.pl
        t = T // self.world
        self.Z = [torch.empty(T, self.n1, dtype=bf, device=dev) for _ in range(pl)]
        self.H = [torch.empty(T, self.fp, dtype=bf, device=dev) for _ in range(pl)]
        self.dZ = [torch.empty(T, self.n1, dtype=bf, device=dev) for _ in range(pl)]
        self.dW1 = [torch.empty_like(w) for w in self.W1]
        self.dW2 = [torch.empty_like(w) for w in self.W2]
        self.db1 = [torch.empty(self.n1, dtype=torch.float32, device=dev) for _ in range(pl)] if self.bias else None
        self.db2 = torch.empty(h, dtype=torch.float32, device=dev) if self.bias else None
        if self.comm == "peer":
            self.close_peer()
            self.peer = PeerGroup(T * h, self.group, dev)
            if not self.sp:   # outputs the other ranks push their row blocks into
                self.Ymem = PeerMemory(2 * T * h, self.group, dev)
                self.dXmem = PeerMemory(2 * T * h, self.group, dev)
                self.Yp, self.dXp = self.Ymem.bf16(0, (T, h)), self.dXmem.bf16(0, (T, h))
            else:             # gathered inputs the other ranks push their sequence shards into
                self.Yp = self.dXp = None
                self.Umem = PeerMemory(2 * T * h, self.group, dev)
                self.dYmem = PeerMemory(2 * T * h, self.group, dev)
        else:
            self.Yp = torch.empty(T, h, dtype=bf, device=dev)     # local sum, then the all-reduced Y
            self.dXp = torch.empty(T, h, dtype=bf, device=dev)
        if self.sp:
            self.Xn = torch.empty(t, h, dtype=bf, device=dev)   # LayerNorm of the local shard
            self.U = (self.Umem.bf16(0, (T, h)) if self.comm == "peer" else
                      torch.empty(T, h, dtype=bf, device=dev))  # gathered LayerNorm output
            self.mean = torch.empty(t, dtype=torch.float32, device=dev)
            self.rstd = torch.empty(t, dtype=torch.float32, device=dev)
            self.Y_seq = torch.empty(t, h, dtype=bf, device=dev)
            self.dY_full = (self.dYmem.bf16(0, (T, h)) if self.comm == "peer" else
                            torch.empty(T, h, dtype=bf, device=dev))
            self.dU_seq = torch.empty(t, h, dtype=bf, device=dev)
            self.dX_seq = torch.empty(t, h, dtype=bf, device=dev)
            self.dgamma = torch.empty(h, dtype=torch.float32, device=dev)
            self.dbeta = torch.empty(h, dtype=torch.float32, device=dev)

    def forward(self, X: torch.Tensor, residual=None):
        """Non-SP: X [T, h] replicated; returns Y [T, h] (replicated).
        SP: X is this rank's sequence shard [T/N, h]; returns its shard of Y."""
        pl, g = self.plan, self.group
        if self.sp:
            t = X.shape[0]
            T = t * self.world
            self.alloc(T)
            self.X_in = X
            if self.comm == "peer":   # LayerNorm pushed into every rank's U at this rank's rows
                e = self.peer.next_epoch()
                self.ln.layernorm_all_gather_push_peer(self.peer.c, t, X, self.gamma, self.beta,
                                                       self._blocks(self.Umem, T), self.mean, self.rstd, e)
                tp.peer_wait(self.peer.c, e)
            else:
                self.ln.layernorm_fwd(t, X, self.gamma, self.beta, self.Xn, self.mean, self.rstd)
                gather_seq(self.Xn, self.U, g)
            Xin = self.U
        else:
            T = X.shape[0]
            self.alloc(T)
            Xin = X
        self.X = Xin
        pl.column_fwd("mlp", T, Xin, self.W1, self.b1, self.Z if self.act != "none" else None, self.H)
        if self.comm == "peer":
            e = self.peer.next_epoch()
            pl.row_fwd_push_peer("mlp", T, self.H, self.W2, self.peer.c, e)
            t, r = T // self.world, self.rank
            if self.sp:
                self.peer.reduce(T, self.h, self.b2, residual, [self.Y_seq], e)
                return self.Y_seq
            res = residual[r * t:(r + 1) * t] if residual is not None else None
            self.peer.reduce(T, self.h, self.b2, res, self._blocks(self.Ymem, T), e)
            return self.Yp
        res = None if self.sp else once_on_rank0(residual, self.rank)
        pl.row_fwd_reduce("mlp", T, self.H, self.W2, once_on_rank0(self.b2, self.rank), res, self.Yp)
        if self.sp:
            scatter_seq_sum(self.Yp, self.Y_seq, g)
            if residual is not None:
                self.Y_seq.add_(residual)
            return self.Y_seq
        return sum_over_ranks(self.Yp, g)

    def backward(self, dY: torch.Tensor):
        """Non-SP: dY [T, h] replicated; returns dX [T, h]. SP: dY is this
        rank's sequence shard; returns the gradient of its input shard (the
        LayerNorm's dgamma, dbeta are summed over ranks)."""
        pl, g = self.plan, self.group
        T = self._T
        if self.sp:
            if self.comm == "peer":
                e = self.peer.next_epoch()
                tp.all_gather_push_peer(self.peer.c, T // self.world, self.h, dY, self._blocks(self.dYmem, T), e)
                tp.peer_wait(self.peer.c, e)
            else:
                gather_seq(dY, self.dY_full, g)
            dYf = self.dY_full
        else:
            dYf = dY
        pl.row_bwd("mlp", T, dYf, self.H, self.W2, self.Z if self.act != "none" else None, self.dZ,
                   self.dW2, self.db2)
        if self.comm == "peer":
            e = self.peer.next_epoch()
            pl.column_bwd_push_peer("mlp", T, self.X, self.dZ, self.W1, self.dW1, self.db1, self.peer.c, e)
            if not self.sp:
                self.peer.reduce(T, self.h, None, None, self._blocks(self.dXmem, T), e)
                return self.dXp
            self.peer.reduce(T, self.h, None, None, [self.dU_seq], e)
            t = T // self.world
            self.ln.layernorm_bwd(t, self.X_in, self.gamma, self.dU_seq, self.mean, self.rstd,
                                  self.dX_seq, self.dgamma, self.dbeta)
            sum_over_ranks(self.dgamma, g)
            sum_over_ranks(self.dbeta, g)
            return self.dX_seq
        pl.column_bwd_reduce("mlp", T, self.X, self.dZ, self.W1, self.dW1, self.db1, self.dXp)
        if not self.sp:
            return sum_over_ranks(self.dXp, g)
        scatter_seq_sum(self.dXp, self.dU_seq, g)
        t = T // self.world
        self.ln.layernorm_bwd(t, self.X_in, self.gamma, self.dU_seq, self.mean, self.rstd,
                              self.dX_seq, self.dgamma, self.dbeta)
        sum_over_ranks(self.dgamma, g)
        sum_over_ranks(self.dbeta, g)
        return self.dX_seq

    def _blocks(self, mem: PeerMemory, T: int) -> list:
        """This rank's row block of the [T, h] output on every rank."""
        off = self.rank * (T // self.world) * self.h * 2
        return [q + off for q in mem.ptrs]

    def close_peer(self):
        for m in (self.peer, self.Ymem, self.dXmem, self.Umem, self.dYmem):
            if m is not None:
                m.close()
        self.peer = self.Ymem = self.dXmem = self.Umem = self.dYmem = None

    def flops(self, T: int) -> float:
        """Useful FLOPs of one forward + backward of the whole layer (all ranks)."""
        n1_total = self.n1 * self.p
        return 3.0 * (2.0 * T * self.h * n1_total + 2.0 * T * self.f * self.h)
