"""The peer-memory all-reduce (tp_row_fwd_push_peer / tp_column_bwd_push_peer,
tp_peer_reduce, tp_peer_wait) with `world` ranks emulated on the one GPU these
tests have: every rank's receive buffer, flag words and outputs are local
buffers, and each step is taken for every rank before the next step begins
(all pushes, then all reduces, then all waits), so every flag a kernel waits
for was raised by a launch that precedes it on the stream: no kernel waits for
a later one. The kernels, pointers and flag protocol are the ones a real
multi-GPU run uses; only the memory is local instead of mapped from a peer.

The sum over all p = world x p_local shards must match the oracle MLP within
the bf16 tolerance on every rank, the ranks' outputs must agree bit for bit,
and a second round with the next epoch must repeat the first exactly."""
import os
import subprocess
import sys

import pytest
import torch

import oracle as O
import tp_synth
from gpu_helpers import TOL_BF16, assert_close, dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class EmulatedRanks:
    """world ranks of one sharded MLP on one GPU, each with its own libtp
    plan, local shards, receive buffer, flags and peer-visible outputs."""

    def __init__(self, world, p_local, T, h, f, act, inp):
        from megatron_tensor_transformer_gemm_b200 import tp
        from megatron_tensor_transformer_gemm_b200.dist import bf16_view, local_mlp_weights
        self.tp, self.world, self.T, self.h, self.act = tp, world, T, h, act
        self.t = T // world
        P = world * p_local
        fl, fp = f // world, f // P
        n1 = 2 * fp if act == "swiglu" else fp
        self.allocs = []

        def alloc(nbytes):
            ptr, _ = tp.peer_alloc(nbytes)
            self.allocs.append(ptr)
            return ptr

        mem = [alloc(tp.PEER_FLAG_BYTES + 2 * T * h) for _ in range(world)]
        self.Yptr = [alloc(2 * T * h) for _ in range(world)]
        self.dXptr = [alloc(2 * T * h) for _ in range(world)]
        self.Y = [bf16_view(q, (T, h), "cuda") for q in self.Yptr]
        self.dX = [bf16_view(q, (T, h), "cuda") for q in self.dXptr]
        self.g = [tp.peer_group(world, r, T * h, mem, [q + tp.PEER_FLAG_BYTES for q in mem]) for r in range(world)]
        bf = torch.bfloat16
        self.ranks = []
        for r in range(world):
            pl = tp.Plan(h, fl, 0, p_local, "bf16", act)
            W1r, W2r = local_mlp_weights(inp.W1, inp.W2, P, world, r, act)
            W1 = [torch.empty(n1, h, dtype=bf, device="cuda") for _ in range(p_local)]
            W2 = [torch.empty(h, fp, dtype=bf, device="cuda") for _ in range(p_local)]
            pl.shard_column("mlp", dev(W1r), W1)
            pl.shard_row("mlp", dev(W2r), W2)
            b1 = None
            if inp.b1 is not None:
                b1 = [torch.empty(n1, dtype=bf, device="cuda") for _ in range(p_local)]
                pl.shard_column_bias("mlp", dev(inp.b1[r * fl:(r + 1) * fl].contiguous()), b1)
            self.ranks.append(dict(
                plan=pl, W1=W1, W2=W2, b1=b1,
                Z=[torch.empty(T, n1, dtype=bf, device="cuda") for _ in range(p_local)],
                H=[torch.empty(T, fp, dtype=bf, device="cuda") for _ in range(p_local)],
                dZ=[torch.empty(T, n1, dtype=bf, device="cuda") for _ in range(p_local)],
                dW1=[torch.empty(n1, h, dtype=bf, device="cuda") for _ in range(p_local)],
                dW2=[torch.empty(h, fp, dtype=bf, device="cuda") for _ in range(p_local)],
                db1=[torch.empty(n1, dtype=torch.float32, device="cuda") for _ in range(p_local)]
                if b1 is not None else None))

    def blocks(self, ptrs, r):
        off = r * self.t * self.h * 2
        return [q + off for q in ptrs]

    def forward(self, X, b2, residual, epoch, sp=False, Y_seq=None):
        tp, t = self.tp, self.t
        for r, k in enumerate(self.ranks):     # step 1 on every rank
            k["plan"].column_fwd("mlp", self.T, X, k["W1"], k["b1"], k["Z"], k["H"])
            k["plan"].row_fwd_push_peer("mlp", self.T, k["H"], k["W2"], self.g[r], epoch)
        for r in range(self.world):            # step 2 on every rank
            res = residual[r * t:(r + 1) * t] if residual is not None else None
            out = [Y_seq[r]] if sp else self.blocks(self.Yptr, r)
            tp.peer_reduce(self.g[r], self.T, self.h, b2, res, out, epoch)
        for r in range(self.world):            # step 3 on every rank
            tp.peer_wait(self.g[r], epoch)

    def backward(self, X, dY, epoch):
        tp = self.tp
        for r, k in enumerate(self.ranks):
            k["plan"].row_bwd("mlp", self.T, dY, k["H"], k["W2"], k["Z"], k["dZ"], k["dW2"], None)
            k["plan"].column_bwd_push_peer("mlp", self.T, X, k["dZ"], k["W1"], k["dW1"], k["db1"],
                                           self.g[r], epoch)
        for r in range(self.world):
            tp.peer_reduce(self.g[r], self.T, self.h, None, None, self.blocks(self.dXptr, r), epoch)
        for r in range(self.world):
            tp.peer_wait(self.g[r], epoch)

    def status(self):
        from megatron_tensor_transformer_gemm_b200 import tp
        torch.cuda.synchronize()
        return tp.lib.tp_get_device_status(None, None)

    def close(self):
        torch.cuda.synchronize()
        for q in self.allocs:
            self.tp.peer_free(q)
        self.allocs = []


CASES = [
    # world, p_local, T, hidden, ffn, act, bias
    (1, 2, 96, 128, 512, "swiglu", False),
    (2, 2, 256, 256, 1024, "swiglu", False),
    (3, 1, 120, 192, 384, "gelu", True),      # 40-row blocks: not whole 32-row slabs
    (4, 2, 520, 256, 1024, "swiglu", False),  # 130-row blocks, ragged last tile
    (8, 1, 1024, 512, 2048, "gelu", False),
]


@pytest.mark.parametrize("world,p_local,T,h,f,act,bias", CASES)
def test_peer_all_reduce_emulated_ranks(world, p_local, T, h, f, act, bias):
    inp = tp_synth.draw_mlp(T, h, f, act, torch.bfloat16, seed=40 + world, bias=bias)
    em = EmulatedRanks(world, p_local, T, h, f, act, inp)
    try:
        X, dY, b2 = dev(inp.X), dev(inp.dY), dev(inp.b2)
        res = (dev(inp.X) * 0.5).contiguous()
        em.forward(X, b2, res, epoch=1)
        em.backward(X, dY, epoch=2)
        assert em.status() == 0, "a peer wait gave up"
        Y0, dX0 = em.Y[0].clone(), em.dX[0].clone()
        for r in range(1, world):
            assert torch.equal(em.Y[r], Y0), f"rank {r}'s Y differs from rank 0's"
            assert torch.equal(em.dX[r], dX0), f"rank {r}'s dX differs from rank 0's"
        Xo, W1, W2, dYo = (O.f64(t) for t in (inp.X, inp.W1, inp.W2, inp.dY))
        b1o = O.f64(inp.b1) if bias else None
        b2o = O.f64(inp.b2) if bias else None
        ref = O.mlp_fwd(Xo, W1, b1o, W2, b2o, act, residual=O.f64(res))
        gr = O.mlp_bwd(Xo, W1, W2, ref["Z"], ref["H"], dYo, act)
        assert_close(Y0, ref["Y"], TOL_BF16, "Y")
        assert_close(dX0, gr["dX"], TOL_BF16, "dX")
        P = world * p_local
        for r, k in enumerate(em.ranks):      # weight gradients of the rank's global shards
            for j in range(p_local):
                i = r * p_local + j
                dW1_i = O.shard_gate_up(gr["dW1"], P, i) if act == "swiglu" else O.shard_rows(gr["dW1"], P, i)
                assert_close(k["dW1"][j], dW1_i, TOL_BF16, f"dW1 shard {i}")
                assert_close(k["dW2"][j], O.shard_cols(gr["dW2"], P, i), TOL_BF16, f"dW2 shard {i}")
                if bias:
                    assert_close(k["db1"][j][None, :], O.shard_vec(gr["db1"], P, i)[None, :], TOL_BF16,
                                 f"db1 shard {i}")
        # the next epochs reuse the buffers and flags and repeat the result exactly
        for y in em.Y:
            y.zero_()
        em.forward(X, b2, res, epoch=3)
        em.backward(X, dY, epoch=4)
        assert em.status() == 0
        for r in range(world):
            assert torch.equal(em.Y[r], Y0) and torch.equal(em.dX[r], dX0), f"rank {r}: second round differs"
    finally:
        em.close()


def test_peer_reduce_scatter_sequence_parallel_emulated():
    """n_out = 1: each rank keeps its own row block (the Megatron-SP
    reduce-scatter), with bias and the rank's residual shard added once."""
    world, p_local, T, h, f = 4, 1, 256, 256, 1024
    inp = tp_synth.draw_mlp(T, h, f, "gelu", torch.bfloat16, seed=51, bias=True)
    em = EmulatedRanks(world, p_local, T, h, f, "gelu", inp)
    try:
        t = T // world
        X, b2 = dev(inp.X), dev(inp.b2)
        res = (dev(inp.X) * -0.25).contiguous()
        Y_seq = [torch.empty(t, h, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
        em.forward(X, b2, res, epoch=1, sp=True, Y_seq=Y_seq)
        assert em.status() == 0
        Xo, W1, W2 = (O.f64(v) for v in (inp.X, inp.W1, inp.W2))
        ref = O.mlp_fwd(Xo, W1, O.f64(inp.b1), W2, O.f64(inp.b2), "gelu", residual=O.f64(res))
        for r in range(world):
            assert_close(Y_seq[r], ref["Y"][r * t:(r + 1) * t], TOL_BF16, f"Y_seq[{r}]")
    finally:
        em.close()


def test_peer_wait_times_out_without_arrivals():
    """A wait on flags that nothing raises gives up after the wait limit, sets
    TP_ERR_TIMEOUT in the device status word and leaves the context usable."""
    from megatron_tensor_transformer_gemm_b200 import tp
    world, T, h = 2, 64, 128
    mem = [tp.peer_alloc(tp.PEER_FLAG_BYTES + 2 * T * h)[0] for _ in range(world)]
    out = torch.full((T // world, h), 7.0, dtype=torch.bfloat16, device="cuda")
    try:
        g = tp.peer_group(world, 0, T * h, mem, [q + tp.PEER_FLAG_BYTES for q in mem])
        tp.peer_set_wait_limit(2_000_000)   # 2 ms
        tp.peer_wait(g, 1)
        torch.cuda.synchronize()
        assert tp.lib.tp_get_device_status(None, None) == tp.STATUS.index("TP_ERR_TIMEOUT")
        tp.peer_reduce(g, T, h, None, None, [out], 1)   # no block arrived: the reduce must not write
        torch.cuda.synchronize()
        assert tp.lib.tp_get_device_status(None, None) == tp.STATUS.index("TP_ERR_TIMEOUT")
        assert bool((out == 7.0).all()), "a reduce that gave up wrote its output"
        assert tp.lib.tp_get_device_status(None, None) == 0   # read-and-clear
    finally:
        tp.peer_set_wait_limit(0)
        torch.cuda.synchronize()
        for q in mem:
            tp.peer_free(q)


_CHILD = r"""
import sys, torch
from megatron_tensor_transformer_gemm_b200 import tp
from megatron_tensor_transformer_gemm_b200.dist import bf16_view
rows, h = int(sys.argv[2]), int(sys.argv[3])
torch.cuda.set_device(0)
ptr = tp.peer_open(bytes.fromhex(sys.argv[1]))
plan = tp.Plan(h, 0, 0, 1, "bf16", "none")
src = bf16_view(ptr, (rows, h), "cuda")
got = torch.empty(rows, h, dtype=torch.bfloat16, device="cuda")
plan.all_gather_seq(rows, [src], got)            # libtp's copy kernel reads the mapped memory
back = (got.float() + 1.0).to(torch.bfloat16)
plan.all_gather_seq(rows, [back], src)           # and writes into it
torch.cuda.synchronize()
print(float(got.float().sum()))
tp.peer_close(ptr)
"""


def test_peer_memory_maps_into_another_process():
    """tp_peer_alloc's handle opened in a second process on the same GPU
    (tp_peer_open): the child reads the parent's values through the mapping
    with libtp's copy kernel and writes values + 1 back. No kernel waits for
    the other process."""
    from megatron_tensor_transformer_gemm_b200 import tp
    from megatron_tensor_transformer_gemm_b200.dist import bf16_view
    rows, h = 64, 256
    ptr, handle = tp.peer_alloc(2 * rows * h)
    try:
        v = bf16_view(ptr, (rows, h), "cuda")
        vals = (torch.arange(rows * h, device="cuda") % 251 - 125).to(torch.bfloat16).view(rows, h)
        v.copy_(vals)
        torch.cuda.synchronize()
        r = subprocess.run([sys.executable, "-c", _CHILD, handle.hex(), str(rows), str(h)], cwd=ROOT,
                           capture_output=True, text=True, timeout=300,
                           env=dict(os.environ, PYTHONPATH=ROOT))
        assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
        assert float(r.stdout.strip().splitlines()[-1]) == float(vals.float().sum())
        assert torch.equal(v, (vals.float() + 1.0).to(torch.bfloat16))
    finally:
        torch.cuda.synchronize()
        tp.peer_free(ptr)


def test_peer_steps_at_the_edges():
    """T = 0 still takes every flag step (the epochs stay in step across the
    ranks), and the largest group, 16 emulated ranks of one shard each, sums
    and gathers like the smaller ones."""
    from megatron_tensor_transformer_gemm_b200 import tp
    world, T, h, f = 16, 512, 128, 512
    inp = tp_synth.draw_mlp(T, h, f, "gelu", torch.bfloat16, seed=61)
    em = EmulatedRanks(world, 1, T, h, f, "gelu", inp)
    try:
        X = dev(inp.X)
        # an empty exchange first: no rows, but every rank's flags advance to epoch 1
        for r, k in enumerate(em.ranks):
            k["plan"].row_fwd_push_peer("mlp", 0, k["H"], k["W2"], em.g[r], 1)
        for r in range(world):
            tp.peer_reduce(em.g[r], 0, h, None, None, em.blocks(em.Yptr, r), 1)
        for r in range(world):
            tp.peer_wait(em.g[r], 1)
        assert em.status() == 0
        em.forward(X, None, None, epoch=2)
        assert em.status() == 0
        Xo, W1, W2 = (O.f64(v) for v in (inp.X, inp.W1, inp.W2))
        ref = O.mlp_fwd(Xo, W1, None, W2, None, "gelu")
        for r in range(world):
            assert torch.equal(em.Y[r], em.Y[0])
        assert_close(em.Y[0], ref["Y"], TOL_BF16, "Y")
    finally:
        em.close()


@pytest.mark.parametrize("world,t,h", [(2, 64, 256), (3, 40, 128), (8, 32, 512)])
def test_peer_all_gathers_emulated(world, t, h):
    """The Megatron-SP all-gathers over peer memory with `world` emulated
    ranks (all pushes, then all waits): every rank's gathered buffer equals
    the concatenation of the shards bit for bit (tp_all_gather_push_peer), and
    with the LayerNorm fused in (tp_layernorm_all_gather_push_peer) equals the
    single-GPU LayerNorm + all-gather bit for bit (same arithmetic) and the
    oracle's LayerNorm within the bf16 tolerance; mean and rstd match too."""
    from megatron_tensor_transformer_gemm_b200 import tp
    from megatron_tensor_transformer_gemm_b200.dist import bf16_view
    T = world * t
    gen = torch.Generator().manual_seed(70 + world)
    xs = [torch.randn(t, h, generator=gen).to(torch.bfloat16).cuda() for _ in range(world)]
    gamma = (1 + 0.1 * torch.randn(h, generator=gen)).to(torch.bfloat16).cuda()
    beta = (0.1 * torch.randn(h, generator=gen)).to(torch.bfloat16).cuda()
    mem = [tp.peer_alloc(tp.PEER_FLAG_BYTES + 2 * T * h)[0] for _ in range(world)]
    outs = [tp.peer_alloc(2 * T * h)[0] for _ in range(world)]
    try:
        g = [tp.peer_group(world, r, T * h, mem, [q + tp.PEER_FLAG_BYTES for q in mem]) for r in range(world)]
        U = [bf16_view(q, (T, h), "cuda") for q in outs]
        blocks = lambda r: [q + r * t * h * 2 for q in outs]
        for r in range(world):
            tp.all_gather_push_peer(g[r], t, h, xs[r], blocks(r), 1)
        for r in range(world):
            tp.peer_wait(g[r], 1)
        torch.cuda.synchronize()
        assert tp.lib.tp_get_device_status(None, None) == 0
        full = torch.cat(xs)
        for r in range(world):
            assert torch.equal(U[r], full), f"rank {r}'s gathered buffer"
        plan = tp.Plan(h, 0, 0, 1, "bf16", "none")
        mean = [torch.empty(t, dtype=torch.float32, device="cuda") for _ in range(world)]
        rstd = [torch.empty(t, dtype=torch.float32, device="cuda") for _ in range(world)]
        for r in range(world):
            plan.layernorm_all_gather_push_peer(g[r], t, xs[r], gamma, beta, blocks(r), mean[r], rstd[r], 2)
        for r in range(world):
            tp.peer_wait(g[r], 2)
        ref = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
        mref = torch.empty(T, dtype=torch.float32, device="cuda")
        rref = torch.empty(T, dtype=torch.float32, device="cuda")
        plan.layernorm_all_gather_seq(T, xs, gamma, beta, ref, mref, rref)
        torch.cuda.synchronize()
        assert tp.lib.tp_get_device_status(None, None) == 0
        for r in range(world):
            assert torch.equal(U[r], ref), f"rank {r}'s LayerNorm all-gather"
        assert torch.equal(torch.cat(mean), mref) and torch.equal(torch.cat(rstd), rref)
        y, _, _ = O.layernorm_fwd(O.f64(full), O.f64(gamma), O.f64(beta))
        assert_close(U[0], y, TOL_BF16, "LayerNorm")
    finally:
        torch.cuda.synchronize()
        for q in mem + outs:
            tp.peer_free(q)
