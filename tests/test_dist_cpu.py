"""Host logic of tensor parallelism across ranks (dist.py) on CPU gloo ranks,
world size 2 and 4: which shards a rank owns, the weight slices that make its
local split equal the global one, and the exchange steps (all-reduce,
sequence reduce-scatter and all-gather) with the bias / residual entering
once. Each rank's local partial sums come from the oracle; integer-valued
data make every sum exact, so the collective results are checked bit for bit
against the oracle's single-process definitions."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _ints(gen, *shape):
    return torch.randint(-8, 9, shape, generator=gen).double()


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import oracle as O
    from megatron_tensor_transformer_gemm_b200 import dist as D
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        p, T, h, f = 8, 8 * world, 16, 64
        gen = torch.Generator().manual_seed(5)            # same draws on every rank
        W1 = _ints(gen, 2 * f, h)
        W2 = _ints(gen, h, f)
        H = [_ints(gen, T, f // p) for _ in range(p)]
        b2 = _ints(gen, h)
        resid = _ints(gen, T, h)
        sh = D.rank_shards(p, world, rank)
        # 1. the rank's weight slices, split locally, are the global shards it owns
        pl = p // world
        for act in ("swiglu", "gelu"):
            W1a = W1 if act == "swiglu" else W1[:f]
            W1r, W2r = D.local_mlp_weights(W1a, W2, p, world, rank, act)
            for j, i in enumerate(sh):
                if act == "swiglu":
                    ok1 = np.array_equal(O.shard_gate_up(W1r.numpy(), pl, j), O.shard_gate_up(W1a.numpy(), p, i))
                else:
                    ok1 = np.array_equal(O.shard_rows(W1r.numpy(), pl, j), O.shard_rows(W1a.numpy(), p, i))
                ok2 = np.array_equal(O.shard_cols(W2r.numpy(), pl, j), O.shard_cols(W2.numpy(), p, i))
                res.setdefault("slices", []).append(bool(ok1 and ok2))
        # 2. all-reduce of the local shard sums, bias and residual once (rank 0)
        Hn = [x.numpy() for x in H]
        parts = [O.row_partial(Hn[i], O.shard_cols(W2.numpy(), p, i)) for i in range(p)]
        local = O.reduce_partials([parts[i] for i in sh])
        b = D.once_on_rank0(b2, rank)
        r = D.once_on_rank0(resid, rank)
        if b is not None:
            local = local + b.numpy()[None, :]
        if r is not None:
            local = local + r.numpy()
        Y = D.sum_over_ranks(torch.from_numpy(local.copy()))
        res["allreduce"] = bool(np.array_equal(Y.numpy(), O.reduce_partials(parts, b2.numpy(), resid.numpy())))
        # the bias on every rank instead would be (world - 1) * b too much
        wrong = D.sum_over_ranks(torch.from_numpy(O.reduce_partials([parts[i] for i in sh]) + b2.numpy()[None, :]))
        res["bias_once_matters"] = bool(np.array_equal(
            wrong.numpy() - O.reduce_partials(parts, b2.numpy()),
            np.broadcast_to((world - 1) * b2.numpy(), (T, h))))
        # 3. Megatron-SP: reduce-scatter of the full-shape local sums
        local_nb = O.reduce_partials([parts[i] for i in sh])
        if rank == 0:
            local_nb = local_nb + b2.numpy()[None, :]
        out = torch.empty(T // world, h, dtype=torch.float64)
        D.scatter_seq_sum(torch.from_numpy(local_nb.copy()), out)
        ref = O.reduce_scatter_seq(parts, b2.numpy())
        # the oracle scatters over len(P) = p shards; the ranks own world blocks of rows
        rows = slice(rank * (T // world), (rank + 1) * (T // world))
        res["reduce_scatter"] = bool(np.array_equal(out.numpy(), O.all_gather_seq(ref)[rows]))
        # 4. all-gather along the sequence
        shard = torch.from_numpy(Y.numpy()[rows].copy())
        full = torch.empty(T, h, dtype=torch.float64)
        D.gather_seq(shard, full)
        res["all_gather"] = bool(np.array_equal(full.numpy(), Y.numpy()))
        res["shards"] = list(sh)
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 4])
def test_dist_host_logic_on_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 30500 + (os.getpid() % 1000) + 10 * world
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    out = sorted(q.get(timeout=200) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    owned = []
    for rank, res in out:
        assert all(res["slices"]), (rank, res["slices"])
        assert res["allreduce"], rank
        assert res["bias_once_matters"], rank
        assert res["reduce_scatter"], rank
        assert res["all_gather"], rank
        owned += res["shards"]
    assert owned == list(range(8))      # every shard owned by exactly one rank, in order


def test_rank_shards_rejects_uneven_splits():
    sys.path.insert(0, ROOT)
    from megatron_tensor_transformer_gemm_b200 import dist as D
    assert list(D.rank_shards(8, 4, 3)) == [6, 7]
    with pytest.raises(ValueError):
        D.rank_shards(8, 3, 0)
    with pytest.raises(ValueError):
        D.rank_shards(8, 2, 2)
