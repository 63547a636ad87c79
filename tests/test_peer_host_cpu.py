"""Host logic of the peer-memory exchange (dist.py PeerMemory / PeerGroup /
DistTPMLP._blocks) on CPU gloo ranks, world size 2 and 3, with libtp's
device calls (tp_peer_alloc / open / close / free) replaced by fakes that
hand out and record synthetic addresses: every rank must see every other
rank's block through exactly the handle that rank published, its own block
through its own pointer, the tp_peer_group fields in rank order, the receive
buffers behind the flag words, and each rank's row block of an output at
rank * (T / world) rows on every rank. No device memory is touched."""
import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from megatron_tensor_transformer_gemm_b200 import dist as D
    from megatron_tensor_transformer_gemm_b200 import tp

    log = {"opened": [], "closed": [], "freed": []}
    base = (rank + 1) << 40

    def fake_alloc(nbytes):
        ptr = base + 4096 * len(log.setdefault("allocs", []))
        log["allocs"].append((ptr, nbytes))
        return ptr, ptr.to_bytes(8, "little") + bytes(tp.PEER_HANDLE_BYTES - 8)

    def fake_open(handle):
        owner_ptr = int.from_bytes(handle[:8], "little")
        mapped = owner_ptr + (1 << 36) * (rank + 1)   # another address for the same block
        log["opened"].append((owner_ptr, mapped))
        return mapped

    tp.peer_alloc = fake_alloc
    tp.peer_open = fake_open
    tp.peer_close = lambda p: log["closed"].append(p)
    tp.peer_free = lambda p: log["freed"].append(p)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        T, h = 12 * world, 32
        g = D.PeerGroup(T * h, device="cpu")
        # what each rank allocated, gathered, to check the mapping of every block
        allocs = [None] * world
        dist.all_gather_object(allocs, log["allocs"][0][0])
        res["world_rank"] = (g.world, g.rank) == (world, rank)
        res["own_ptr"] = g.mem.ptrs[rank] == allocs[rank]
        res["peers"] = all(g.mem.ptrs[d] == allocs[d] + (1 << 36) * (rank + 1)
                           for d in range(world) if d != rank)
        res["opened_each_peer_once"] = sorted(o for o, _ in log["opened"]) == \
            sorted(allocs[d] for d in range(world) if d != rank)
        res["size"] = log["allocs"][0][1] == tp.PEER_FLAG_BYTES + 2 * T * h
        c = g.c
        res["struct"] = (c.world == world and c.rank == rank and c.recv_elems == T * h and
                         all(c.flags[d] == g.mem.ptrs[d] for d in range(world)) and
                         all(c.recv[d] == g.mem.ptrs[d] + tp.PEER_FLAG_BYTES for d in range(world)))
        res["epochs"] = [g.next_epoch() for _ in range(3)] == [1, 2, 3]
        g.epoch = 0xFFFFFFFF
        res["epoch_wraps"] = g.next_epoch() == 0
        # DistTPMLP._blocks: this rank's row block on every rank's output
        m = object.__new__(D.DistTPMLP)
        m.rank, m.world, m.h = rank, world, h
        out = D.PeerMemory(2 * T * h, device="cpu")
        blocks = m._blocks(out, T)
        res["blocks"] = blocks == [q + rank * (T // world) * h * 2 for q in out.ptrs]
        out.close()
        g.close()
        res["closed"] = sorted(log["closed"]) == sorted(
            [mp_ for _, mp_ in log["opened"]])
        res["freed"] = sorted(log["freed"]) == sorted(p for p, _ in log["allocs"])
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 3])
def test_peer_exchange_host_logic_on_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31700 + (os.getpid() % 1000) + 10 * world
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    out = sorted(q.get(timeout=200) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    assert [r for r, _ in out] == list(range(world))
    for rank, res in out:
        for k, v in res.items():
            assert v, (rank, k)
