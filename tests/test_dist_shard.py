"""Token-sharded layer, host side, on CPU: the exchange step over world-size-2 and -3 gloo groups
(every shard's demand gathered in rank order, the integer statistics partials summed exactly),
and the identity the shard kernels rely on: first-come slots over the whole batch equal each
shard's local first-come positions offset by the earlier shards' demand, cut at the batch's C."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, E, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from mixture_experts_layer_57_b200 import moe
    dist.init_process_group("gloo", rank=rank, world_size=world)
    g = torch.Generator().manual_seed(100 + rank)
    demand = torch.randint(0, 50, (E,), generator=g, dtype=torch.int32)
    # partials near 2^62 check that the sum is exact 64-bit integer arithmetic
    partials = torch.randint(0, 1 << 40, (4 * E + 1,), generator=g, dtype=torch.int64)
    partials[0] = (1 << 62) // world + rank
    demand_all, totals = moe.exchange_shard_routing(demand, partials)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, demand.numpy(), partials.numpy(), demand_all.numpy(), totals.numpy()))


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_gloo(world):
    E = 37
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, E, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want_all = np.stack([r[1] for r in res])
    want_tot = np.sum(np.stack([r[2] for r in res]), axis=0, dtype=np.int64)
    for r in res:
        assert np.array_equal(r[3], want_all)        # rank order
        assert np.array_equal(r[4], want_tot)        # exact int64 sums


@pytest.mark.parametrize("T,E,k,cf,shards", [
    (1000, 8, 2, 1.0, [256, 256, 488]), (777, 37, 3, 1.25, [0, 400, 377]),
    (300, 4, 1, 0.5, [100, 100, 100]), (64, 128, 1, 2.0, [64]),
])
def test_global_first_come_from_shards(T, E, k, cf, shards):
    rng = np.random.default_rng(T + E)
    p = 1.0 / np.arange(1, E + 1) ** 1.2
    p /= p.sum()
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    C = oracle.capacity(T, E, k, cf)
    slot_all, counts_all = oracle.assign_slots(ids, E, C)
    base = np.zeros(E, dtype=np.int64)
    t0 = 0
    for n in shards:
        sid = ids[t0:t0 + n]
        pos, demand = oracle.assign_slots(sid, E, 1 << 30)   # local first-come positions
        cap_local = np.clip(C - base, 0, demand)
        for t in range(n):
            for j in range(k):
                e = sid[t, j]
                want = slot_all[t0 + t, j]
                if pos[t, j] < cap_local[e]:
                    assert want == base[e] + pos[t, j]
                else:
                    assert want == -1
        base += demand
        t0 += n
    assert np.array_equal(base, counts_all)
