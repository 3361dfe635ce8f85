"""Matrix ownership plan and the exchange step of the sharded optimizer step,
on CPU ranks (gloo, world_size 2 and 3)."""
import os
import socket

import numpy as np
import pytest

import workloads as WL
from aurora_orthogonalised_optimizer_b200 import sharding as SH


def test_lpt_assigns_each_matrix_once_and_is_deterministic():
    shapes = WL.llama_3p8b_shapes()
    costs = SH.step_costs(shapes)
    for world in (1, 2, 3, 4, 8):
        owned = SH.lpt_partition(costs, world)
        flat = sorted(i for o in owned for i in o)
        assert flat == list(range(len(shapes)))
        assert owned == SH.lpt_partition(costs, world)


def test_lpt_balances_better_than_modulo():
    shapes = WL.llama_3p8b_shapes()
    costs = np.array(SH.step_costs(shapes))
    for world in (2, 4, 8):
        lpt = max(costs[o].sum() for o in map(np.array, SH.lpt_partition(costs, world)))
        mod = max(costs[o].sum() for o in map(np.array, SH.modulo_partition(len(shapes), world)))
        ideal = costs.sum() / world
        assert lpt <= mod
        assert lpt / ideal < 1.05


def test_lpt_single_rank_and_more_ranks_than_matrices():
    assert SH.lpt_partition([3.0, 1.0], 1) == [[0, 1]]
    owned = SH.lpt_partition([3.0, 1.0], 4)
    assert sorted(i for o in owned for i in o) == [0, 1]
    with pytest.raises(ValueError):
        SH.lpt_partition([1.0], 0)


def test_flat_layout_disjoint_and_aligned():
    shapes = WL.gpt2_124m_shapes()
    owned = SH.lpt_partition(SH.step_costs(shapes), 3)
    lay = SH.flat_layout(shapes, owned, align_elems=64)
    spans = sorted((lay.offset[i], lay.offset[i] + m * n) for i, (m, n) in enumerate(shapes))
    for (a0, a1), (b0, _) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert spans[-1][1] <= lay.total_elems
    for i in range(len(shapes)):
        assert lay.offset[i] % 64 == 0
        r = lay.owner[i]
        assert r * lay.shard_elems <= lay.offset[i] < (r + 1) * lay.shard_elems


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, shapes, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        owned = SH.lpt_partition(SH.step_costs(shapes), world)
        lay = SH.flat_layout(shapes, owned)
        flat = torch.full((lay.total_elems,), -1.0, dtype=torch.float32)
        v = SH.views(flat, lay, shapes)
        for i in owned[rank]:                       # "update" only the matrices this rank owns
            v[i].fill_(float(i + 1))
        SH.exchange(flat, lay, rank)
        ok = all(bool(torch.all(v[i] == float(i + 1))) for i in range(len(shapes)))
        q.put((rank, ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shapes", [
    (2, [(48, 16), (16, 48), (32, 32), (8, 100), (100, 8)]),
    (3, [(48, 16), (16, 48), (32, 32), (8, 100), (100, 8)]),
    (3, [(48, 16), (16, 48)]),                          # one rank owns nothing
])
def test_exchange_gives_every_rank_every_update(world, shapes):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shapes, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert all(res[r] for r in range(world)), res
