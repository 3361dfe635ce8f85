"""Matrix ownership across ranks and the one exchange step of a sharded step.

The modded-nanogpt 2024-11-10 record write-up (section "训练管线与系统实现 /
四路优化器分工") runs Muon data-parallel: matrix i is updated on rank
i % world_size and the updates are exchanged with one all-reduce of a
zero-padded flat buffer.  Here each matrix is owned by one rank chosen by
longest-processing-time-first on its Newton-Schulz cost (the modulo rule is
unbalanced for mixed shapes), each rank's owned parameters sit contiguously
in its slice of one flat buffer, and a single all-gather of that buffer
replaces the all-reduce (half the bytes, no zero padding beyond the slice
alignment).  Everything here is host-side planning plus one
``torch.distributed`` collective; the step itself runs in the library.
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence, Tuple


def matrix_cost(m: int, n: int, ns_steps: int = 12, polars: int = 1) -> float:
    """Nominal Newton-Schulz flops of one matrix (plus its element-wise passes)."""
    s, l = min(m, n), max(m, n)
    return polars * ns_steps * (4.0 * s * s * l + 2.0 * s ** 3) + 64.0 * m * n


def step_costs(shapes: Sequence[Tuple[int, int]], ns_steps: int = 12, aurora: bool = True,
               pp_iterations: int = 2) -> List[float]:
    out = []
    for m, n in shapes:
        polars = pp_iterations if (aurora and m != n) else 1
        out.append(matrix_cost(m, n, ns_steps, polars))
    return out


def lpt_partition(costs: Sequence[float], world: int) -> List[List[int]]:
    """Greedy longest-processing-time assignment; deterministic (ties: lower index, lower rank)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    load = [0.0] * world
    owned: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owned[r].append(i)
        load[r] += costs[i]
    return [sorted(o) for o in owned]


def modulo_partition(n: int, world: int) -> List[List[int]]:
    """The pages' rule: matrix i on rank i % world."""
    return [[i for i in range(n) if i % world == r] for r in range(world)]


@dataclasses.dataclass
class FlatLayout:
    """Placement of every matrix in a [world, shard_elems] flat parameter buffer."""
    world: int
    shard_elems: int
    owner: List[int]              # rank owning each matrix
    offset: List[int]             # element offset of each matrix inside the whole flat buffer

    @property
    def total_elems(self) -> int:
        return self.world * self.shard_elems


def flat_layout(shapes: Sequence[Tuple[int, int]], owned: List[List[int]], align_elems: int = 64) -> FlatLayout:
    world = len(owned)
    owner = [-1] * len(shapes)
    local = [0] * len(shapes)
    sizes = []
    for r, ids in enumerate(owned):
        off = 0
        for i in ids:
            owner[i] = r
            local[i] = off
            m, n = shapes[i]
            off += (m * n + align_elems - 1) // align_elems * align_elems
        sizes.append(off)
    if any(o < 0 for o in owner):
        raise ValueError("every matrix needs an owner")
    shard = max(sizes) if sizes else 0
    shard = max(align_elems, (shard + align_elems - 1) // align_elems * align_elems)
    offset = [owner[i] * shard + local[i] for i in range(len(shapes))]
    return FlatLayout(world, shard, owner, offset)


def views(flat, layout: FlatLayout, shapes: Sequence[Tuple[int, int]]):
    """Per-matrix views into the flat buffer (any torch tensor with .narrow/.view)."""
    return [flat.narrow(0, layout.offset[i], m * n).view(m, n) for i, (m, n) in enumerate(shapes)]


def exchange(flat, layout: FlatLayout, rank: int, group=None):
    """All-gather every rank's slice so each rank holds all updated parameters."""
    import torch.distributed as dist
    mine = flat.narrow(0, rank * layout.shard_elems, layout.shard_elems)
    dist.all_gather_into_tensor(flat, mine, group=group)
