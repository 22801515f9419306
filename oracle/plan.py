"""Oracle of the balance-aware owner planner (test infrastructure only).

Source: "MatrixFSDP: communication-free matrix optimizers under ZeRO-3
parameter sharding", arxivlens summary page, Abstract (MatrixShard metadata and
a balance-aware owner planner; every 2D weight has exactly one data-parallel
owner, the other ranks hold empty shards; non-matrix tensors are packed into
tail owners) and the gist.science French summary, Methodologie section 2,
"Metadonnees MatrixShard & Planificateur Global" (the global planner assigns
owners so that resident bytes and optimizer work are balanced across ranks).

The pages give no algorithm.  Reading taken here (a greedy longest-processing-
time assignment on two balanced resources):

* cost of a matrix of shape rows x cols, r = min, c = max:
    Newton-Schulz FLOPs  f = steps * (4 r^2 c + 2 r^3)     (A = X X^T, A A, B X; dense count)
    resident bytes       b = rows * cols * (param + grad + fp32 momentum bytes)
                           = 8 per element for bf16 params/grads, 12 for fp32
* matrices in the order (-f, -b, parameter id);
* each goes to the rank minimising, in this order,
    max((F_r + f) / Fbar, (B_r + b) / Bbar),  then F_r + f,  then the rank id,
  with Fbar, Bbar the per-rank means of the matrices' totals;
* the tail (all non-matrix tensors, p/g/m/v in fp32 = 16 bytes per element)
  is one unit placed afterwards on the rank with the fewest resident bytes
  (lowest id on ties);
* an owner's local buffer holds its matrices in parameter-id order;
  ``owner_offset`` is the element offset of a matrix in that buffer, and of a
  tail tensor in the packed tail;
* the heaviest rank has the largest F_r, then the largest B_r, then the lowest id.

Pins (tests/test_oracle_plan.py): every parameter owned exactly once; the
result does not depend on the input order of equal items; brute-force optimal
makespan on tiny instances within Graham's LPT bound; hand-checked balance of
the Llama-shaped share plans.

Owner-shard checkpoint resharding.  Source: the gist.science French and
Portuguese summaries, Methodologie / Metodologia section 2, "Checkpointing et
Routage" (checkpoints save the placement layout, the optimizer state is routed
to the right owners through the MatrixShard metadata - Muon state for
matrices, AdamW state for tails - and resharding works across world sizes).
Reading taken here: a checkpoint holds each rank's owner-local buffers laid out
by a saved plan; restoring on another world size plans the same parameters
for the new world with the same rule, and every parameter's state is routed
from (old owner, old offset) to (new owner, new offset).  The state that
travels is the parameter and its fp32 momentum for a matrix, and fp32 p, m, v
for a tail element.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Sequence, Tuple

MATRIX = 0
TAIL = 1

_DTYPE_BYTES = {"f32": 4, "bf16": 2}


@dataclasses.dataclass(frozen=True)
class PlanEntry:
    pid: int
    rows: int
    cols: int
    kind: int
    owner: int
    transposed: bool
    ns_flops: float
    resident_bytes: int
    owner_offset: int
    shape_scale: float


def ns_flops(rows: int, cols: int, steps: int = 5) -> float:
    r, c = min(rows, cols), max(rows, cols)
    return float(steps * (4 * r * r * c + 2 * r * r * r))


def resident_bytes(rows: int, cols: int, kind: int, dtype: str) -> int:
    n = rows * cols
    if kind == TAIL:
        return 16 * n
    e = _DTYPE_BYTES[dtype]
    return n * (e + e + 4)


def plan_owners(params: Sequence, world_size: int, steps: int = 5) -> Tuple[List[PlanEntry], List[float], List[int]]:
    """Plan owners for ``params`` (objects with pid, rows, cols, kind, dtype).

    Returns (entries in input order, per-rank NS FLOPs, per-rank resident bytes).
    """
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    R = world_size
    mats = [p for p in params if p.kind == MATRIX]
    tails = [p for p in params if p.kind != MATRIX]
    cost = {p.pid: (ns_flops(p.rows, p.cols, steps), resident_bytes(p.rows, p.cols, MATRIX, p.dtype)) for p in mats}
    total_f = sum(cost[p.pid][0] for p in mats)
    total_b = sum(cost[p.pid][1] for p in mats)
    fbar = total_f / R
    bbar = total_b / R
    F = [0.0] * R
    B = [0] * R
    owner = {}
    order = sorted(mats, key=lambda p: (-cost[p.pid][0], -cost[p.pid][1], p.pid))
    for p in order:
        f, b = cost[p.pid]
        best, best_key = -1, None
        for r in range(R):
            rf = (F[r] + f) / fbar if fbar > 0 else 0.0
            rb = (B[r] + b) / bbar if bbar > 0 else 0.0
            key = (max(rf, rb), F[r] + f, r)
            if best_key is None or key < best_key:
                best, best_key = r, key
        owner[p.pid] = best
        F[best] += f
        B[best] += b
    if tails:
        tail_bytes = sum(resident_bytes(p.rows, p.cols, TAIL, "f32") for p in tails)
        t_owner = min(range(R), key=lambda r: (B[r], r))
        for p in tails:
            owner[p.pid] = t_owner
        B[t_owner] += tail_bytes
    # owner-local offsets in parameter-id order
    offsets = {}
    next_off = [0] * R
    tail_off = 0
    for p in sorted(params, key=lambda q: q.pid):
        if p.kind == MATRIX:
            offsets[p.pid] = next_off[owner[p.pid]]
            next_off[owner[p.pid]] += p.rows * p.cols
        else:
            offsets[p.pid] = tail_off
            tail_off += p.rows * p.cols
    entries = []
    for p in params:
        is_mat = p.kind == MATRIX
        entries.append(PlanEntry(
            pid=p.pid, rows=p.rows, cols=p.cols, kind=MATRIX if is_mat else TAIL,
            owner=owner[p.pid],
            transposed=bool(is_mat and p.rows > p.cols),
            ns_flops=cost[p.pid][0] if is_mat else 0.0,
            resident_bytes=cost[p.pid][1] if is_mat else resident_bytes(p.rows, p.cols, TAIL, "f32"),
            owner_offset=offsets[p.pid],
            shape_scale=math.sqrt(max(1.0, p.rows / p.cols)) if is_mat else 1.0,
        ))
    return entries, F, B


def heaviest_rank(rank_flops: Sequence[float], rank_bytes: Sequence[int]) -> int:
    return min(range(len(rank_flops)), key=lambda r: (-rank_flops[r], -rank_bytes[r], r))


@dataclasses.dataclass(frozen=True)
class ReshardRoute:
    pid: int
    kind: int
    src_rank: int
    src_offset: int
    dst_rank: int
    dst_offset: int
    elems: int
    state_bytes: int


def state_bytes(rows: int, cols: int, kind: int, dtype: str) -> int:
    """Checkpointed state per parameter: the parameter and its fp32 momentum
    (matrix) or fp32 p, m and v (tail element)."""
    n = rows * cols
    if kind == TAIL:
        return 12 * n
    return n * (_DTYPE_BYTES[dtype] + 4)


def reshard(params: Sequence, old_entries: Sequence[PlanEntry], new_world: int,
            steps: int = 5) -> Tuple[List[PlanEntry], List[ReshardRoute], int]:
    """Plan ``params`` for ``new_world`` ranks and route every parameter's
    state from its place in ``old_entries`` (a saved plan of the same
    parameters, any world size) to its place in the new plan.

    Returns (new entries, one route per parameter in input order, bytes of
    state whose owner rank changes).
    """
    if len(old_entries) != len(params):
        raise ValueError("the saved layout must describe the same parameters")
    for p, e in zip(params, old_entries):
        is_mat = p.kind == MATRIX
        if e.pid != p.pid or e.rows != p.rows or e.cols != p.cols or e.kind != (MATRIX if is_mat else TAIL):
            raise ValueError(f"saved record of parameter {p.pid} does not match its descriptor")
    new_entries, _, _ = plan_owners(params, new_world, steps)
    routes = []
    for p, old, new in zip(params, old_entries, new_entries):
        kind = MATRIX if p.kind == MATRIX else TAIL
        routes.append(ReshardRoute(
            pid=p.pid, kind=kind, src_rank=old.owner, src_offset=old.owner_offset,
            dst_rank=new.owner, dst_offset=new.owner_offset, elems=p.rows * p.cols,
            state_bytes=state_bytes(p.rows, p.cols, kind, p.dtype if kind == MATRIX else "f32")))
    moved = sum(r.state_bytes for r in routes if r.src_rank != r.dst_rank)
    return new_entries, routes, moved
