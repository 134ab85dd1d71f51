"""Data-parallel sharding of the optimizer step across ranks (one process per GPU).

Every matrix's step is independent ("Muon: the orthogonalized optimizer explained", the
per-parameter Muon.step loop; "Hierarchical Muon", independent tiles), so under data
parallelism each rank owns a subset of the matrices: it keeps their momentum buffers,
runs the step for them only, and then every rank receives the updated weights of all
matrices in one all-gather (NCCL over NVLink on GPUs, gloo on CPU).

Ownership is a greedy longest-processing-time partition by Newton-Schulz work, so the
ranks finish their local steps at about the same time.  This module holds only host-side
bookkeeping and the exchange; the step itself is whatever callable the caller passes
(normally the library's hyperball_step on the owned matrices).
"""
from __future__ import annotations

import heapq
from dataclasses import dataclass

import torch


def ns_cost(rows: int, cols: int, steps: int = 5) -> float:
    """NS work of one matrix: K (3 r^2 s + r^3), r = min, s = max (symmetric products once)."""
    r, s = min(rows, cols), max(rows, cols)
    return float(steps) * (3.0 * r * r * s + r ** 3)


def lpt_partition(costs, world: int):
    """Owner rank of every item: items in decreasing cost go to the least-loaded rank
    (ties to the lower rank; equal costs keep their input order)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    heap = [(0.0, r) for r in range(world)]
    owner = [0] * len(costs)
    for i in order:
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + costs[i], r))
    return owner


@dataclass
class ShardPlan:
    owner: list          # owner rank per matrix
    world: int
    rank: int

    @property
    def local(self):
        """Indices of the matrices this rank owns, in global order."""
        return [i for i, r in enumerate(self.owner) if r == self.rank]

    def loads(self, costs):
        out = [0.0] * self.world
        for i, r in enumerate(self.owner):
            out[r] += costs[i]
        return out


def make_plan(shapes, world: int, rank: int, steps: int = 5) -> ShardPlan:
    costs = [ns_cost(r, c, steps) for r, c in shapes]
    return ShardPlan(lpt_partition(costs, world), world, rank)


def all_gather_weights(weights, plan: ShardPlan, group=None) -> None:
    """In place: every rank's copy of matrix i becomes the owner's copy.

    The owned matrices of each rank are packed into one flat buffer (padded to the
    largest rank's size) and exchanged with a single all_gather_into_tensor; each rank
    then unpacks every other rank's matrices into place.  All weights share one dtype and
    device (the buffer is of that dtype, so a mixed set would be rounded); any strides."""
    import torch.distributed as dist
    world = plan.world
    if world == 1 or not weights:
        return
    dtype = weights[0].dtype
    device = weights[0].device
    if any(w.dtype != dtype or w.device != device for w in weights):
        raise ValueError("all_gather_weights needs every weight in one dtype on one device")
    per_rank = [[i for i, r in enumerate(plan.owner) if r == k] for k in range(world)]
    sizes = [sum(weights[i].numel() for i in idx) for idx in per_rank]
    cap = max(sizes)
    send = torch.zeros(cap, dtype=dtype, device=device)
    off = 0
    for i in per_rank[plan.rank]:
        n = weights[i].numel()
        send[off:off + n].copy_(weights[i].reshape(-1))
        off += n
    recv = torch.empty(world * cap, dtype=dtype, device=device)
    if hasattr(dist, "all_gather_into_tensor") and device.type == "cuda":
        dist.all_gather_into_tensor(recv, send, group=group)
    else:
        dist.all_gather(list(recv.chunk(world)), send, group=group)
    for k in range(world):
        if k == plan.rank:
            continue
        base = k * cap
        off = 0
        for i in per_rank[k]:
            n = weights[i].numel()
            weights[i].copy_(recv[base + off:base + off + n].view(weights[i].shape))
            off += n


def sharded_step(step_fn, weights, plan: ShardPlan, group=None) -> None:
    """Runs `step_fn(local_indices)` (which updates those weights in place) and exchanges
    the results so that every rank ends with all updated weights."""
    step_fn(plan.local)
    all_gather_weights(weights, plan, group)
