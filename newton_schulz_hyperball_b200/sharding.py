"""Data-parallel sharding of the optimizer step across ranks (one process per GPU).

Every matrix's step is independent ("Muon: the orthogonalized optimizer explained", the
per-parameter Muon.step loop; "Hierarchical Muon", independent tiles), so under data
parallelism each rank owns a subset of the matrices: it keeps their momentum buffers,
runs the step for them only, and then every rank receives the updated weights of all
matrices in one all-gather (NCCL over NVLink on GPUs, gloo on CPU).

Ownership is a greedy longest-processing-time partition by Newton-Schulz work, so the
ranks finish their local steps at about the same time.  Before the step, the gradients
that every rank computed on its own batch are summed (or averaged) onto the owner of each
matrix with one reduce-scatter, so the owner holds its matrices' full gradients.

`sharded_step` takes the local step as a callable (the tests pass the oracle on CPU);
`ShardedOptimizer` drives the library's own step on the owned matrices.  The exchange
uses only collectives of torch.distributed (NCCL or gloo): peer data arrives in local
memory before any kernel reads it.
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

    def owned_by(self, k):
        """Indices of the matrices rank k owns, in global order."""
        return [i for i, r in enumerate(self.owner) if r == k]

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


def reduce_scatter_grads(grads, plan: ShardPlan, out, group=None, average: bool = True) -> None:
    """The owner of every matrix receives the sum over ranks of that matrix's gradient.

    grads: this rank's gradient of every matrix (its own batch), one dtype and device.
    out: one buffer per matrix this rank owns (the order of plan.local), of the gradient's
    shape; it receives the sum over ranks, divided by the world size when `average`.
    Each rank packs its gradients owner by owner into one flat buffer (segment k holds
    rank k's matrices, padded to the largest segment) and a single reduce_scatter_tensor
    leaves segment `rank`, summed over the ranks, on this rank."""
    import torch.distributed as dist
    world = plan.world
    local = plan.local
    if len(out) != len(local):
        raise ValueError("out needs one buffer per owned matrix")
    if world == 1:
        for o, i in zip(out, local):
            o.copy_(grads[i])
        return
    dtype = grads[0].dtype
    device = grads[0].device
    if any(g.dtype != dtype or g.device != device for g in grads):
        raise ValueError("reduce_scatter_grads needs every gradient in one dtype on one device")
    per_rank = [plan.owned_by(k) for k in range(world)]
    cap = max(sum(grads[i].numel() for i in idx) for idx in per_rank)
    send = torch.zeros(world * cap, dtype=dtype, device=device)
    for k in range(world):
        off = k * cap
        for i in per_rank[k]:
            n = grads[i].numel()
            send[off:off + n].copy_(grads[i].reshape(-1))
            off += n
    recv = torch.empty(cap, dtype=dtype, device=device)
    dist.reduce_scatter_tensor(recv, send, op=dist.ReduceOp.SUM, group=group)
    if average:
        recv.div_(world)
    off = 0
    for o, i in zip(out, local):
        n = grads[i].numel()
        o.copy_(recv[off:off + n].view(o.shape))
        off += n


def sharded_step(step_fn, weights, plan: ShardPlan, group=None) -> None:
    """Runs `step_fn(local_indices)` (which updates those weights in place) and exchanges
    the results so that every rank ends with all updated weights."""
    step_fn(plan.local)
    all_gather_weights(weights, plan, group)


class ShardedOptimizer:
    """Data-parallel optimizer step over the ranks of a process group, on the library.

    weights: every matrix's weight (CUDA, one dtype), identical on every rank; rho: a CUDA
    float32 tensor with every matrix's radius.  Each rank keeps the momentum buffers and
    the gradient buffers of the matrices it owns (LPT by NS work), and one step is

        reduce-scatter of the ranks' gradients onto the owners (sum, or mean)
        -> the library's step ("hyperball", "muon", "brake" or "himuon") on the owned matrices
        -> all-gather of the updated weights.

    Keyword arguments go to the library's nshb_params (eta, tile, lr, ...)."""

    def __init__(self, weights, rho, plan: ShardPlan, kind: str = "hyperball", group=None, average: bool = True,
                 **params):
        import newton_schulz_hyperball_b200 as nshb
        self.nshb = nshb
        self.W = weights
        self.plan = plan
        self.group = group
        self.average = average
        self.local = plan.local
        dev = weights[0].device
        self.G = [torch.empty_like(weights[i]) for i in self.local]
        self.M = [torch.zeros(weights[i].shape, dtype=torch.float32, device=dev) for i in self.local]
        self.kind = kind
        self.fn = {"hyperball": nshb.hyperball_step, "muon": nshb.muon_step, "brake": nshb.radial_brake_step,
                   "himuon": nshb.himuon_step}[kind]
        op = {"hyperball": nshb.NSHB_OP_HYPERBALL, "muon": nshb.NSHB_OP_MUON, "brake": nshb.NSHB_OP_RADIAL_BRAKE,
              "himuon": nshb.NSHB_OP_HIMUON}[kind]
        self.mats = None
        if self.local:
            idx = torch.tensor(self.local, dtype=torch.long, device=rho.device)
            self.rho = rho.index_select(0, idx).contiguous()
            if kind in ("hyperball", "himuon"):
                params["rho"] = self.rho
            self.p = nshb.params(**params)
            self.mats = nshb.matrices([weights[i] for i in self.local], self.G, self.M)
            self.ws = nshb.workspace(self.mats, self.p, op, device=dev)

    def step(self, grads, stream=None) -> None:
        """One step with this rank's gradients of every matrix (`grads`, in matrix order)."""
        reduce_scatter_grads(grads, self.plan, self.G, self.group, self.average)
        self.local_step(stream)
        all_gather_weights(self.W, self.plan, self.group)

    def local_step(self, stream=None) -> None:
        """The library's step on the owned matrices, with the gradients already in self.G."""
        if self.mats is not None:
            self.fn(self.mats, self.p, self.ws, stream)

    def device_status(self) -> int:
        return self.nshb.device_status(self.ws) if self.mats is not None else 0
