"""Multi-rank host logic on CPU: LPT ownership and the all-gather of updated weights,
run as two or three gloo ranks (spawned processes).  Each rank steps only its own matrices with the
oracle; after the exchange every rank must hold exactly the single-process result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from newton_schulz_hyperball_b200 import sharding
from newton_schulz_hyperball_b200 import workloads as wl


def test_lpt_partition_balances_gpt2_set():
    shapes = [(r, c) for _, r, c in wl.gpt2_small_shapes(12)]
    costs = [sharding.ns_cost(r, c) for r, c in shapes]
    for world in (1, 2, 4, 8):
        owner = sharding.lpt_partition(costs, world)
        assert sorted(set(owner)) == list(range(min(world, len(shapes))))
        loads = sharding.ShardPlan(owner, world, 0).loads(costs)
        # LPT bound: max load <= average + largest item
        assert max(loads) <= sum(costs) / world + max(costs) + 1e-6
    assert sharding.lpt_partition([3.0, 1.0, 2.0], 2) == [0, 1, 1]
    with pytest.raises(ValueError):
        sharding.lpt_partition([1.0], 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, shapes, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    from datetime import timedelta
    from oracle import nshb_oracle as o
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        plan = sharding.make_plan(shapes, world, rank)
        W = [torch.from_numpy(wl.init_weight(31, i, r, c, bf16=False).astype(np.float64)) for i, (r, c) in enumerate(shapes)]
        # matrix 0 held as a transposed view (non-contiguous storage), as a framework may hold it
        W[0] = W[0].t().contiguous().t()
        assert not W[0].is_contiguous()
        M = [torch.zeros_like(w) for w in W]
        rho = [float(torch.linalg.norm(w)) for w in W]
        for step in range(2):
            def step_fn(local):
                for i in local:
                    r, c = shapes[i]
                    G = wl.gradient(31, i, step, r, c, bf16=False).astype(np.float64)
                    Wn, Mn, _, _ = o.hyperball_step(W[i].numpy(), G, M[i].numpy(), eta=0.02, rho=rho[i])
                    W[i].copy_(torch.from_numpy(Wn))
                    M[i].copy_(torch.from_numpy(Mn))
            sharding.sharded_step(step_fn, W, plan)
        torch.save([w.clone() for w in W], os.path.join(out_dir, f"w{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shapes", [
    (2, [(24, 16), (16, 40), (32, 32), (8, 20), (48, 12)]),
    (3, [(24, 16), (16, 40), (32, 32), (8, 20), (48, 12)]),   # uneven ownership
    (3, [(24, 16), (16, 40)]),                                # one rank owns nothing
])
def test_gloo_ranks_match_single_process(tmp_path, world, shapes):
    from oracle import nshb_oracle as o
    mp.start_processes(_worker, args=(world, _free_port(), shapes, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = [torch.load(tmp_path / f"w{r}.pt") for r in range(world)]
    # single-process oracle
    W = [wl.init_weight(31, i, r, c, bf16=False).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    M = [np.zeros_like(w) for w in W]
    rho = [float(np.linalg.norm(w)) for w in W]
    for step in range(2):
        for i, (r, c) in enumerate(shapes):
            G = wl.gradient(31, i, step, r, c, bf16=False).astype(np.float64)
            W[i], M[i], _, _ = o.hyperball_step(W[i], G, M[i], eta=0.02, rho=rho[i])
    for i in range(len(shapes)):
        # every rank holds the owner's bits ...
        for r in range(1, world):
            assert torch.equal(got[0][i], got[r][i]), (i, r)
        # ... which equal the single-process result up to BLAS summation order across processes
        assert float((got[0][i] - torch.from_numpy(W[i])).abs().max()) <= 1e-13, i


def test_all_gather_rejects_mixed_dtypes():
    plan = sharding.ShardPlan([0, 1], 2, 0)
    with pytest.raises(ValueError):
        sharding.all_gather_weights([torch.zeros(2, 2), torch.zeros(2, 2, dtype=torch.bfloat16)], plan)


def _rs_worker(rank, world, port, shapes, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    from datetime import timedelta
    from oracle import nshb_oracle as o
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        plan = sharding.make_plan(shapes, world, rank)
        # this rank's own gradients of every matrix (its "batch"): seeded by rank
        grads = [torch.from_numpy(wl.gradient(40 + rank, i, 0, r, c, bf16=False).astype(np.float64))
                 for i, (r, c) in enumerate(shapes)]
        grads[1] = grads[1].t().contiguous().t()      # a strided gradient view
        out = [torch.empty(shapes[i], dtype=torch.float64) for i in plan.local]
        sharding.reduce_scatter_grads(grads, plan, out)
        torch.save({i: t for i, t in zip(plan.local, out)}, os.path.join(out_dir, f"g{rank}.pt"))
        # the whole data-parallel step: mean gradient on the owner, oracle step, all-gather
        W = [torch.from_numpy(wl.init_weight(41, i, r, c, bf16=False).astype(np.float64))
             for i, (r, c) in enumerate(shapes)]
        M = {i: np.zeros(shapes[i]) for i in plan.local}
        rho = [float(torch.linalg.norm(w)) for w in W]
        owned = dict(zip(plan.local, out))

        def step_fn(local):
            for i in local:
                Wn, M[i], _, _ = o.hyperball_step(W[i].numpy(), owned[i].numpy(), M[i], eta=0.02, rho=rho[i])
                W[i].copy_(torch.from_numpy(Wn))
        sharding.sharded_step(step_fn, W, plan)
        torch.save([w.clone() for w in W], os.path.join(out_dir, f"w{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_reduce_scatter_gives_each_owner_the_mean_gradient(tmp_path, world):
    """Every rank holds its own gradient of every matrix; after reduce_scatter_grads the
    owner of matrix i holds the mean over ranks, and the data-parallel step (mean gradient ->
    owner's step -> all-gather) equals the single-process step on the mean gradient."""
    from oracle import nshb_oracle as o
    shapes = [(24, 16), (16, 40), (32, 32), (8, 20), (48, 12)]
    mp.start_processes(_rs_worker, args=(world, _free_port(), shapes, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    mean = [sum(wl.gradient(40 + r, i, 0, a, b, bf16=False).astype(np.float64) for r in range(world)) / world
            for i, (a, b) in enumerate(shapes)]
    seen = set()
    for r in range(world):
        for i, g in torch.load(tmp_path / f"g{r}.pt").items():
            assert sharding.make_plan(shapes, world, r).owner[i] == r
            assert float((g - torch.from_numpy(mean[i])).abs().max()) <= 1e-15 * world, (r, i)
            seen.add(i)
    assert seen == set(range(len(shapes)))
    got = [torch.load(tmp_path / f"w{r}.pt") for r in range(world)]
    for i, (a, b) in enumerate(shapes):
        W0 = wl.init_weight(41, i, a, b, bf16=False).astype(np.float64)
        Wr, _, _, _ = o.hyperball_step(W0, mean[i], np.zeros_like(W0), eta=0.02, rho=o.fro(W0))
        for r in range(world):
            assert float((got[r][i] - torch.from_numpy(Wr)).abs().max()) <= 1e-12, (i, r)
