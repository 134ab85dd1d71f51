"""The data-parallel sharded step on the library (one GPU).

Two ranks are emulated in one process: each rank's ShardedOptimizer runs the library's
step on the matrices it owns (LPT by NS work), and the all-gather is replaced by copying
each owner's matrices into the result.  Every matrix's arithmetic is independent of the
other matrices of a call, so the sharded result equals the unsharded step bit for bit.  A
world-1 ShardedOptimizer (no process group needed) goes through the whole step() path.
The collectives themselves are covered by the gloo tests on CPU."""
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import newton_schulz_hyperball_b200 as nshb  # noqa: E402
from newton_schulz_hyperball_b200 import sharding  # noqa: E402
from newton_schulz_hyperball_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"


def device_set(shapes, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    W = [(0.02 * torch.randn(r, c, device=DEV, generator=g)).to(torch.bfloat16) for r, c in shapes]
    G = [(1e-3 * torch.randn(r, c, device=DEV, generator=g)).to(torch.bfloat16) for r, c in shapes]
    return W, G


@pytest.mark.parametrize("kind,kw", [("hyperball", dict(eta=0.02)), ("himuon", dict(eta=0.02, tile=256))])
def test_sharded_step_equals_unsharded_bitwise(kind, kw):
    shapes = [(r, c) for _, r, c in wl.gpt2_small_shapes(2)] + [(1024, 4096), (300, 700)]
    W, G = device_set(shapes, 71)
    rho = torch.stack([w.float().norm() for w in W])
    # unsharded reference: one call on every matrix
    Wa = [w.clone() for w in W]
    Ma = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W]
    mats = nshb.matrices(Wa, G, Ma)
    op = nshb.NSHB_OP_HYPERBALL if kind == "hyperball" else nshb.NSHB_OP_HIMUON
    p = nshb.params(rho=rho, **kw)
    ws = nshb.workspace(mats, p, op)
    getattr(nshb, kind + "_step")(mats, p, ws)
    assert nshb.device_status(ws) == 0
    # two emulated ranks, each stepping the matrices it owns
    world = 2
    out = [w.clone() for w in W]
    copies = [[w.clone() for w in W] for _ in range(world)]
    opts = [sharding.ShardedOptimizer(copies[k], rho, sharding.make_plan(shapes, world, k), kind, **kw)
            for k in range(world)]
    assert sorted(sum((o.local for o in opts), [])) == list(range(len(shapes)))
    for o in opts:
        for j, i in enumerate(o.local):
            o.G[j].copy_(G[i])
        o.local_step()
        assert o.device_status() == 0
        for i in o.local:
            out[i].copy_(o.W[i])
    for i in range(len(shapes)):
        assert torch.equal(out[i], Wa[i]), i
    # world 1: the full step() path (copy-through reduce-scatter, step, no gather)
    Wb = [w.clone() for w in W]
    one = sharding.ShardedOptimizer(Wb, rho, sharding.make_plan(shapes, 1, 0), kind, **kw)
    one.step(G)
    assert one.device_status() == 0
    for i in range(len(shapes)):
        assert torch.equal(Wb[i], Wa[i]), i


@pytest.mark.parametrize("kind,kw", [("hyperball", {}), ("himuon", {"tile": 256})])
def test_a_ragged_neighbour_does_not_change_a_matrix_bitwise(kind, kw):
    """A matrix's step does not depend on the other matrices of its call: adding a ragged
    matrix (element-wise loads and masked blocks in the same launches) leaves the results of
    the aligned ones bit for bit unchanged, momentum buffers included."""
    aligned = [(768, 768), (3072, 768), (768, 3072), (1024, 4096)]
    W, G = device_set(aligned + [(300, 700)], 73)
    rho = torch.stack([w.float().norm() for w in W])
    op = nshb.NSHB_OP_HYPERBALL if kind == "hyperball" else nshb.NSHB_OP_HIMUON
    outs = []
    for n in (len(aligned), len(aligned) + 1):
        Wc = [w.clone() for w in W[:n]]
        Mc = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W[:n]]
        mats = nshb.matrices(Wc, G[:n], Mc)
        p = nshb.params(rho=rho[:n].contiguous(), **kw)
        ws = nshb.workspace(mats, p, op)
        for _ in range(2):
            getattr(nshb, kind + "_step")(mats, p, ws)
        assert nshb.device_status(ws) == 0
        outs.append((Wc, Mc))
    for i in range(len(aligned)):
        assert torch.equal(outs[0][1][i], outs[1][1][i]), i
        assert torch.equal(outs[0][0][i], outs[1][0][i]), i
