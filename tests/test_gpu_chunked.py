"""Memory-bounded steps and tile-size schedules on the GPU: a step run in workspace-sized
chunks equals the unchunked step bit for bit (every matrix's arithmetic is independent of
the others and fixed in order), and Hierarchical Muon follows the oracle when T changes
from step to step."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import newton_schulz_hyperball_b200 as nshb  # noqa: E402
from newton_schulz_hyperball_b200 import workloads as wl  # noqa: E402
from oracle import nshb_oracle as o  # noqa: E402
from gpu_harness import GpuSet, rel_fro  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"


def device_set(shapes, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    W = [(0.02 * torch.randn(r, c, device=DEV, generator=g)).to(torch.bfloat16) for r, c in shapes]
    G = []
    for r, c in shapes:
        a = torch.randn(r, 8, device=DEV, generator=g)
        b = torch.randn(c, 8, device=DEV, generator=g)
        G.append((1e-3 * (torch.randn(r, c, device=DEV, generator=g) + (10 / 8 ** 0.5) * (a @ b.T))).to(torch.bfloat16))
    return W, G


def run(op, shapes, seed, p_kw, chunk_frac=None):
    W, G = device_set(shapes, seed)
    M = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W]
    O = [torch.empty_like(w) for w in W]
    rho = torch.stack([w.float().norm() for w in W])
    mats = nshb.matrices(W, G, M, O)
    p = nshb.params(rho=rho, **p_kw)
    full = nshb.workspace_size(mats, p, op)
    if chunk_frac is None:
        ws = torch.empty(full, dtype=torch.uint8, device=DEV)
        n = nshb.step_chunked(op, mats, p, ws)
        assert n == 1
    else:
        least = nshb.workspace_size_min(mats, p, op)
        size = max(least, int(full * chunk_frac) // 256 * 256)
        ws = torch.empty(size, dtype=torch.uint8, device=DEV)
        n = nshb.step_chunked(op, mats, p, ws)
        assert n > 1
    assert nshb.device_status(ws) == 0
    torch.cuda.synchronize()
    return [w.clone() for w in W], [m.clone() for m in M], [x.clone() for x in O], n


def test_chunked_hyperball_equals_unchunked_bitwise():
    shapes = [(r, c) for _, r, c in wl.gpt2_small_shapes(3)]
    a = run(nshb.NSHB_OP_HYPERBALL, shapes, 61, dict(eta=0.02))
    b = run(nshb.NSHB_OP_HYPERBALL, shapes, 61, dict(eta=0.02), chunk_frac=0.3)
    for x, y in zip(a[:3], b[:3]):
        for u, v in zip(x, y):
            assert torch.equal(u, v)


def test_chunked_himuon_8b_width_layer_equals_unchunked_bitwise():
    shapes = [(r, c) for _, r, c in wl.width_8b_shapes(1)]
    a = run(nshb.NSHB_OP_HIMUON, shapes, 62, dict(eta=0.02, tile=256))
    b = run(nshb.NSHB_OP_HIMUON, shapes, 62, dict(eta=0.02, tile=256), chunk_frac=0.35)
    assert b[3] >= 3
    for x, y in zip(a[:3], b[:3]):
        for u, v in zip(x, y):
            assert torch.equal(u, v)
    del a, b
    torch.cuda.empty_cache()


def test_himuon_tile_schedule_follows_oracle():
    """T = 512, 256, 128 on three consecutive steps (state carried by both sides)."""
    cfg = 63
    shapes = [(512, 512), (256, 1024), (1024, 512)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    Wr = [w.copy() for w in Ws]
    Mr = [np.zeros_like(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    rho = torch.tensor(rhos, dtype=torch.float32, device=DEV)
    for step, T in enumerate((512, 256, 128)):
        Gs = [wl.gradient(cfg, i, step, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
        gs.set_grads(Gs)
        assert gs.step("himuon", nshb.params(eta=0.02, rho=rho, tile=T)) == 0
        Wg, Mg, Og = gs.host()
        for i in range(len(shapes)):
            Wr[i], Mr[i], Or, _ = o.himuon_step(Wr[i], Gs[i], Mr[i], tile=T, eta=0.02, rho=rhos[i])
            assert rel_fro(Mg[i], Mr[i]) <= 1e-6 * (step + 1), (step, i)
            assert rel_fro(Og[i], Or) <= 2e-2, (step, i, rel_fro(Og[i], Or))


def test_chunked_step_keeps_a_flag_raised_in_the_first_chunk():
    """A NaN gradient in the first chunk's matrix sets NSHB_DEV_NONFINITE; the later chunks
    add their flags to the same status word without clearing it, so the flag is still there
    when the call returns.  The matrix with the NaN keeps its weights, the others step."""
    shapes = [(r, c) for _, r, c in wl.gpt2_small_shapes(3)]
    W, G = device_set(shapes, 64)
    G[0][3, 5] = float("nan")
    W0 = [w.clone() for w in W]
    M = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W]
    rho = torch.stack([w.float().norm() for w in W])
    mats = nshb.matrices(W, G, M)
    p = nshb.params(rho=rho, eta=0.02)
    op = nshb.NSHB_OP_HYPERBALL
    full = nshb.workspace_size(mats, p, op)
    size = max(nshb.workspace_size_min(mats, p, op), int(full * 0.3) // 256 * 256)
    ws = torch.empty(size, dtype=torch.uint8, device=DEV)
    n = nshb.step_chunked(op, mats, p, ws)
    assert n >= 3
    flags = nshb.device_status(ws)
    assert flags & nshb.NSHB_DEV_NONFINITE
    assert torch.equal(W[0], W0[0])
    assert not torch.equal(W[-1], W0[-1])
    for w in W[1:]:
        assert torch.isfinite(w.float()).all()
