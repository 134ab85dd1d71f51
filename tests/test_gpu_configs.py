"""Full-size GPU runs of the benchmarked matrix sets, one step call per set (every matrix
of the set in the same launches, as bench.py runs it).

Matrices whose outputs are compared with the oracle are drawn from the seeded host
generators; the others are drawn on the device (seeded torch generator) and checked
through properties that hold at any size: the Hyperball radius, finiteness.
Tolerances as in test_gpu_parity.py: O within 2e-2 relative Frobenius error of the
oracle, momentum within 1e-6, radius within 1e-5 plus the bf16 storage term.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import newton_schulz_hyperball_b200 as nshb  # noqa: E402
from newton_schulz_hyperball_b200 import workloads as wl  # noqa: E402
from oracle import nshb_oracle as o  # noqa: E402
from gpu_harness import rel_fro, to_dev, to_host  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"


def radius_ok(w: torch.Tensor, rho: float) -> bool:
    x = w.float()
    n2 = float((x.double() ** 2).sum())
    tol = 1e-5 + 6 * (2.0 ** -9 / math.sqrt(3)) * math.sqrt(float((x.double() ** 4).sum())) / n2
    return abs(math.sqrt(n2) - rho) / rho <= tol


def device_inputs(shapes, sampled, cfg, step=0):
    """W (bf16), G (bf16) per matrix: host-seeded for the sampled indices, device-drawn
    otherwise (N(0, 0.02^2) weights, N(0, 1e-3^2) noise plus a rank-8 spike)."""
    g = torch.Generator(device=DEV)
    g.manual_seed(1000 * cfg + step)
    W, G = [], []
    for i, (r, c) in enumerate(shapes):
        if i in sampled:
            W.append(to_dev(wl.init_weight(cfg, i, r, c, bf16=True), True))
            G.append(to_dev(wl.gradient(cfg, i, step, r, c, bf16=True), True))
        else:
            W.append((0.02 * torch.randn(r, c, device=DEV, generator=g)).to(torch.bfloat16))
            a = torch.randn(r, 8, device=DEV, generator=g)
            b = torch.randn(c, 8, device=DEV, generator=g)
            G.append((1e-3 * (torch.randn(r, c, device=DEV, generator=g) + (10 / math.sqrt(8)) * (a @ b.T)))
                     .to(torch.bfloat16))
    return W, G


def run_set(shapes, sampled, cfg, kind, **kw):
    W, G = device_inputs(shapes, sampled, cfg)
    M = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W]
    O = [torch.empty_like(W[i]) if i in sampled else None for i in range(len(W))]
    rho = torch.stack([w.float().norm() for w in W])
    mats = nshb.matrices(W, G, M)
    for i in sampled:
        mats[i].O_out = O[i].data_ptr()
    op = {"hyperball": nshb.NSHB_OP_HYPERBALL, "brake": nshb.NSHB_OP_RADIAL_BRAKE,
          "himuon": nshb.NSHB_OP_HIMUON}[kind]
    p = nshb.params(rho=rho, **kw)
    ws = nshb.workspace(mats, p, op)
    host_w0 = {i: to_host(W[i]) for i in sampled}
    getattr(nshb, {"hyperball": "hyperball_step", "brake": "radial_brake_step", "himuon": "himuon_step"}[kind])(
        mats, p, ws)
    flags = nshb.device_status(ws)
    return W, M, O, rho, flags, host_w0


def check_sampled(shapes, sampled, cfg, kind, W, M, O, rho, host_w0, **kw):
    for i in sampled:
        r, c = shapes[i]
        G = wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64)
        W0 = host_w0[i]
        M0 = np.zeros_like(W0)
        if kind == "hyperball":
            _, Mr, Or, _ = o.hyperball_step(W0, G, M0, eta=kw["eta"], rho=float(rho[i]))
        elif kind == "brake":
            _, Mr, Or = o.radial_brake_step(W0, G, M0, lr=kw["lr"], outward=kw["brake_out"], inward=kw["brake_in"])
        else:
            _, Mr, Or, _ = o.himuon_step(W0, G, M0, tile=kw["tile"], eta=kw["eta"], rho=float(rho[i]))
        assert rel_fro(to_host(M[i]), Mr) <= 1e-6, i
        assert rel_fro(to_host(O[i]), Or) <= 2e-2, (i, rel_fro(to_host(O[i]), Or))


def test_gpt2_small_full_set_all_matrices():
    """72 GPT-2-small matrices in one hyperball_step; every matrix against the oracle."""
    cfg = wl.CFG_GPT2_SMALL
    shapes = [(r, c) for _, r, c in wl.gpt2_small_shapes(12)]
    sampled = set(range(len(shapes)))
    W, M, O, rho, flags, w0 = run_set(shapes, sampled, cfg, "hyperball", eta=0.02)
    assert flags == 0
    check_sampled(shapes, sampled, cfg, "hyperball", W, M, O, rho, w0, eta=0.02)
    for i in range(len(shapes)):
        assert radius_ok(W[i], float(rho[i])), i


@pytest.mark.parametrize("kind", ["hyperball", "brake"])
def test_qwen3_1b_full_set(kind):
    """196 Qwen3-style matrices (1.41B parameters) in one call; layer 0 (all seven shapes)
    against the oracle, every matrix through the radius (Hyperball) or finiteness check."""
    cfg = wl.CFG_QWEN3_1B
    shapes = [(r, c) for _, r, c in wl.qwen3_1b_shapes(28)]
    sampled = set(range(7)) if kind == "hyperball" else {1, 6}
    kw = dict(eta=0.02) if kind == "hyperball" else dict(lr=0.02, brake_out=0.5, brake_in=1.0)
    W, M, O, rho, flags, w0 = run_set(shapes, sampled, cfg, kind, **kw)
    assert flags == 0
    check_sampled(shapes, sampled, cfg, kind, W, M, O, rho, w0, **kw)
    for i in range(len(shapes)):
        assert torch.isfinite(W[i].float()).all(), i
        if kind == "hyperball":
            assert radius_ok(W[i], float(rho[i])), i
    del W, M, O
    torch.cuda.empty_cache()


@pytest.mark.parametrize("tile,layers", [(256, 32), (512, 32), (128, 4)])
def test_8b_width_himuon(tile, layers):
    """8B-width matrices (32 layers: 224 matrices, 6.98B parameters) with every T x T tile
    batched in one himuon_step.  Checked tile by tile against the oracle: one matrix of every
    shape of layer 0 (4096^2, 1024x4096, 14336x4096, 4096x14336) and two of the last layer
    (its 1024x4096 and 4096x14336); the radius of every matrix checked."""
    cfg = wl.CFG_8B_WIDTH
    shapes = [(r, c) for _, r, c in wl.width_8b_shapes(layers)]
    last = 7 * (layers - 1)
    sampled = {0, 2, 4, 6, last + 3, last + 6}
    W, M, O, rho, flags, w0 = run_set(shapes, sampled, cfg, "himuon", tile=tile, eta=0.02)
    assert flags == 0
    check_sampled(shapes, sampled, cfg, "himuon", W, M, O, rho, w0, tile=tile, eta=0.02)
    for i in range(len(shapes)):
        assert radius_ok(W[i], float(rho[i])), i
    del W, M, O
    torch.cuda.empty_cache()


def test_8b_width_himuon_large_tile_equals_full_muon():
    """T >= both dims makes the tiled map the full-matrix map: blocks cut from 8B-width
    matrices (512 x 512, 128 x 512, 512 x 448) with T = 512 against hyperball_step."""
    cfg = wl.CFG_8B_WIDTH
    shapes = [(512, 512), (128, 512), (512, 448)]
    W = [to_dev(wl.init_weight(cfg, 500 + i, r, c, bf16=True), True) for i, (r, c) in enumerate(shapes)]
    G = [to_dev(wl.gradient(cfg, 500 + i, 0, r, c, bf16=True), True) for i, (r, c) in enumerate(shapes)]
    outs = {}
    for kind in ("himuon", "hyperball"):
        Wk = [w.clone() for w in W]
        M = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W]
        O = [torch.empty_like(w) for w in W]
        mats = nshb.matrices(Wk, G, M, O)
        p = nshb.params(tile=512, eta=0.02)
        op = nshb.NSHB_OP_HIMUON if kind == "himuon" else nshb.NSHB_OP_HYPERBALL
        ws = nshb.workspace(mats, p, op)
        getattr(nshb, kind + "_step")(mats, p, ws)
        assert nshb.device_status(ws) == 0
        outs[kind] = [to_host(x) for x in O]
    for i in range(len(shapes)):
        assert rel_fro(outs["himuon"][i], outs["hyperball"][i]) <= 2e-2


def test_newton_muon_gpt2_full():
    """Newton-Muon on all 72 GPT-2 matrices: 48 layer inputs Z (d_in x 8192 tokens,
    per-feature scales log-uniform in [0.1, 10]), ridge 1e-3 tr(ZZ^T)/d_in; every matrix
    against the oracle's plain linear solve + NS + Hyperball."""
    from gpu_harness import GpuSet, newton_step
    cfg = wl.CFG_NEWTON_GPT2
    named = wl.gpt2_small_shapes(12)
    shapes = [(r, c) for _, r, c in named]
    zi, zrows = wl.newton_gpt2_z_index(named)
    n_tok = 8192
    Zs = [wl.layer_input(cfg, j, d, n_tok) for j, d in enumerate(zrows)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    for k in range(len(shapes)):
        gs.mats[k].z_index = zi[k]
    gs.set_grads(Gs)
    rho_dev = torch.tensor(rhos, dtype=torch.float32, device=DEV)
    p = nshb.params(eta=0.02, rho=rho_dev, ridge_rel=1e-3)
    assert newton_step(gs, Zs, n_tok, p) == 0
    Wg, Mg, Og = gs.host()
    for i in range(len(shapes)):
        _, Mr, Or, _ = o.newton_muon_step(Ws[i], Gs[i], np.zeros_like(Ws[i]), Zs[zi[i]].astype(np.float64),
                                          ridge_rel=1e-3, eta=0.02, rho=rhos[i])
        assert rel_fro(Mg[i], Mr) <= 1e-6, i
        assert rel_fro(Og[i], Or) <= 2e-2, (i, rel_fro(Og[i], Or))
        assert radius_ok(gs.W[i], rhos[i]), i
