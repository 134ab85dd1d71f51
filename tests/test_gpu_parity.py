"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle on the same
seeded inputs.

Tolerances (written per test):
  * fp32 NS path: relative Frobenius error of O and of the weight change <= 1e-4;
  * bf16 tensor-core NS path: relative Frobenius error of O <= 2e-2;
  * momentum buffer (fp32): relative error <= 1e-6;
  * radius: | ||W|| - rho | / rho <= 1e-5 for fp32 weights; for bf16 weights the stored
    value carries the bf16 rounding of every element, so the bound is 1e-5 plus six
    standard deviations of that rounding's effect on the norm (2^-9/sqrt(3) per element,
    relative), computed from the weights themselves.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

from newton_schulz_hyperball_b200 import workloads as wl  # noqa: E402
from oracle import nshb_oracle as o  # noqa: E402
import newton_schulz_hyperball_b200 as nshb  # noqa: E402
from gpu_harness import GpuSet, rel_fro  # noqa: E402

pytestmark = pytest.mark.gpu


def radius_tol(W, bf16):
    if not bf16:
        return 1e-5
    w2 = np.sum(W * W)
    return 1e-5 + 6 * (2.0 ** -9 / math.sqrt(3)) * math.sqrt(np.sum(W ** 4)) / w2


def bf16_w_tol(W_ref, eta):
    """Frobenius bound on W_gpu - W_ref for bf16 weights: half an ulp per element of
    storage rounding plus the 2e-2 relative error of the unit update direction."""
    a = np.abs(W_ref)
    e = np.floor(np.log2(np.maximum(a, 1e-38)))
    half_ulp = np.where(a > 0, 2.0 ** (e - 8), 0.0)
    return float(np.linalg.norm(half_ulp)) + 2 * 2e-2 * eta + 1e-6 * float(np.linalg.norm(W_ref))


# ------------------------------------------------------------------ fp32 path
def test_fp32_single_matrix_hyperball_10_steps():
    """256x256 fp32, W0 ~ N(0, 0.02^2), G ~ N(0, 1e-2^2) fresh each step, beta 0.95 Nesterov,
    K = 5, Hyperball rho = ||W0||, eta = 0.02, 10 steps."""
    cfg = wl.CFG_SINGLE_F32
    W = wl.init_weight(cfg, 0, 256, 256, bf16=False).astype(np.float64)
    rho = o.fro(W)
    gs = GpuSet([W], bf16=False)
    rho_dev = torch.tensor([rho], dtype=torch.float32, device="cuda")
    p = nshb.params(ns_precision=nshb.NSHB_F32, eta=0.02, rho=rho_dev)
    Wr, Mr = W.copy(), np.zeros_like(W)
    for step in range(10):
        G = wl.plain_gradient(cfg, 0, step, 256, 256, 1e-2, bf16=False)
        gs.set_grads([G])
        W_prev = Wr.copy()
        flags = gs.step("hyperball", p)
        assert flags == 0
        Wr, Mr, Or, _ = o.hyperball_step(Wr, G, Mr, eta=0.02, rho=rho)
        Wg, Mg, Og = gs.host()
        assert rel_fro(Mg[0], Mr) <= 1e-6
        assert rel_fro(Og[0], Or) <= 1e-4
        assert rel_fro(Wg[0] - W_prev, Wr - W_prev) <= 1e-4
        assert abs(o.fro(Wg[0]) - rho) / rho <= 1e-5


@pytest.mark.parametrize("shape", [(96, 200), (200, 96), (5, 7), (7, 5), (1, 9), (9, 1), (130, 130)])
def test_fp32_shapes_muon_and_hyperball(shape):
    cfg = 11
    m, n = shape
    W = wl.init_weight(cfg, 1, m, n, bf16=False).astype(np.float64)
    G = wl.gradient(cfg, 1, 0, m, n, bf16=False)
    for kind in ("muon", "hyperball"):
        gs = GpuSet([W], bf16=False)
        gs.set_grads([G])
        p = nshb.params(ns_precision=nshb.NSHB_F32, eta=0.01, lr=0.05, weight_decay=0.1)
        flags = gs.step(kind, p)
        assert flags == 0
        Wg, Mg, Og = gs.host()
        if kind == "muon":
            Wr, Mr, Or = o.muon_step(W, G, np.zeros_like(W), lr=0.05, weight_decay=0.1)
        else:
            Wr, Mr, Or, _ = o.hyperball_step(W, G, np.zeros_like(W), eta=0.01, rho=None)
            assert abs(o.fro(Wg[0]) - o.fro(W)) / o.fro(W) <= 1e-5
        assert rel_fro(Mg[0], Mr) <= 1e-6
        assert rel_fro(Og[0], Or) <= 1e-4
        assert rel_fro(Wg[0] - W, Wr - W) <= 1e-4


# ------------------------------------------------------------------ bf16 path
PHASE_SHAPES = [(256, 256), (256, 512), (512, 256), (300, 700), (700, 300), (5, 7), (128, 1000)]


@pytest.mark.parametrize("coeffs", [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (0.5, -0.25, 0.125)])
@pytest.mark.parametrize("shape", PHASE_SHAPES)
def test_bf16_single_iteration_phases(shape, coeffs):
    """One NS iteration with chosen (a, b, c) isolates the Gram (b), polynomial (c) and
    update (a) phases of the tensor-core chain."""
    cfg = 12
    m, n = shape
    W = wl.init_weight(cfg, 2, m, n, bf16=True).astype(np.float64)
    G = wl.gradient(cfg, 2, 0, m, n, bf16=True).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    p = nshb.params(ns_steps=1, coeffs=[coeffs], lr=0.0)
    assert gs.step("muon", p) == 0
    _, Mg, Og = gs.host()
    _, U = o.momentum(np.zeros_like(G), G, 0.95, True)
    Or = o.newton_schulz(U, 1, coeffs=[coeffs])
    assert rel_fro(Mg[0], (1 - 0.95) * G) <= 1e-6
    assert rel_fro(Og[0], Or) <= 1e-2


@pytest.mark.parametrize("shape", PHASE_SHAPES + [(768, 768), (3072, 768), (768, 3072)])
def test_bf16_ns_five_steps(shape):
    cfg = 13
    m, n = shape
    W = wl.init_weight(cfg, 3, m, n, bf16=True).astype(np.float64)
    G = wl.gradient(cfg, 3, 0, m, n, bf16=True).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    p = nshb.params(lr=0.0)
    assert gs.step("muon", p) == 0
    Wg, _, Og = gs.host()
    _, U = o.momentum(np.zeros_like(G), G, 0.95, True)
    assert rel_fro(Og[0], o.newton_schulz(U)) <= 2e-2
    assert np.array_equal(Wg[0], W)     # lr = 0 leaves W bit-exact


def test_bf16_compensated_iterations_beat_plain_chain():
    """The plain bf16 chain (every X rounded to bf16, as newton_schulz5 does) loses the
    small singular directions of a spiked gradient to the rounding of U; carrying X as a
    hi/lo pair through the first two a*X terms recovers them."""
    cfg = 13
    W = wl.init_weight(cfg, 3, 256, 256, bf16=True).astype(np.float64)
    G = wl.gradient(cfg, 3, 0, 256, 256, bf16=True).astype(np.float64)
    _, U = o.momentum(np.zeros_like(G), G, 0.95, True)
    ref = o.newton_schulz(U)
    errs = {}
    for comp in (0, 1, 2, 5):
        gs = GpuSet([W], bf16=True)
        gs.set_grads([G])
        assert gs.step("muon", nshb.params(lr=0.0, ns_compensated=comp)) == 0
        errs[comp] = rel_fro(gs.host()[2][0], ref)
    assert errs[2] <= 1e-2 and errs[5] <= 1e-2
    assert errs[2] < errs[1] < errs[0]


def gpt2_layer(cfg, layer, step):
    shapes = wl.gpt2_small_shapes(1)
    Ws, Gs = [], []
    for k, (_, r, c) in enumerate(shapes):
        idx = layer * 6 + k
        Ws.append(wl.init_weight(cfg, idx, r, c, bf16=True).astype(np.float64))
        Gs.append(wl.gradient(cfg, idx, step, r, c, bf16=True).astype(np.float64))
    return Ws, Gs


def test_bf16_hyperball_gpt2_layer_two_steps():
    cfg = wl.CFG_GPT2_SMALL
    Ws, _ = gpt2_layer(cfg, 0, 0)
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    rho_dev = torch.tensor(rhos, dtype=torch.float32, device="cuda")
    p = nshb.params(eta=0.02, rho=rho_dev)
    Wr = [w.copy() for w in Ws]
    Mr = [np.zeros_like(w) for w in Ws]
    for step in range(2):
        _, Gs = gpt2_layer(cfg, 0, step)
        gs.set_grads(Gs)
        assert gs.step("hyperball", p) == 0
        Wg, Mg, Og = gs.host()
        for i in range(len(Ws)):
            # Each side keeps its own state: the oracle in fp64, the GPU in bf16 / fp32.
            Wr[i], Mr[i], On, _ = o.hyperball_step(Wr[i], Gs[i], Mr[i], eta=0.02, rho=rhos[i])
            assert rel_fro(Mg[i], Mr[i]) <= 1e-6
            assert rel_fro(Og[i], On) <= 2e-2, i
            # bf16 storage rounding accumulates once per step.
            assert np.linalg.norm(Wg[i] - Wr[i]) <= (step + 1) * bf16_w_tol(Wr[i], 0.02), i
            assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True), i


def test_bf16_hyperball_gpt2_two_layers_six_steps():
    """Six MuonH steps on two GPT-2 layers (12 matrices), each side keeping its own state:
    the deviation of W may grow by one step's bound per step, the momentum stays at fp32
    accuracy, every step's O within the NS tolerance, and the radius after every step."""
    cfg = wl.CFG_GPT2_SMALL
    Ws = gpt2_layer(cfg, 0, 0)[0] + gpt2_layer(cfg, 1, 0)[0]
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    p = nshb.params(eta=0.02, rho=torch.tensor(rhos, dtype=torch.float32, device="cuda"))
    Wr = [w.copy() for w in Ws]
    Mr = [np.zeros_like(w) for w in Ws]
    for step in range(6):
        Gs = gpt2_layer(cfg, 0, step)[1] + gpt2_layer(cfg, 1, step)[1]
        gs.set_grads(Gs)
        assert gs.step("hyperball", p) == 0
        Wg, Mg, Og = gs.host()
        for i in range(len(Ws)):
            Wr[i], Mr[i], On, _ = o.hyperball_step(Wr[i], Gs[i], Mr[i], eta=0.02, rho=rhos[i])
            assert rel_fro(Mg[i], Mr[i]) <= 1e-6, (step, i)
            assert rel_fro(Og[i], On) <= 2e-2, (step, i)
            assert np.linalg.norm(Wg[i] - Wr[i]) <= (step + 1) * bf16_w_tol(Wr[i], 0.02), (step, i)
            assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True), (step, i)


def test_bf16_hyperball_gpt2_full_set_three_steps():
    """All 72 GPT-2-small matrices in one call per step, three MuonH steps, each side keeping
    its own state: every matrix's O, M, W and radius after every step."""
    cfg = wl.CFG_GPT2_SMALL
    Ws = [w for layer in range(12) for w in gpt2_layer(cfg, layer, 0)[0]]
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    p = nshb.params(eta=0.02, rho=torch.tensor(rhos, dtype=torch.float32, device="cuda"))
    Wr = [w.copy() for w in Ws]
    Mr = [np.zeros_like(w) for w in Ws]
    for step in range(3):
        Gs = [wl.gradient(cfg, i, step, *w.shape, bf16=True).astype(np.float64) for i, w in enumerate(Ws)]
        gs.set_grads(Gs)
        assert gs.step("hyperball", p) == 0
        Wg, Mg, Og = gs.host()
        for i in range(len(Ws)):
            Wr[i], Mr[i], On, _ = o.hyperball_step(Wr[i], Gs[i], Mr[i], eta=0.02, rho=rhos[i])
            assert rel_fro(Mg[i], Mr[i]) <= 1e-6, (step, i)
            assert rel_fro(Og[i], On) <= 2e-2, (step, i, rel_fro(Og[i], On))
            assert np.linalg.norm(Wg[i] - Wr[i]) <= (step + 1) * bf16_w_tol(Wr[i], 0.02), (step, i)
            assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True), (step, i)


def test_bf16_muon_and_brake_steps():
    cfg = 14
    shapes = [(256, 512), (512, 256), (300, 300)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    for kind in ("muon", "brake"):
        gs = GpuSet(Ws, bf16=True)
        gs.set_grads(Gs)
        p = nshb.params(lr=0.02, weight_decay=0.0, brake_out=0.5, brake_in=1.0)
        assert gs.step(kind, p) == 0
        Wg, _, Og = gs.host()
        for i, W in enumerate(Ws):
            if kind == "muon":
                Wr, _, Or = o.muon_step(W, Gs[i], np.zeros_like(W), lr=0.02)
            else:
                Wr, _, Or = o.radial_brake_step(W, Gs[i], np.zeros_like(W), lr=0.02, outward=0.5, inward=1.0)
            assert rel_fro(Og[i], Or) <= 2e-2
            step_len = 0.02 * o.shape_scale(*W.shape) * o.fro(Or)
            assert np.linalg.norm(Wg[i] - Wr) <= bf16_w_tol(Wr, step_len)


# ---------------------------------------------------- page pins on the GPU
def test_bf16_768_five_directions_page_pin():
    """Muon explainer, code section: bf16 NS of a 768x768 matrix with singular values
    0.9, 0.3, 0.1, 0.01, 0.001 (the other 763 about 0.011) lands within 0.005 of the scalar
    polynomial.  Read as: the stretch along each of the five named singular directions,
    u_k^T O v_k, is within 0.005 of phi^5 applied to that direction's normalised input
    stretch; the full sorted spectrum is checked as well, with its own bound."""
    import json, pathlib
    g = json.loads((pathlib.Path(__file__).parent / "golden" / "page_values.json").read_text())["bf16_768_example"]
    n = g["n"]
    sig = np.array(g["sigma_top"] + [g["bulk_sigma"]] * (n - 5))
    U32, q1, q2 = wl.spectrum_matrix(5, n, n, sig, factors=True)
    U = wl.round_to_bf16(U32).astype(np.float64)
    # With M = 0 and beta = 0 the Nesterov update is U = G.
    gs = GpuSet([np.zeros((n, n))], bf16=True)
    gs.set_grads([U])
    assert gs.step("muon", nshb.params(beta=0.0, lr=0.0)) == 0
    O = gs.host()[2][0]
    nrm = np.sqrt(np.sum(U * U)) + o.NS_EPS
    for k in range(5):
        d_in = q1[:, k] @ U @ q2[:, k]
        d_out = q1[:, k] @ O @ q2[:, k]
        assert abs(d_out - o.scalar_ns(d_in / nrm, 5)) <= g["abs_tol"], k
    # The whole spectrum, sorted, against the oracle's map of the same bf16 input (whose
    # singular values are the scalar polynomial of the input's, to rounding).  The 763
    # filler values sit where the five-step map is steep (slope about 80 at 0.011), so the
    # chain's bf16 rounding moves them more than the five named directions: measured 0.0070
    # on B200, bounded here by 0.01.
    s_gpu = np.sort(np.linalg.svd(O, compute_uv=False))
    s_ref = np.sort(np.linalg.svd(o.newton_schulz(U), compute_uv=False))
    assert np.max(np.abs(s_gpu - s_ref)) <= 0.01


def test_bf16_random_3072x768_band_page_pin():
    import json, pathlib
    g = json.loads((pathlib.Path(__file__).parent / "golden" / "page_values.json").read_text())["random_3072x768_band"]
    rng = np.random.default_rng(7)
    U = wl.round_to_bf16(rng.standard_normal((g["rows"], g["cols"])).astype(np.float32)).astype(np.float64)
    gs = GpuSet([np.zeros_like(U)], bf16=True)
    gs.set_grads([U])
    assert gs.step("muon", nshb.params(beta=0.0, lr=0.0)) == 0
    _, _, Og = gs.host()
    s = np.linalg.svd(Og[0], compute_uv=False)
    assert s.min() >= g["lo"] - 0.01 and s.max() <= g["hi"] + 0.01


# ------------------------------------------------------------ Hierarchical Muon
@pytest.mark.parametrize("T", [128, 256, 512])
def test_bf16_himuon_tiles(T):
    """Each T x T tile (edge tiles the remainder, grid anchored at (0, 0)) gets its own
    normalisation and NS map; Hyperball then acts on the whole matrix."""
    cfg = 15
    shapes = [(512, 768), (768, 512), (300, 700)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    gs.set_grads(Gs)
    rho_dev = torch.tensor(rhos, dtype=torch.float32, device="cuda")
    assert gs.step("himuon", nshb.params(tile=T, eta=0.02, rho=rho_dev)) == 0
    Wg, Mg, Og = gs.host()
    for i, W in enumerate(Ws):
        Wr, Mr, Or, _ = o.himuon_step(W, Gs[i], np.zeros_like(W), tile=T, eta=0.02, rho=rhos[i])
        assert rel_fro(Mg[i], Mr) <= 1e-6
        assert rel_fro(Og[i], Or) <= 2e-2, (i, rel_fro(Og[i], Or))
        assert np.linalg.norm(Wg[i] - Wr) <= bf16_w_tol(Wr, 0.02)
        assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True)


def test_bf16_himuon_large_tile_equals_full_muon():
    """T >= both dims: the tiled map is the full-matrix map (same O up to bf16 noise)."""
    cfg = 16
    shapes = [(256, 384), (384, 256), (200, 500)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    a = GpuSet(Ws, bf16=True)
    a.set_grads(Gs)
    assert a.step("himuon", nshb.params(tile=512, eta=0.02)) == 0
    b = GpuSet(Ws, bf16=True)
    b.set_grads(Gs)
    assert b.step("hyperball", nshb.params(eta=0.02)) == 0
    for i in range(len(Ws)):
        assert rel_fro(a.host()[2][i], b.host()[2][i]) <= 2e-2
        _, U = o.momentum(np.zeros_like(Gs[i]), Gs[i], 0.95, True)
        assert rel_fro(a.host()[2][i], o.newton_schulz(U)) <= 2e-2


def test_fro_norms_match_numpy():
    cfg = 17
    shapes = [(768, 768), (3072, 768), (5, 7), (300, 700)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    gs = GpuSet(Ws, bf16=True, want_o=False)
    out = torch.zeros(len(Ws), dtype=torch.float32, device="cuda")
    ws = nshb.workspace(gs.mats, nshb.params(), nshb.NSHB_OP_MUON)
    nshb.fro_norms(gs.mats, out, ws)
    got = out.cpu().numpy().astype(np.float64)
    for i, W in enumerate(Ws):
        assert abs(got[i] - o.fro(W)) <= 1e-6 * o.fro(W)


def test_zero_norm_fallback_keeps_radius():
    """rho = eta and an update that exactly cancels W: the step is skipped and W stays on
    its sphere (status bit NSHB_DEV_ZERO_NORM_FALLBACK).  The GPU's own U_hat differs from
    W by bf16 rounding, so 'numerical zero' is set by hb_eps above that residual."""
    cfg = 18
    m, n = 256, 256
    G = wl.gradient(cfg, 0, 0, m, n, bf16=True).astype(np.float64)
    _, U = o.momentum(np.zeros_like(G), G, 0.95, True)
    O = o.newton_schulz(U)
    eta = 0.02
    W = wl.round_to_bf16((eta * O / o.fro(O)).astype(np.float32)).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    rho_dev = torch.tensor([eta], dtype=torch.float32, device="cuda")
    flags = gs.step("hyperball", nshb.params(eta=eta, rho=rho_dev, hb_eps=0.05 * eta))
    assert flags & nshb.NSHB_DEV_ZERO_NORM_FALLBACK
    Wg = gs.host()[0][0]
    assert abs(o.fro(Wg) - eta) / eta <= radius_tol(Wg, True)
    assert rel_fro(Wg / o.fro(Wg), W / o.fro(W)) <= 1e-2
    # the oracle on the same inputs takes the same branch when its own residual is below hb_eps
    Wr, fb = o.hyperball_apply(W, O, eta, eta, eps=0.05 * eta)
    assert fb and abs(o.fro(Wr) - eta) < 1e-12


def test_nonfinite_gradient_sets_status_and_keeps_weights():
    W = wl.init_weight(19, 0, 128, 256, bf16=True).astype(np.float64)
    G = np.full(W.shape, np.nan)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    flags = gs.step("hyperball", nshb.params(eta=0.02))
    assert flags & nshb.NSHB_DEV_NONFINITE
    assert np.array_equal(gs.host()[0][0], W)


def test_device_wait_limit_reports_timeout_without_faulting():
    """A bounded wait that runs out: with debug_flags bits 0|1 the MMA warp withholds its
    first accumulator hand-off, the epilogue's wait (limit ~1 ms) gives up, the kernel sets
    NSHB_DEV_TIMEOUT, frees its tensor memory and returns.  The context stays usable: the
    next normal step on the same buffers succeeds and matches the oracle."""
    W = wl.init_weight(20, 0, 256, 256, bf16=True).astype(np.float64)
    G = wl.gradient(20, 0, 0, 256, 256, bf16=True).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    flags = gs.step("hyperball", nshb.params(eta=0.02, debug_flags=3))
    assert flags & nshb.NSHB_DEV_TIMEOUT
    # short limit alone: nothing runs out
    gs2 = GpuSet([W], bf16=True)
    gs2.set_grads([G])
    assert gs2.step("hyperball", nshb.params(eta=0.02, debug_flags=1)) == 0
    _, _, Og = gs2.host()
    _, U = o.momentum(np.zeros_like(G), G, 0.95, True)
    assert rel_fro(Og[0], o.newton_schulz(U)) <= 2e-2


@pytest.mark.parametrize("T", [128, 256])
def test_tile_resident_himuon_wait_limit_reports_timeout(T):
    """The tile-resident HiMuon kernels' bounded waits: with debug_flags bits 0|1 the MMA
    thread withholds the first Gram hand-off of its first tile (the MMAs still complete on a
    spare barrier), the epilogue waits (limit ~1 ms) give up, the kernel sets NSHB_DEV_TIMEOUT,
    frees its tensor memory and returns.  A normal step on the same buffers then follows the
    oracle."""
    W = wl.init_weight(21, T, 2 * T, 3 * T, bf16=True).astype(np.float64)
    G = wl.gradient(21, T, 0, 2 * T, 3 * T, bf16=True).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    flags = gs.step("himuon", nshb.params(eta=0.02, tile=T, debug_flags=3))
    assert flags & nshb.NSHB_DEV_TIMEOUT
    gs2 = GpuSet([W], bf16=True)
    gs2.set_grads([G])
    assert gs2.step("himuon", nshb.params(eta=0.02, tile=T, debug_flags=1)) == 0
    _, Mr, Or, _ = o.himuon_step(W, G, np.zeros_like(W), tile=T, eta=0.02, rho=o.fro(W))
    assert rel_fro(gs2.host()[2][0], Or) <= 2e-2


# ---------------------------------------------------------------- Newton-Muon
def test_bf16_newton_muon_small():
    """P = U (Z Z^T + lambda I)^-1 through the tensor-core Gram, the blocked Cholesky with
    256-wide diagonal blocks and split-precision products, and the block solves; then bf16
    NS and Hyperball; against the oracle's plain linear solve.  Layer inputs of 128, 256, 320
    and 576 rows (one to three diagonal blocks, the last one partly padding), matrices with
    row counts that are not multiples of 256, wide and tall."""
    from gpu_harness import newton_step
    cfg = wl.CFG_NEWTON_GPT2
    n_tok = 512
    Zs = [wl.layer_input(cfg, 0, 128, n_tok), wl.layer_input(cfg, 1, 256, n_tok),
          wl.layer_input(cfg, 2, 320, n_tok), wl.layer_input(cfg, 3, 576, n_tok)]
    shapes = [(192, 128), (128, 256), (320, 256), (64, 128), (100, 320), (700, 320), (600, 576)]
    zi = [0, 1, 1, 0, 2, 2, 3]
    Ws = [wl.init_weight(cfg, 40 + i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, 40 + i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    for k in range(len(shapes)):
        gs.mats[k].z_index = zi[k]
    gs.set_grads(Gs)
    rho_dev = torch.tensor(rhos, dtype=torch.float32, device="cuda")
    p = nshb.params(eta=0.02, rho=rho_dev, ridge_rel=1e-3)
    assert newton_step(gs, Zs, n_tok, p) == 0
    Wg, Mg, Og = gs.host()
    for i, W in enumerate(Ws):
        Wr, Mr, Or, _ = o.newton_muon_step(W, Gs[i], np.zeros_like(W), Zs[zi[i]].astype(np.float64),
                                           ridge_rel=1e-3, eta=0.02, rho=rhos[i])
        assert rel_fro(Mg[i], Mr) <= 1e-6
        assert rel_fro(Og[i], Or) <= 2e-2, (i, rel_fro(Og[i], Or))
        assert np.linalg.norm(Wg[i] - Wr) <= bf16_w_tol(Wr, 0.02)
        assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True)


def test_bf16_newton_muon_odd_token_panels():
    """A token count of 320 (five 64-wide panels, so the last 128-deep stage of S = Z Z^T
    runs past the end of Z, where the tensor map reads zeros) and layer inputs of 192 and
    448 rows (the last 256-row tile of S partly past Z's rows)."""
    from gpu_harness import newton_step
    cfg = wl.CFG_NEWTON_GPT2
    n_tok = 320
    Zs = [wl.layer_input(cfg, 20, 192, n_tok), wl.layer_input(cfg, 21, 448, n_tok)]
    shapes = [(256, 192), (130, 448), (448, 448)]
    zi = [0, 1, 1]
    Ws = [wl.init_weight(cfg, 80 + i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, 80 + i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    for k in range(len(shapes)):
        gs.mats[k].z_index = zi[k]
    gs.set_grads(Gs)
    rho_dev = torch.tensor(rhos, dtype=torch.float32, device="cuda")
    p = nshb.params(eta=0.02, rho=rho_dev, ridge_rel=1e-3)
    assert newton_step(gs, Zs, n_tok, p) == 0
    Wg, Mg, Og = gs.host()
    for i, W in enumerate(Ws):
        Wr, Mr, Or, _ = o.newton_muon_step(W, Gs[i], np.zeros_like(W), Zs[zi[i]].astype(np.float64),
                                           ridge_rel=1e-3, eta=0.02, rho=rhos[i])
        assert rel_fro(Og[i], Or) <= 2e-2, (i, rel_fro(Og[i], Or))
        assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True)


def test_bf16_newton_muon_five_diagonal_blocks():
    """A layer input of 1280 rows: five 256-blocks, so the backward runs by 512-wide blocks
    {0, 1}, {2, 3} and a last single block {4}, with the lower-left blocks of the 512-block
    inverses formed at steps 1 and 3; a 300-row input (two blocks, one 512-block) and a 64-row
    one (whose stages start late, staggered across the launches beside the diagonal blocks)
    share the step."""
    from gpu_harness import newton_step
    cfg = wl.CFG_NEWTON_GPT2
    n_tok = 512
    Zs = [wl.layer_input(cfg, 30, 1280, n_tok), wl.layer_input(cfg, 31, 320, n_tok),
          wl.layer_input(cfg, 32, 64, n_tok)]
    shapes = [(384, 1280), (1300, 1280), (320, 320), (96, 64), (64, 64), (200, 320)]
    zi = [0, 0, 1, 2, 2, 1]
    Ws = [wl.init_weight(cfg, 90 + i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, 90 + i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    gs = GpuSet(Ws, bf16=True)
    for k in range(len(shapes)):
        gs.mats[k].z_index = zi[k]
    gs.set_grads(Gs)
    rho_dev = torch.tensor(rhos, dtype=torch.float32, device="cuda")
    p = nshb.params(eta=0.02, rho=rho_dev, ridge_rel=1e-3)
    assert newton_step(gs, Zs, n_tok, p) == 0
    Wg, Mg, Og = gs.host()
    for i, W in enumerate(Ws):
        Wr, Mr, Or, _ = o.newton_muon_step(W, Gs[i], np.zeros_like(W), Zs[zi[i]].astype(np.float64),
                                           ridge_rel=1e-3, eta=0.02, rho=rhos[i])
        assert rel_fro(Og[i], Or) <= 2e-2, (i, rel_fro(Og[i], Or))
        # On a small matrix the step moves most elements by less than half a bf16 ulp, so the
        # storage rounding is correlated with the step and the rounded norm misses rho by more
        # than independent rounding would (2.6e-4 for the 64 x 64 one): the bound adds what the
        # exact projection itself loses when rounded to bf16.
        own = abs(o.fro(wl.round_to_bf16(Wr)) - rhos[i]) / rhos[i]
        assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True) + own


def test_bf16_newton_muon_without_compensated_iterations():
    """ns_compensated = 0: the NS keeps no low part of X, so P's low part, which the
    backward solve needs, gets a buffer of its own (with compensation, the solve writes P's
    hi / lo panels straight into the NS operand).  The preconditioned P has a wide spectrum,
    so the plain bf16 chain loses its small directions to the rounding of X0 (measured: 4.2e-2
    from the oracle here, 9e-3 with the two compensated iterations of the default); the
    bound checks that the step is the plain chain's, not the specification's 2e-2."""
    from gpu_harness import newton_step
    cfg = wl.CFG_NEWTON_GPT2
    n_tok = 512
    Zs = [wl.layer_input(cfg, 40, 576, n_tok), wl.layer_input(cfg, 41, 128, n_tok)]
    shapes = [(700, 576), (300, 576), (128, 128)]
    zi = [0, 0, 1]
    Ws = [wl.init_weight(cfg, 110 + i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, 110 + i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    refs = [o.newton_muon_step(W, Gs[i], np.zeros_like(W), Zs[zi[i]].astype(np.float64),
                               ridge_rel=1e-3, eta=0.02, rho=rhos[i]) for i, W in enumerate(Ws)]
    errs = {}
    for comp in (0, 2):
        gs = GpuSet(Ws, bf16=True)
        for k in range(len(shapes)):
            gs.mats[k].z_index = zi[k]
        gs.set_grads(Gs)
        rho_dev = torch.tensor(rhos, dtype=torch.float32, device="cuda")
        p = nshb.params(eta=0.02, rho=rho_dev, ridge_rel=1e-3, ns_compensated=comp)
        assert newton_step(gs, Zs, n_tok, p) == 0
        Wg, Mg, Og = gs.host()
        errs[comp] = [rel_fro(Og[i], refs[i][2]) for i in range(len(Ws))]
        for i in range(len(Ws)):
            own = abs(o.fro(wl.round_to_bf16(refs[i][0])) - rhos[i]) / rhos[i]
            assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], True) + own
    assert max(errs[2]) <= 2e-2, errs
    assert max(errs[0]) <= 6e-2, errs
    assert all(e0 > e2 for e0, e2 in zip(errs[0], errs[2])), errs


# ------------------------------------------------- determinism, schedules, graphs
def test_steps_are_bit_deterministic():
    """Fixed-order reductions, no float atomics: two runs on the same inputs agree bit for bit."""
    cfg = 21
    shapes = [(768, 768), (3072, 768), (768, 3072), (300, 700)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    outs = []
    for _ in range(2):
        gs = GpuSet(Ws, bf16=True)
        gs.set_grads(Gs)
        assert gs.step("hyperball", nshb.params(eta=0.02)) == 0
        outs.append(gs.host())
    for a, b in zip(outs[0], outs[1]):
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_radial_brake_page_targets_on_gpu():
    """PR #224 test targets 7.5 and 9.0 with exactly representable norms: ||w_prev|| = 5 and
    a plain step to ||w|| = 10 (outward 0.5 -> 7.5); ||w_prev|| = 10 to ||w|| = 8
    (inward 0.5 -> 9.0).  The update is forced through O by a rank-1 gradient whose NS
    output is known: with K = 1 and (a, b, c) = (1, 0, 0), O = U / (||U|| + eps)."""
    import json, pathlib
    g = json.loads((pathlib.Path(__file__).parent / "golden" / "page_values.json").read_text())["radial_brake_targets"]
    for w_prev, w_new, s_out, s_in, target in (([3.0, 4.0], [6.0, 8.0], 0.5, 1.0, g["outward_target"]),
                                               ([6.0, 8.0], [4.8, 6.4], 1.0, 0.5, g["inward_target"])):
        W = np.zeros((8, 8))
        W[0, :2] = w_prev
        D = np.zeros((8, 8))
        D[0, :2] = np.array(w_prev) - np.array(w_new)        # W - lr * O = w_new  =>  lr * O = D
        lr = float(np.linalg.norm(D))                       # O = D / ||D|| (unit), so lr = ||D||
        gs = GpuSet([W], bf16=False)
        gs.set_grads([D])                                   # beta = 0: U = G = D
        p = nshb.params(ns_precision=nshb.NSHB_F32, beta=0.0, ns_steps=1, coeffs=[(1.0, 0.0, 0.0)],
                        lr=lr, brake_out=s_out, brake_in=s_in, ns_eps=1e-30)
        assert gs.step("brake", p) == 0
        assert abs(np.linalg.norm(gs.host()[0][0]) - target) <= 1e-5 * target


def test_momentum_closed_form_on_gpu():
    """Constant G from M0 = 0: after t steps M_t = (1 - beta^t) G (fp32 buffer)."""
    G = wl.gradient(22, 0, 0, 256, 512, bf16=True).astype(np.float64)
    W = wl.init_weight(22, 0, 256, 512, bf16=True).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    beta = 0.9
    for t in range(1, 6):
        assert gs.step("muon", nshb.params(beta=beta, lr=0.0)) == 0
        assert rel_fro(gs.host()[1][0], (1 - beta ** t) * G) <= 1e-6


def test_per_iteration_coefficient_schedule():
    """Per-iteration (a, b, c) rows (the two-stage schedule of the Muon explainer: Keller's
    coefficients, then (2, -1.5, 0.5)) on the tensor-core path."""
    cfg = 23
    table = [o.KELLER_ABC] * 3 + [o.SETTLE_ABC] * 2
    for shape in [(768, 768), (3072, 768)]:
        W = wl.init_weight(cfg, 0, *shape, bf16=True).astype(np.float64)
        G = wl.gradient(cfg, 0, 0, *shape, bf16=True).astype(np.float64)
        gs = GpuSet([W], bf16=True)
        gs.set_grads([G])
        assert gs.step("muon", nshb.params(lr=0.0, coeffs=table)) == 0
        _, U = o.momentum(np.zeros_like(G), G, 0.95, True)
        assert rel_fro(gs.host()[2][0], o.newton_schulz(U, 5, coeffs=table)) <= 2e-2


def test_step_captures_in_a_cuda_graph():
    """The step enqueues only kernels and one memset on the caller's stream: it can be
    captured once and replayed; the replay equals a direct call on the same inputs."""
    cfg = 24
    shapes = [(768, 768), (768, 3072), (3072, 768)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    direct = GpuSet(Ws, bf16=True)
    direct.set_grads(Gs)
    assert direct.step("hyperball", nshb.params(eta=0.02)) == 0
    graphed = GpuSet(Ws, bf16=True)
    graphed.set_grads(Gs)
    p = nshb.params(eta=0.02)
    need = nshb.workspace_size(graphed.mats, p, nshb.NSHB_OP_HYPERBALL)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    nshb.hyperball_step(graphed.mats, p, ws)        # first call outside capture (module set-up)
    torch.cuda.synchronize()
    # reset state and capture
    for w, w0 in zip(graphed.W, Ws):
        w.copy_(torch.from_numpy(w0.astype(np.float32)).to("cuda").to(torch.bfloat16))
    for m in graphed.M:
        m.zero_()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            nshb.hyperball_step(graphed.mats, p, ws, s)
    # capture does not execute: the state is still initial; replay runs the step once
    graph.replay()
    torch.cuda.synchronize()
    assert nshb.device_status(ws) == 0
    for a, b in zip(direct.host(), graphed.host()):
        for x, y in zip(a, b):
            assert np.array_equal(x, y)



def test_newton_muon_step_captures_in_a_cuda_graph():
    """The Newton-Muon step (its launches that run beside the diagonal blocks and wait for
    them at their end included) can be captured once and replayed; the replay equals a direct
    call on the same inputs bit for bit.  Layer inputs of 256 and 768 rows: one and three
    diagonal blocks, so the staged backward of the narrow one runs inside the wide one's
    forward sweep."""
    cfg = wl.CFG_NEWTON_GPT2
    n_tok = 512
    Zs = [wl.layer_input(cfg, 10, 256, n_tok), wl.layer_input(cfg, 11, 768, n_tok)]
    shapes = [(256, 256), (512, 768), (300, 256), (768, 768)]
    zi = [0, 1, 0, 1]
    Ws = [wl.init_weight(cfg, 60 + i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, 60 + i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rho = torch.tensor([o.fro(w) for w in Ws], dtype=torch.float32, device="cuda")
    p = nshb.params(eta=0.02, rho=rho, ridge_rel=1e-3)
    Zd = [torch.from_numpy(z.astype(np.float32)).to("cuda").to(torch.bfloat16) for z in Zs]
    z_rows = [z.shape[0] for z in Zs]

    def make_set():
        gs = GpuSet(Ws, bf16=True)
        for k in range(len(shapes)):
            gs.mats[k].z_index = zi[k]
        gs.set_grads(Gs)
        need = nshb.workspace_size(gs.mats, p, nshb.NSHB_OP_NEWTON_MUON, z_rows, n_tok)
        return gs, torch.empty(need, dtype=torch.uint8, device="cuda")

    direct, ws_d = make_set()
    nshb.newton_muon_step(direct.mats, Zd, n_tok, p, ws_d)
    assert nshb.device_status(ws_d) == 0
    graphed, ws = make_set()
    nshb.newton_muon_step(graphed.mats, Zd, n_tok, p, ws)   # first call outside capture (module set-up)
    torch.cuda.synchronize()
    for w, w0 in zip(graphed.W, Ws):
        w.copy_(torch.from_numpy(w0.astype(np.float32)).to("cuda").to(torch.bfloat16))
    for m in graphed.M:
        m.zero_()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            nshb.newton_muon_step(graphed.mats, Zd, n_tok, p, ws, s)
    graph.replay()
    torch.cuda.synchronize()
    assert nshb.device_status(ws) == 0
    for a, b in zip(direct.host(), graphed.host()):
        for x, y in zip(a, b):
            assert np.array_equal(x, y)

def test_thirteen_shapes_in_one_call():
    """Thirteen distinct padded shapes in one call (every GEMM launch mixes problems of
    different sizes and k depths); every matrix against the oracle, and the first two run
    alone agree with their results in the mixed call."""
    cfg = 25
    shapes = [(256 * a, 256 * b) for a, b in [(1, 1), (1, 2), (2, 1), (1, 3), (3, 1), (2, 2), (1, 4), (4, 1),
                                                (2, 3), (3, 2), (1, 5), (5, 1), (3, 3)]]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    gs = GpuSet(Ws, bf16=True)
    gs.set_grads(Gs)
    assert gs.step("muon", nshb.params(lr=0.0)) == 0
    Og = gs.host()[2]
    for i in range(len(shapes)):
        _, U = o.momentum(np.zeros_like(Gs[i]), Gs[i], 0.95, True)
        assert rel_fro(Og[i], o.newton_schulz(U)) <= 2e-2, i
    single = GpuSet(Ws[:2], bf16=True)
    single.set_grads(Gs[:2])
    assert single.step("muon", nshb.params(lr=0.0)) == 0
    for i in range(2):
        assert rel_fro(single.host()[2][i], Og[i]) <= 2e-2


# ------------------------------------------------------------------ degenerate inputs
@pytest.mark.parametrize("shape", [(1, 1), (1, 9), (9, 1), (1, 300), (300, 1)])
def test_bf16_degenerate_shapes_hyperball(shape):
    """Single rows, columns and scalars on the tensor-core path (padded to 256 inside): a
    rank-1 U has one singular value, normalised to 1, mapped by the scalar polynomial."""
    cfg = 26
    W = wl.init_weight(cfg, 0, *shape, bf16=True).astype(np.float64)
    G = wl.gradient(cfg, 0, 0, *shape, bf16=True).astype(np.float64)
    rho = o.fro(W)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    rho_dev = torch.tensor([rho], dtype=torch.float32, device="cuda")
    assert gs.step("hyperball", nshb.params(eta=0.02, rho=rho_dev)) == 0
    Wg, Mg, Og = gs.host()
    Wr, Mr, Or, fb = o.hyperball_step(W, G, np.zeros_like(W), eta=0.02, rho=rho)
    assert rel_fro(Mg[0], Mr) <= 1e-6
    assert rel_fro(Og[0], Or) <= 2e-2
    assert np.linalg.norm(Wg[0] - Wr) <= bf16_w_tol(Wr, 0.02)
    # the single stretch of a rank-1 U is the scalar map of ||U|| / (||U|| + eps)
    _, U = o.momentum(np.zeros_like(G), G, 0.95, True)
    s = np.linalg.svd(Og[0], compute_uv=False)[0]
    assert abs(s - float(o.scalar_ns(o.fro(U) / (o.fro(U) + o.NS_EPS), 5))) <= 2e-2


def test_zero_gradient_leaves_weights_on_their_sphere():
    """G = 0: U = 0, the NS output is 0 (0 / (0 + eps)), U_hat = 0, and W <- rho W / ||W||."""
    shapes = [(256, 256), (768, 3072), (5, 7)]
    Ws = [wl.init_weight(27, i, r, c, bf16=True).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    gs = GpuSet(Ws, bf16=True)
    gs.set_grads([np.zeros_like(w) for w in Ws])
    rho = torch.tensor([o.fro(w) for w in Ws], dtype=torch.float32, device="cuda")
    assert gs.step("hyperball", nshb.params(eta=0.02, rho=rho)) == 0
    Wg, Mg, Og = gs.host()
    for i, W in enumerate(Ws):
        assert not np.any(Og[i]) and not np.any(Mg[i])
        Wr, fb = o.hyperball_apply(W, np.zeros_like(W), 0.02, o.fro(W))
        assert not fb
        assert np.linalg.norm(Wg[i] - Wr) <= bf16_w_tol(Wr, 0.0), i


def test_zero_weight_with_current_norm_as_radius_reports_zero_radius():
    """rho taken from the current norm (NULL rho) of an all-zero W: the hook's error case;
    here the status bit NSHB_DEV_ZERO_RADIUS is set and W stays zero."""
    W = np.zeros((128, 256))
    G = wl.gradient(28, 0, 0, 128, 256, bf16=True).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    flags = gs.step("hyperball", nshb.params(eta=0.02))
    assert flags & nshb.NSHB_DEV_ZERO_RADIUS
    assert not np.any(gs.host()[0][0])


# ------------------------------------- partials from the Newton-Schulz epilogues
@pytest.mark.parametrize("kind,ld_pad,w_dtype", [
    ("hyperball", 8, torch.bfloat16),    # rows 16-byte aligned: vector reads of W in the epilogue
    ("hyperball", 5, torch.bfloat16),    # odd leading dimension: element reads
    ("hyperball", 0, torch.float32),     # fp32 weights with the bf16 chain
    ("brake", 3, torch.bfloat16),
    ("himuon256", 5, torch.bfloat16),    # tile-resident kernels
    ("himuon128", 8, torch.bfloat16),
    ("himuon512", 3, torch.bfloat16),    # tiles on the pair GEMM
])
def test_partials_from_ns_epilogue_follow_the_oracle(kind, ld_pad, w_dtype):
    """||O||^2, <W,O> and ||W||^2 come from the epilogue that writes the final O, which reads
    the caller's W there: wide, tall (the transposed read) and ragged shapes, W held as a
    strided view (ld > cols) and as fp32.  W after the step against the oracle and on its
    sphere."""
    cfg = 29
    shapes = [(300, 700), (700, 300), (512, 256), (256, 1024)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=w_dtype == torch.bfloat16).astype(np.float64)
          for i, (r, c) in enumerate(shapes)]
    Gs = [wl.gradient(cfg, i, 0, r, c, bf16=w_dtype == torch.bfloat16).astype(np.float64)
          for i, (r, c) in enumerate(shapes)]
    W, G, M, O = [], [], [], []
    for (r, c), w0, g0 in zip(shapes, Ws, Gs):
        big = torch.zeros(r, c + ld_pad, dtype=w_dtype, device="cuda")
        W.append(big[:, :c])
        W[-1].copy_(torch.from_numpy(w0.astype(np.float32)))
        gbig = torch.zeros_like(big)
        G.append(gbig[:, :c])
        G[-1].copy_(torch.from_numpy(g0.astype(np.float32)))
        M.append(torch.zeros(r, c + ld_pad, dtype=torch.float32, device="cuda")[:, :c])
        O.append(torch.empty(r, c, dtype=w_dtype, device="cuda"))
    rho = torch.tensor([o.fro(w) for w in Ws], dtype=torch.float32, device="cuda")
    mats = nshb.matrices(W, G, M, O)
    tile = int(kind[6:]) if kind.startswith("himuon") else 256
    if kind == "brake":
        p = nshb.params(lr=0.02, brake_out=0.5, brake_in=1.0)
        op, fn = nshb.NSHB_OP_RADIAL_BRAKE, nshb.radial_brake_step
    elif kind == "hyperball":
        p = nshb.params(eta=0.02, rho=rho)
        op, fn = nshb.NSHB_OP_HYPERBALL, nshb.hyperball_step
    else:
        p = nshb.params(eta=0.02, rho=rho, tile=tile)
        op, fn = nshb.NSHB_OP_HIMUON, nshb.himuon_step
    ws = nshb.workspace(mats, p, op)
    fn(mats, p, ws)
    assert nshb.device_status(ws) == 0
    bf16 = w_dtype == torch.bfloat16
    for i, (w0, g0) in enumerate(zip(Ws, Gs)):
        if kind == "brake":
            Wr, _, Or = o.radial_brake_step(w0, g0, np.zeros_like(w0), lr=0.02, outward=0.5, inward=1.0)
        elif kind == "hyperball":
            Wr, _, Or, _ = o.hyperball_step(w0, g0, np.zeros_like(w0), eta=0.02, rho=o.fro(w0))
        else:
            Wr, _, Or, _ = o.himuon_step(w0, g0, np.zeros_like(w0), tile=tile, eta=0.02, rho=o.fro(w0))
        Wg = W[i].double().cpu().numpy()
        assert rel_fro(O[i].double().cpu().numpy(), Or) <= 2e-2, i
        step_len = 0.02 * (o.shape_scale(*w0.shape) * o.fro(Or) if kind == "brake" else 1.0)
        tol = bf16_w_tol(Wr, step_len) if bf16 else 2 * 2e-2 * step_len + 1e-6 * o.fro(Wr)
        assert np.linalg.norm(Wg - Wr) <= tol, (i, np.linalg.norm(Wg - Wr), tol)
        if kind != "brake":
            assert abs(o.fro(Wg) - o.fro(w0)) / o.fro(w0) <= radius_tol(Wg, bf16), i
