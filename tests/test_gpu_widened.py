"""GPU parity of the widened update rules against the oracle: the RelativeUpdate hook on
Muon and AdamH (Hyperball around Adam's bias-corrected direction).  Seeded inputs from
the shared generators; the oracle keeps its own state across steps."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import newton_schulz_hyperball_b200 as nshb  # noqa: E402
from newton_schulz_hyperball_b200 import workloads as wl  # noqa: E402
from oracle import nshb_oracle as o  # noqa: E402
from gpu_harness import GpuSet, rel_fro, to_dev, to_host  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"
# The ABI carries Adam's parameters in fp32; the oracle gets the same (rounded) values.
B1, B2, AEPS = (float(np.float32(x)) for x in (o.ADAM_BETA1, o.ADAM_BETA2, o.ADAM_EPS))


def half_ulp_norm(W):
    a = np.abs(W)
    e = np.floor(np.log2(np.maximum(a, 1e-38)))
    return float(np.linalg.norm(np.where(a > 0, 2.0 ** (e - 8), 0.0)))


def radius_tol(W, bf16):
    if not bf16:
        return 1e-5
    w2 = np.sum(W * W)
    return 1e-5 + 6 * (2.0 ** -9 / math.sqrt(3)) * math.sqrt(np.sum(W ** 4)) / w2


# ------------------------------------------------------------------ RelativeUpdate
@pytest.mark.parametrize("bf16", [True, False])
def test_relative_update_matches_oracle(bf16):
    """Step length lr * ||W|| along O: W within storage rounding plus the 2e-2 direction
    error (bf16 NS) or 1e-4 (fp32 NS) of the oracle, two steps with the oracle's own state."""
    cfg = 51
    shapes = [(768, 768), (3072, 768), (768, 3072), (300, 700)] if bf16 else [(256, 256), (192, 320)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=bf16).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    Ms = [np.zeros_like(w) for w in Ws]
    Wr = [w.copy() for w in Ws]
    gs = GpuSet(Ws, bf16=bf16)
    lr, wd = 0.02, 0.1
    kw = dict(lr=lr, weight_decay=wd) if bf16 else dict(lr=lr, weight_decay=wd, ns_precision=nshb.NSHB_F32)
    for step in range(2):
        Gs = [wl.gradient(cfg, i, step, r, c, bf16=bf16).astype(np.float64) for i, (r, c) in enumerate(shapes)]
        gs.set_grads(Gs)
        W_before = gs.host()[0]
        need = nshb.workspace_size(gs.mats, nshb.params(**kw), nshb.NSHB_OP_RELATIVE_UPDATE)
        ws = torch.empty(need, dtype=torch.uint8, device=DEV)
        nshb.relative_update_step(gs.mats, nshb.params(**kw), ws)
        assert nshb.device_status(ws) == 0
        Wg, Mg, Og = gs.host()
        for i in range(len(shapes)):
            Wr[i], Ms[i], Or = o.relative_update_step(Wr[i], Gs[i], Ms[i], lr=lr, weight_decay=wd)
            step_len = lr * o.fro(W_before[i])
            if bf16:
                tol = (step + 1) * (half_ulp_norm(Wr[i]) + 2 * 2e-2 * step_len)
            else:
                tol = (step + 1) * 1e-4 * step_len + 1e-6 * o.fro(Wr[i])
            assert np.linalg.norm(Wg[i] - Wr[i]) <= tol, (i, np.linalg.norm(Wg[i] - Wr[i]), tol)
            # the defining property on the GPU's own numbers: ||(1 - lr wd) W - W_new|| = lr ||W||
            d = o.fro((1 - lr * wd) * W_before[i] - Wg[i])
            assert abs(d - step_len) <= (2e-3 if bf16 else 1e-5) * step_len + half_ulp_norm(Wg[i]) * bf16, i


# ------------------------------------------------------------------ AdamH
@pytest.mark.parametrize("bf16", [True, False])
def test_adamh_three_steps_match_oracle(bf16):
    cfg = 52
    shapes = [(768, 768), (3072, 768), (300, 700), (5, 7)] if bf16 else [(256, 256), (192, 320), (5, 7)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=bf16).astype(np.float64) for i, (r, c) in enumerate(shapes)]
    rhos = [o.fro(w) for w in Ws]
    Mr = [np.zeros_like(w) for w in Ws]
    Vr = [np.zeros_like(w) for w in Ws]
    Wr = [w.copy() for w in Ws]
    gs = GpuSet(Ws, bf16=bf16)
    V = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in Ws]
    rho_dev = torch.tensor(rhos, dtype=torch.float32, device=DEV)
    eta = 0.02
    p = nshb.params(eta=eta, rho=rho_dev)
    need = nshb.workspace_size(gs.mats, p, nshb.NSHB_OP_ADAMH)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    for t in range(1, 4):
        Gs = [wl.gradient(cfg, i, t, r, c, bf16=bf16).astype(np.float64) for i, (r, c) in enumerate(shapes)]
        gs.set_grads(Gs)
        nshb.adamh_step(gs.mats, V, nshb.adam_params(step=t), p, ws)
        assert nshb.device_status(ws) == 0
        Wg, Mg, Ug = gs.host()
        for i in range(len(shapes)):
            Wr[i], Mr[i], Vr[i], Ur, fb = o.adamh_step(Wr[i], Gs[i], Mr[i], Vr[i], t=t, eta=eta, rho=rhos[i],
                                                       beta1=B1, beta2=B2, adam_eps=AEPS)
            assert not fb
            assert rel_fro(Mg[i], Mr[i]) <= 1e-6, (t, i)
            assert rel_fro(to_host(V[i]), Vr[i]) <= 1e-6, (t, i)
            # U~ is kept in the weight dtype: bf16 rounding (2^-9 relative per entry)
            assert rel_fro(Ug[i], Ur) <= (4e-3 if bf16 else 1e-5), (t, i, rel_fro(Ug[i], Ur))
            tol = t * (half_ulp_norm(Wr[i]) + 2 * 4e-3 * eta) if bf16 else t * 1e-5 * eta + 1e-6 * rhos[i]
            assert np.linalg.norm(Wg[i] - Wr[i]) <= tol, (t, i, np.linalg.norm(Wg[i] - Wr[i]), tol)
            assert abs(o.fro(Wg[i]) - rhos[i]) / rhos[i] <= radius_tol(Wg[i], bf16), (t, i)


def test_adamh_first_step_is_the_sign_direction():
    """Step 1 from zero moments: U~ = g / (|g| + eps) = sign(g) for gradients far above eps."""
    cfg = 53
    W = wl.init_weight(cfg, 0, 512, 384, bf16=True).astype(np.float64)
    G = wl.gradient(cfg, 0, 0, 512, 384, bf16=True).astype(np.float64)
    gs = GpuSet([W], bf16=True)
    gs.set_grads([G])
    V = [torch.zeros(W.shape, dtype=torch.float32, device=DEV)]
    p = nshb.params(eta=0.02)
    ws = torch.empty(nshb.workspace_size(gs.mats, p, nshb.NSHB_OP_ADAMH), dtype=torch.uint8, device=DEV)
    nshb.adamh_step(gs.mats, V, nshb.adam_params(), p, ws)
    assert nshb.device_status(ws) == 0
    U = gs.host()[2][0]
    big = np.abs(G) > 1e-5
    assert np.array_equal(np.sign(U[big]), np.sign(G[big]))
    assert np.allclose(np.abs(U[big]), 1.0, rtol=2e-3)


def test_adamh_full_gpt2_set_radius_and_sampled_parity():
    """All 72 GPT-2-small matrices in one call (as the bench times it): the radius of every
    matrix, and layer 0's six matrices against the oracle."""
    cfg = wl.CFG_GPT2_SMALL
    shapes = [(r, c) for _, r, c in wl.gpt2_small_shapes(12)]
    Ws = [wl.init_weight(cfg, i, r, c, bf16=True).astype(np.float64) if i < 6 else None
          for i, (r, c) in enumerate(shapes)]
    g = torch.Generator(device=DEV)
    g.manual_seed(7)
    W = [to_dev(Ws[i], True) if i < 6 else (0.02 * torch.randn(r, c, device=DEV, generator=g)).to(torch.bfloat16)
         for i, (r, c) in enumerate(shapes)]
    Gh = [wl.gradient(cfg, i, 0, r, c, bf16=True).astype(np.float64) if i < 6 else None
          for i, (r, c) in enumerate(shapes)]
    G = [to_dev(Gh[i], True) if i < 6 else (1e-3 * torch.randn(r, c, device=DEV, generator=g)).to(torch.bfloat16)
         for i, (r, c) in enumerate(shapes)]
    M = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W]
    V = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in W]
    rho = torch.stack([w.float().norm() for w in W])
    mats = nshb.matrices(W, G, M)
    p = nshb.params(eta=0.02, rho=rho)
    ws = nshb.workspace(mats, p, nshb.NSHB_OP_ADAMH)
    nshb.adamh_step(mats, V, nshb.adam_params(), p, ws)
    assert nshb.device_status(ws) == 0
    for i in range(len(shapes)):
        w = to_host(W[i])
        assert abs(o.fro(w) - float(rho[i])) / float(rho[i]) <= radius_tol(w, True), i
    for i in range(6):
        Wn, _, _, _, _ = o.adamh_step(Ws[i], Gh[i], np.zeros_like(Ws[i]), np.zeros_like(Ws[i]), t=1, eta=0.02,
                                      rho=float(rho[i]), beta1=B1, beta2=B2, adam_eps=AEPS)
        assert np.linalg.norm(to_host(W[i]) - Wn) <= half_ulp_norm(Wn) + 2 * 4e-3 * 0.02, i
