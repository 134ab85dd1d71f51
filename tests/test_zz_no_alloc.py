"""The allocation-free norm entry point (nshb_fro_norms_static).

It serves callers that cannot allocate device memory and so cannot pass a workspace: its
scratch is a fixed array inside the library.  The GPU test checks it against the
workspace-based nshb_fro_norms on two calls in a row (the shared scratch keeps the previous
call's contents, which must not leak into the next result).  This file is collected last.
"""

import numpy as np
import pytest

import newton_schulz_hyperball_b200 as nshb


def _fake(shapes):
    arr = (nshb.nshb_matrix * len(shapes))()
    for i, (r, c) in enumerate(shapes):
        arr[i].rows, arr[i].cols, arr[i].ld = r, c, c
        arr[i].w_dtype = nshb.NSHB_BF16
        arr[i].W = 0x10000000 * (i + 1)
    return arr


def test_static_norms_reject_sizes_beyond_the_scratch():
    lib = nshb.lib()
    big = _fake([(30000, 30000)])              # 469^2 blocks > the fixed capacity
    assert lib.nshb_fro_norms_static(big, 1, 0x1000, None) == nshb.NSHB_ERR_WORKSPACE
    many = _fake([(8, 8)] * 193)               # more matrices than one call handles
    assert lib.nshb_fro_norms_static(many, 193, 0x1000, None) == nshb.NSHB_ERR_WORKSPACE
    assert lib.nshb_fro_norms_static(_fake([(8, 8)]), 1, None, None) == nshb.NSHB_ERR_NULL


@pytest.mark.gpu
def test_static_norms_match_workspace_norms_twice():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from newton_schulz_hyperball_b200 import workloads as wl
    dev = "cuda"
    shapes = [(768, 768), (3072, 768), (768, 3072), (5, 7), (300, 700), (130, 1)]
    for call, seed in enumerate((21, 22)):     # two calls in a row, different weights
        W = [torch.from_numpy(wl.init_weight(seed, i, r, c, bf16=True)).to(dev).to(torch.bfloat16)
             for i, (r, c) in enumerate(shapes)]
        W.append(torch.from_numpy(wl.init_weight(seed, 9, 257, 129, bf16=False)).to(dev))
        G = [torch.zeros_like(w) for w in W]
        M = [torch.zeros(w.shape, dtype=torch.float32, device=dev) for w in W]
        mats = nshb.matrices(W, G, M)
        ref = torch.full((len(W),), -1.0, dtype=torch.float32, device=dev)
        got = torch.full((len(W),), -1.0, dtype=torch.float32, device=dev)
        ws = nshb.workspace(mats, nshb.params(), nshb.NSHB_OP_MUON)
        nshb.fro_norms(mats, ref, ws)
        nshb.fro_norms_static(mats, got)
        torch.cuda.synchronize()
        r = ref.cpu().numpy().astype(np.float64)
        g = got.cpu().numpy().astype(np.float64)
        exact = np.array([np.linalg.norm(w.float().cpu().numpy().astype(np.float64)) for w in W])
        assert np.all(np.abs(g - r) <= 1e-6 * r), (call, g, r)
        assert np.all(np.abs(g - exact) <= 1e-5 * exact), (call, g, exact)
