"""Helpers for the GPU parity tests: move seeded host arrays to the device, run a step
through the C ABI, bring the results back as float64 NumPy arrays."""
from __future__ import annotations

import numpy as np
import torch

import newton_schulz_hyperball_b200 as nshb

DEV = "cuda"


def to_dev(x: np.ndarray, bf16: bool) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(DEV)
    return t.to(torch.bfloat16) if bf16 else t


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class GpuSet:
    """Device copies of W, G, M (+ O_out) for a list of matrices."""

    def __init__(self, Ws, bf16: bool, want_o: bool = True):
        self.bf16 = bf16
        self.W = [to_dev(w, bf16) for w in Ws]
        self.G = [torch.zeros_like(w) for w in self.W]
        self.M = [torch.zeros(w.shape, dtype=torch.float32, device=DEV) for w in self.W]
        self.O = [torch.zeros_like(w) for w in self.W] if want_o else None
        self.mats = nshb.matrices(self.W, self.G, self.M, self.O)
        self.ws = None

    def set_grads(self, Gs):
        for g, h in zip(self.G, Gs):
            g.copy_(to_dev(h, self.bf16))

    def step(self, kind: str, p):
        op = {"muon": nshb.NSHB_OP_MUON, "hyperball": nshb.NSHB_OP_HYPERBALL,
              "brake": nshb.NSHB_OP_RADIAL_BRAKE, "himuon": nshb.NSHB_OP_HIMUON}[kind]
        need = nshb.workspace_size(self.mats, p, op)
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=DEV)
        getattr(nshb, {"muon": "muon_step", "hyperball": "hyperball_step", "brake": "radial_brake_step",
                       "himuon": "himuon_step"}[kind])(self.mats, p, self.ws)
        return nshb.device_status(self.ws)

    def host(self):
        return ([to_host(w) for w in self.W], [to_host(m) for m in self.M],
                [to_host(o) for o in self.O] if self.O is not None else None)


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def newton_step(gs: "GpuSet", Zs, n_tokens: int, p):
    """Runs newton_muon_step on a GpuSet whose matrices carry z_index; Zs are host arrays."""
    Zd = [to_dev(z, True) for z in Zs]
    need = nshb.workspace_size(gs.mats, p, nshb.NSHB_OP_NEWTON_MUON, [z.shape[0] for z in Zs], n_tokens)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=DEV)
    nshb.newton_muon_step(gs.mats, Zd, n_tokens, p, ws)
    return nshb.device_status(ws)
