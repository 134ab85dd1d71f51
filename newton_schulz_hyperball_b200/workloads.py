"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module only draws random numbers and shapes; it holds none of the
optimizer's arithmetic.  Every array is produced on the host from
``numpy.random.SeedSequence([config, matrix, step, tag])`` so that both sides
of a parity check receive the very same stored values.

Tags: 0 = W0, 1 = gradient noise E, 2 = spike factor A, 3 = spike factor B,
4 = per-matrix sigma, 5 = Z, 6 = Z per-feature scales.

Shapes follow the matrix sets the optimizer papers train: GPT-2 small,
a Qwen3-style ~1.2B model, 8B-width layers (Hierarchical Muon) and the GPT-2
layer inputs for Newton-Muon.
"""
from __future__ import annotations

import numpy as np

CFG_SINGLE_F32 = 1
CFG_GPT2_SMALL = 2
CFG_QWEN3_1B = 3
CFG_8B_WIDTH = 4
CFG_NEWTON_GPT2 = 5


def gpt2_small_shapes(layers: int = 12):
    """12 x {Wq, Wk, Wv, Wo 768x768; W_fc 3072x768; W_proj 768x3072} (rows x cols)."""
    out = []
    for l in range(layers):
        for name, r, c in (("wq", 768, 768), ("wk", 768, 768), ("wv", 768, 768), ("wo", 768, 768),
                           ("w_fc", 3072, 768), ("w_proj", 768, 3072)):
            out.append((f"h{l}.{name}", r, c))
    return out


def qwen3_1b_shapes(layers: int = 28):
    """28 x {Wq 2048^2, Wk/Wv 1024x2048, Wo 2048^2, gate/up 6144x2048, down 2048x6144}."""
    out = []
    for l in range(layers):
        for name, r, c in (("wq", 2048, 2048), ("wk", 1024, 2048), ("wv", 1024, 2048), ("wo", 2048, 2048),
                           ("gate", 6144, 2048), ("up", 6144, 2048), ("down", 2048, 6144)):
            out.append((f"l{l}.{name}", r, c))
    return out


def width_8b_shapes(layers: int = 32):
    """32 x {4096^2 x2, 1024x4096 x2, 14336x4096 x2, 4096x14336}."""
    out = []
    for l in range(layers):
        for name, r, c in (("wq", 4096, 4096), ("wo", 4096, 4096), ("wk", 1024, 4096), ("wv", 1024, 4096),
                           ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336)):
            out.append((f"l{l}.{name}", r, c))
    return out


def newton_gpt2_z_index(shapes):
    """Which layer input each GPT-2 matrix right-multiplies: Wq/Wk/Wv share one Z,
    Wo, W_fc and W_proj get their own.  Returns (z_index per matrix, z_rows per Z)."""
    z_index, z_rows = [], []
    cur_layer, qkv = None, None
    for name, r, c in shapes:
        layer, kind = name.split(".")
        if kind in ("wq", "wk", "wv"):
            if qkv is None or cur_layer != layer:
                qkv = len(z_rows)
                z_rows.append(c)
                cur_layer = layer
            z_index.append(qkv)
        else:
            z_index.append(len(z_rows))
            z_rows.append(c)
    return z_index, z_rows


def _rng(cfg: int, matrix: int, step: int, tag: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg, matrix, step, tag])))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def init_weight(cfg: int, idx: int, rows: int, cols: int, bf16: bool, std: float = 0.02) -> np.ndarray:
    """W0 ~ N(0, std^2)."""
    w = _rng(cfg, idx, 0, 0).standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    return round_to_bf16(w) if bf16 else w


def grad_sigma(cfg: int, idx: int, lo: float = 1e-4, hi: float = 1e-2) -> float:
    """Per-matrix gradient scale, log-uniform in [lo, hi]."""
    u = _rng(cfg, idx, 0, 4).random()
    return float(np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo))))


def gradient(cfg: int, idx: int, step: int, rows: int, cols: int, bf16: bool,
             sigma: float | None = None, spike_rank: int = 8, spike_rms: float = 10.0) -> np.ndarray:
    """G = sigma * (E + (spike_rms / sqrt(k)) * A B^T): Gaussian noise plus a fixed
    rank-k spike whose entries have RMS spike_rms * sigma.  E is fresh each step,
    the spike factors A (rows x k) and B (cols x k) are fixed per matrix."""
    if sigma is None:
        sigma = grad_sigma(cfg, idx)
    g = _rng(cfg, idx, step, 1).standard_normal((rows, cols), dtype=np.float32)
    if spike_rank > 0:
        a = _rng(cfg, idx, 0, 2).standard_normal((rows, spike_rank), dtype=np.float32)
        b = _rng(cfg, idx, 0, 3).standard_normal((cols, spike_rank), dtype=np.float32)
        g += np.float32(spike_rms / np.sqrt(spike_rank)) * (a @ b.T)
    g *= np.float32(sigma)
    return round_to_bf16(g) if bf16 else g


def plain_gradient(cfg: int, idx: int, step: int, rows: int, cols: int, std: float, bf16: bool) -> np.ndarray:
    """G ~ N(0, std^2) with no spike (the single-matrix fp32 case)."""
    g = _rng(cfg, idx, step, 1).standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    return round_to_bf16(g) if bf16 else g


def layer_input(cfg: int, zidx: int, d_in: int, n_tokens: int, lo: float = 0.1, hi: float = 10.0,
                step: int = 0) -> np.ndarray:
    """Z = diag(e^u) E with E ~ N(0,1) (d_in x n_tokens) and u ~ U(ln lo, ln hi); bf16 values."""
    u = _rng(cfg, zidx, step, 6).uniform(np.log(lo), np.log(hi), size=(d_in, 1)).astype(np.float32)
    e = _rng(cfg, zidx, step, 5).standard_normal((d_in, n_tokens), dtype=np.float32)
    return round_to_bf16(np.exp(u) * e)


def spectrum_matrix(seed: int, rows: int, cols: int, sigma, factors: bool = False):
    """A rows x cols float32 matrix Q1 diag(sigma) Q2^T with random orthonormal factors
    (singular values given; the rest zero).  With factors=True also returns (Q1, Q2)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([99, seed])))
    k = len(sigma)
    q1, _ = np.linalg.qr(rng.standard_normal((rows, k)))
    q2, _ = np.linalg.qr(rng.standard_normal((cols, k)))
    m = ((q1 * np.asarray(sigma, dtype=np.float64)) @ q2.T).astype(np.float32)
    return (m, q1, q2) if factors else m
