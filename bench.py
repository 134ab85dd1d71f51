"""Benchmark of the Muon-Hyperball optimizer step on B200.

Workload (one step = the whole hot path over one batch of synthetic input): the GPT-2-small
matrix set -- 12 layers x {Wq, Wk, Wv, Wo 768x768; W_fc 3072x768; W_proj 768x3072}, 72
matrices, 84,934,656 parameters -- with bf16 weights and gradients, fp32 momentum, Nesterov
beta = 0.95, K = 5 quintic Newton-Schulz iterations on the tensor cores, and the Hyperball
rule with rho = ||W0||_F per matrix and eta = 0.02.  Gradients are seeded N(0, sigma^2) noise
plus a rank-8 spike of RMS 10 sigma, sigma log-uniform in [1e-4, 1e-2] per matrix; four
gradient sets rotate so every step sees a fresh one.  Inputs (W + G + M, 680 MB) are larger
than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One JSON line is printed by rank 0.  Under torchrun (N > 1) every rank runs its own replica
of the matrix set on its own GPU (weak scaling, no collective on the data path); the time is
the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Muon-H optimizer step ms; NS TFLOP/s (% bf16 peak); fused-kernel HBM GB/s"
WORKLOAD = "gpt2-small matrix set, MuonH step (72 bf16 matrices, fp32 momentum, K=5, Hyperball)"
ETA = 0.02
N_GRAD_SETS = 4
E2E_PIPELINE = "H2D of step k+1 on a second stream during step k (2 device buffers)"
DEFAULT_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM read + write per launch of the NS GEMM from the ncu capture summarised in
# profiles/gemm_tc2_gpt2_small_ns_iteration1.md, valid only for the kernel source it was taken on.
GEMM_SOURCE = os.path.join(ROOT, "newton_schulz_hyperball_b200", "csrc", "ns_tc2.cu")
GEMM_TRAFFIC = {"sha256_prefix": "3b2c50016d8520e6", "bytes_per_launch": 372400725}


# DRAM read + write per launch of adam_kernel from the capture summarised in
# profiles/adam_kernel_gpt2_small_step.md, valid only for the source it was taken on.
STREAM_SOURCE = os.path.join(ROOT, "newton_schulz_hyperball_b200", "csrc", "stream_kernels.cu")
ADAM_TRAFFIC = {"sha256_prefix": "705031530c8503d1", "bytes_per_launch": 1814096720}


def source_traffic(path, rec):
    import hashlib
    try:
        with open(path, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return rec["bytes_per_launch"] if h == rec["sha256_prefix"] else None


def gemm_traffic():
    import hashlib
    try:
        with open(GEMM_SOURCE, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return GEMM_TRAFFIC["bytes_per_launch"] if h == GEMM_TRAFFIC["sha256_prefix"] else None


def shapes():
    from newton_schulz_hyperball_b200 import workloads as wl
    return [(r, c) for _, r, c in wl.gpt2_small_shapes(12)]


def ns_flops(shp, K=5, dense=False):
    """Algorithmic NS work per step: K (3 r^2 s + r^3), symmetric products counted once;
    dense=True gives the dense-equivalent K (4 r^2 s + 2 r^3) of the full products."""
    tot = 0.0
    for r, c in shp:
        rr, ss = min(r, c), max(r, c)
        tot += K * ((4.0 * rr * rr * ss + 2.0 * rr ** 3) if dense else (3.0 * rr * rr * ss + rr ** 3))
    return tot


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(DEFAULT_PEAKS), "fallback"


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.02)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ workload
def build_inputs(dev, rank: int):
    """Host-side seeded inputs (bf16 values as float32 arrays) for the 72 matrices."""
    import numpy as np
    from newton_schulz_hyperball_b200 import workloads as wl
    cfg = wl.CFG_GPT2_SMALL
    shp = shapes()
    W0 = [wl.init_weight(cfg, i, r, c, bf16=True) for i, (r, c) in enumerate(shp)]
    G = [[wl.gradient(cfg, i, s, r, c, bf16=True) for i, (r, c) in enumerate(shp)] for s in range(N_GRAD_SETS)]
    return W0, G


def timed_e2e(Gh, W, M, run_step, ws, stream, ke, nshb, torch):
    """End to end through the public API with host buffers: every step's gradients are copied
    host->device from pinned memory and the step's device status word is read back.  The copy
    of step k+1 runs on a second stream while step k computes (two device buffers, events
    in both directions), as an input pipeline would; all copies lie inside the timed region."""
    Gpin = [[torch.from_numpy(g).to(torch.bfloat16).pin_memory() for g in gs] for gs in Gh[:2]]
    bufs = [[torch.empty(g.shape, dtype=torch.bfloat16, device=W[0].device) for g in Gpin[0]] for _ in range(2)]
    mats_b = [nshb.matrices(W, bufs[j], M) for j in range(2)]
    st_host = torch.empty(1, dtype=torch.int32).pin_memory()
    h2d = sum(g.numel() * g.element_size() for g in Gpin[0])
    copy_stream = torch.cuda.Stream(device=W[0].device)
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    copy_stream.wait_event(t0)

    def issue_copy(k):
        j = k % 2
        with torch.cuda.stream(copy_stream):
            if k >= 2:
                copy_stream.wait_event(consumed[j])
            for d, s_ in zip(bufs[j], Gpin[k % 2]):
                d.copy_(s_, non_blocking=True)
            copied[j].record(copy_stream)

    issue_copy(0)
    for k in range(ke):
        if k + 1 < ke:
            issue_copy(k + 1)
        j = k % 2
        stream.wait_event(copied[j])
        run_step(mats_b[j], k)
        consumed[j].record(stream)
        st_host.copy_(ws[:4].view(torch.int32), non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / ke, h2d


def run_cuda(args, rank, world, local_rank):
    import numpy as np
    import torch
    import newton_schulz_hyperball_b200 as nshb

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    shp = shapes()
    W0, Gh = build_inputs(dev, rank)
    W = [torch.from_numpy(w).to(dev).to(torch.bfloat16) for w in W0]
    Gd = [[torch.from_numpy(g).to(dev).to(torch.bfloat16) for g in gs] for gs in Gh]
    M = [torch.zeros(w.shape, dtype=torch.float32, device=dev) for w in W]
    rho = torch.tensor([float(np.linalg.norm(w.astype(np.float64))) for w in W0], dtype=torch.float32, device=dev)
    p = nshb.params(eta=ETA, rho=rho)
    mats = [nshb.matrices(W, Gd[s], M) for s in range(N_GRAD_SETS)]
    ws = nshb.workspace(mats[0], p, nshb.NSHB_OP_HYPERBALL, device=dev)
    n_params = sum(r * c for r, c in shp)

    def step(k):
        nshb.hyperball_step(mats[k % N_GRAD_SETS], p, ws, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(x):
        if world == 1:
            return x
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    # warm-up
    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    flags = nshb.device_status(ws, stream)
    if args.ncu:
        # profiling case: exactly `steps` more steps, nothing else
        for k in range(args.steps):
            step(args.warmup + k)
        torch.cuda.synchronize()
        return None

    # ---- timed region: device-resident inputs
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for k in range(args.steps):
            step(k)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1)) / args.steps

    # ---- per-kernel times (same step, events around each launch)
    nshb.profile_enable(True)
    nshb.profile_read()
    kp = max(10, min(args.steps, 50))
    for k in range(kp):
        step(k)
    torch.cuda.synchronize()
    prof = nshb.profile_read()
    nshb.profile_enable(False)
    launches_per_step = sum(c for _, c in prof.values()) / kp

    # ---- end to end through the public API with host buffers (see timed_e2e)
    def e2e_step(m, k):
        nshb.hyperball_step(m, p, ws, stream)

    ke = max(5, min(args.steps, 30))
    barrier()
    e2e_one, h2d = timed_e2e(Gh, W, M, e2e_step, ws, stream, ke, nshb, torch)
    barrier()
    e2e_ms = max_over_ranks(e2e_one)

    return dict(ms=ms, prof=prof, kp=kp, launches_per_step=launches_per_step, flags=flags,
                clocks=clk.summary(), e2e_ms=e2e_ms, h2d=h2d, d2h=4, n_params=n_params, shp=shp)


# ---------------------------------------------------------------------- AdamH
def run_adamh(args, rank, world, local_rank):
    """AdamH step (Adam moments + Hyperball) on the same matrix set: timed like run_cuda."""
    import numpy as np
    import torch
    import newton_schulz_hyperball_b200 as nshb

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    shp = shapes()
    W0, Gh = build_inputs(dev, rank)
    W = [torch.from_numpy(w).to(dev).to(torch.bfloat16) for w in W0]
    Gd = [[torch.from_numpy(g).to(dev).to(torch.bfloat16) for g in gs] for gs in Gh]
    M = [torch.zeros(w.shape, dtype=torch.float32, device=dev) for w in W]
    V = [torch.zeros(w.shape, dtype=torch.float32, device=dev) for w in W]
    rho = torch.tensor([float(np.linalg.norm(w.astype(np.float64))) for w in W0], dtype=torch.float32, device=dev)
    p = nshb.params(eta=ETA, rho=rho)
    mats = [nshb.matrices(W, Gd[s], M) for s in range(N_GRAD_SETS)]
    ws = nshb.workspace(mats[0], p, nshb.NSHB_OP_ADAMH, device=dev)
    n_params = sum(r * c for r, c in shp)
    count = [0]

    def step(k, m=None):
        count[0] += 1
        nshb.adamh_step(m if m is not None else mats[k % N_GRAD_SETS], V, nshb.adam_params(step=count[0]), p, ws,
                        stream)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    flags = nshb.device_status(ws, stream)
    if args.ncu:
        for k in range(args.steps):
            step(args.warmup + k)
        torch.cuda.synchronize()
        return None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for k in range(args.steps):
            step(k)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    nshb.profile_enable(True)
    nshb.profile_read()
    kp = max(10, min(args.steps, 50))
    for k in range(kp):
        step(k)
    torch.cuda.synchronize()
    prof = nshb.profile_read()
    nshb.profile_enable(False)
    launches_per_step = sum(c for _, c in prof.values()) / kp
    def e2e_step(m, k):
        step(k, m)

    ke = max(5, min(args.steps, 30))
    e2e_ms, h2d = timed_e2e(Gh, W, M, e2e_step, ws, stream, ke, nshb, torch)
    return dict(ms=ms, prof=prof, kp=kp, launches_per_step=launches_per_step, flags=flags,
                clocks=clk.summary(), e2e_ms=e2e_ms, h2d=h2d, d2h=4, n_params=n_params, shp=shp)


def oracle_adamh_sample(layers=12, steps=5):
    """Times the oracle's AdamH step on `layers` GPT-2 layers for `steps` steps and returns
    (seconds per full 72-matrix step, extrapolated by element count when layers < 12,
    sample description)."""
    import numpy as np
    from newton_schulz_hyperball_b200 import workloads as wl
    from oracle import nshb_oracle as o
    cfg = wl.CFG_GPT2_SMALL
    shp = shapes()
    idx = list(range(6 * layers))
    Ws = {i: wl.init_weight(cfg, i, *shp[i], bf16=True).astype(np.float64) for i in idx}
    Ms = {i: np.zeros(shp[i]) for i in idx}
    Vs = {i: np.zeros(shp[i]) for i in idx}
    rho = {i: o.fro(Ws[i]) for i in idx}
    Gs = [{i: wl.gradient(cfg, i, s, *shp[i], bf16=True).astype(np.float64) for i in idx} for s in range(steps)]
    t0 = time.perf_counter()
    for s in range(steps):
        for i in idx:
            Ws[i], Ms[i], Vs[i], _, _ = o.adamh_step(Ws[i], Gs[s][i], Ms[i], Vs[i], t=s + 1, eta=ETA, rho=rho[i])
    timed = time.perf_counter() - t0
    n_all = sum(r * c for r, c in shp)
    n_s = sum(shp[i][0] * shp[i][1] for i in idx)
    return timed / steps * n_all / n_s, sample_desc(len(idx), layers, steps, timed, "element count")


def sample_desc(n_mats, layers, steps, timed, scale_by):
    what = f"{n_mats} of 72 matrices (GPT-2 layers 0..{layers - 1}), {steps} step(s), {timed:.1f} s timed"
    return what if n_mats == 72 else what + f", extrapolated to 72 matrices by {scale_by}"


def report_adamh(args, r, world):
    peaks, peak_src = load_peaks()
    prof, kp, n = r["prof"], r["kp"], r["n_params"]
    adam_ms = prof.get("adam", (0.0, 0))[0] / kp
    apply_ms = prof.get("apply", (0.0, 0))[0] / kp
    peak_bw = peaks.get("hbm_gbs", DEFAULT_PEAKS["hbm_gbs"])
    # Algorithmic HBM bytes: adam 22 B/elem (G 2, M 4+4, V 4+4, W 2, U~ 2), apply 6 (W 2+2, U~ 2).
    adam_gbs = 22.0 * n / (adam_ms * 1e-3) / 1e9 if adam_ms > 0 else None
    fused_gbs = 28.0 * n / ((adam_ms + apply_ms) * 1e-3) / 1e9 if adam_ms + apply_ms > 0 else None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        with OracleThreads() as th:
            full, desc = oracle_adamh_sample()
        cpu = {"value": round(full * 1e3, 3), "unit": "ms", "cores": th.cores, "affinity_cores": th.affinity,
               "kind": "oracle", "sample": desc}
    return {
        "metric": "AdamH optimizer step ms; fused HBM GB/s",
        "value": round(r["ms"], 4), "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(r["ms"], 4), "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 (bf16 storage)",
        "data": "synthetic (seeded W0 ~ N(0, 0.02^2), spiked Gaussian gradients; no dataset)",
        "config": {"workload": "gpt2-small matrix set, AdamH step (72 bf16 matrices, fp32 moments, Hyperball)",
                   "matrices": len(r["shp"]), "params": n,
                   "optimizer": "AdamH (0.9, 0.999, 1e-8, eta 0.02, rho = ||W0||)",
                   "l2": "inputs larger than L2 (W+G+M+V = 1.02 GB per step)", "parallelism": f"replica per GPU x{world}"},
        "throughput": {"value": round(world * n / (r["ms"] * 1e-3), 1), "unit": "params/s"},
        "fused_gbs": None if fused_gbs is None else round(fused_gbs, 1),
        "roofline": {"bound": "hbm", "kernel": "adam_kernel (moments, U~, partials)",
                     "achieved": None if adam_gbs is None else round(adam_gbs, 1), "peak": peak_bw, "unit": "GB/s",
                     "frac": None if adam_gbs is None else round(adam_gbs / peak_bw, 4),
                     "traffic": source_traffic(STREAM_SOURCE, ADAM_TRAFFIC),
                     "peak_source": f"{peak_src} copy bandwidth"},
        "kernels_ms_per_step": {k: round(v[0] / kp, 5) for k, v in prof.items()},
        "gpu_launches": int(round(r["launches_per_step"] * args.steps)),
        "device_status": r["flags"], "clocks": r["clocks"],
        "e2e": {"value": round(r["e2e_ms"], 4), "unit": "ms", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"], "pipeline": E2E_PIPELINE},
        "cpu_baseline": cpu,
    }


# ------------------------------------------------------------ other configurations
CONFIGS = {
    "qwen3": "Qwen3-style 1.4B matrix set (196 matrices), MuonH step",
    "himuon8b": "8B-width matrix set (224 matrices, 6.98B params), Hierarchical Muon + Hyperball step",
    "newton": "GPT-2-small matrix set, Newton-Muon step (48 layer inputs of 8192 tokens) + Hyperball",
}


def device_set(shapes, cfg, dev, torch):
    """W ~ N(0, 0.02^2) and G = sigma (E + (10/sqrt 8) A B^T) drawn on the device with a seeded
    generator (sigma per matrix from the host recipe); bf16."""
    from newton_schulz_hyperball_b200 import workloads as wl
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + cfg)
    W, G = [], []
    for i, (r, c) in enumerate(shapes):
        W.append((0.02 * torch.randn(r, c, device=dev, generator=g)).to(torch.bfloat16))
        a = torch.randn(r, 8, device=dev, generator=g)
        b = torch.randn(c, 8, device=dev, generator=g)
        e = torch.randn(r, c, device=dev, generator=g)
        G.append((wl.grad_sigma(cfg, i) * (e + (10 / 8 ** 0.5) * (a @ b.T))).to(torch.bfloat16))
        del a, b, e
    return W, G


def run_config(args):
    """One of the larger configurations: step ms and algorithmic tensor-core TFLOP/s (1 GPU)."""
    import numpy as np
    import torch
    import newton_schulz_hyperball_b200 as nshb
    from newton_schulz_hyperball_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    Z = None
    if args.config == "qwen3":
        cfg = wl.CFG_QWEN3_1B
        named = wl.qwen3_1b_shapes(28)
        shp = [(r, c) for _, r, c in named]
        op, fn, flops = nshb.NSHB_OP_HYPERBALL, "hyperball_step", ns_flops(shp)
        extra = {}
    elif args.config == "himuon8b":
        cfg = wl.CFG_8B_WIDTH
        named = wl.width_8b_shapes(args.layers)
        shp = [(r, c) for _, r, c in named]
        T = args.tile
        op, fn, flops = nshb.NSHB_OP_HIMUON, "himuon_step", sum(20.0 * r * c * T for r, c in shp)
        extra = {"tile": T}
    else:
        cfg = wl.CFG_NEWTON_GPT2
        named = wl.gpt2_small_shapes(12)
        shp = [(r, c) for _, r, c in named]
        zi, zrows = wl.newton_gpt2_z_index(named)
        n_tok = 8192
        g = torch.Generator(device=dev)
        g.manual_seed(2000 + cfg)
        Z = []
        for d in zrows:     # Z = diag(e^u) E, u ~ U(ln 0.1, ln 10), E ~ N(0, 1)
            u = torch.empty(d, 1, device=dev).uniform_(float(np.log(0.1)), float(np.log(10.0)), generator=g)
            Z.append((torch.exp(u) * torch.randn(d, n_tok, device=dev, generator=g)).to(torch.bfloat16))
        syrk = sum(float(d) * d * n_tok for d in zrows)   # Z Z^T, symmetric half
        op, fn, flops = nshb.NSHB_OP_NEWTON_MUON, "newton_muon_step", ns_flops(shp) + syrk
        extra = {"z_inputs": len(zrows), "tokens": n_tok, "syrk_tflop": round(syrk / 1e12, 3)}
    W, G = device_set(shp, cfg, dev, torch)
    M = [torch.zeros(w.shape, dtype=torch.float32, device=dev) for w in W]
    rho = torch.stack([w.float().norm() for w in W])
    mats = nshb.matrices(W, G, M, z_index=(zi if Z is not None else None))
    p = nshb.params(eta=ETA, rho=rho, **extra_params(extra))
    if Z is not None:
        ws = nshb.workspace(mats, p, op, device=dev, z_rows=[z.shape[0] for z in Z], n_tokens=n_tok)
        step = lambda: nshb.newton_muon_step(mats, Z, n_tok, p, ws, stream)   # noqa: E731
    else:
        ws = nshb.workspace(mats, p, op, device=dev)
        step = lambda: getattr(nshb, fn)(mats, p, ws, stream)   # noqa: E731
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flags = nshb.device_status(ws, stream)
    if args.ncu:
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
        return None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    nshb.profile_enable(True)
    nshb.profile_read()
    kp = 3
    for _ in range(kp):
        step()
    torch.cuda.synchronize()
    prof = nshb.profile_read()
    nshb.profile_enable(False)
    peaks, peak_src = load_peaks()
    peak_tf = peaks.get("bf16_tflops_sustained", DEFAULT_PEAKS["bf16_tflops_sustained"])
    n = sum(r * c for r, c in shp)
    tf = flops / (ms * 1e-3) / 1e12
    return {
        "metric": "optimizer step ms; algorithmic tensor-core TFLOP/s over the whole step",
        "value": round(ms, 3), "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded on the device: W0 ~ N(0, 0.02^2), spiked Gaussian gradients)",
        "config": {"workload": CONFIGS[args.config], "matrices": len(shp), "params": n, **extra,
                   **({"layers": args.layers} if args.config == "himuon8b" else {})},
        "throughput": {"value": round(n / (ms * 1e-3), 1), "unit": "params/s"},
        "step_tflops": round(tf, 1),
        "step_tflops_frac_of_sustained_bf16_peak": round(tf / peak_tf, 4),
        "algorithmic_tflop_per_step": round(flops / 1e12, 3),
        "peak_source": f"{peak_src} bf16 sustained",
        "kernels_ms_per_step": {k: round(v[0] / kp, 4) for k, v in prof.items()},
        "launches_per_step": {k: round(v[1] / kp, 1) for k, v in prof.items()},
        "device_status": flags, "clocks": clk.summary(),
    }


def extra_params(extra):
    return {"tile": extra["tile"]} if "tile" in extra else {}


# --------------------------------------------------------------- CPU baseline
def oracle_sample(layers=12, steps=2):
    """Times the fp64 oracle on `layers` of the 12 GPT-2 layers for `steps` steps and returns
    (seconds per full 72-matrix step extrapolated by NS flops, sample description)."""
    import numpy as np
    from newton_schulz_hyperball_b200 import workloads as wl
    from oracle import nshb_oracle as o
    cfg = wl.CFG_GPT2_SMALL
    shp = shapes()
    idx = list(range(6 * layers))
    Ws = {i: wl.init_weight(cfg, i, *shp[i], bf16=True).astype(np.float64) for i in idx}
    Ms = {i: np.zeros(shp[i]) for i in idx}
    rho = {i: o.fro(Ws[i]) for i in idx}
    Gs = [{i: wl.gradient(cfg, i, s, *shp[i], bf16=True).astype(np.float64) for i in idx} for s in range(steps)]
    t0 = time.perf_counter()
    for s in range(steps):
        for i in idx:
            Ws[i], Ms[i], _, _ = o.hyperball_step(Ws[i], Gs[s][i], Ms[i], eta=ETA, rho=rho[i])
    timed = time.perf_counter() - t0
    full = timed / steps * ns_flops(shp) / ns_flops([shp[i] for i in idx])
    return full, sample_desc(len(idx), layers, steps, timed, "NS flops")


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class OracleThreads:
    """Lets the oracle's BLAS use every core this process may run on (torchrun starts its
    workers with OMP_NUM_THREADS=1) and records the thread count in effect, which is what
    `cores` reports."""

    def __enter__(self):
        import numpy  # noqa: F401  (threadpoolctl sees only BLAS libraries already loaded)
        from threadpoolctl import threadpool_info, threadpool_limits
        self._lim = threadpool_limits(limits=cpu_cores(), user_api="blas")
        self._lim.__enter__()
        self.cores = max([d["num_threads"] for d in threadpool_info() if d["user_api"] == "blas"] or [1])
        self.affinity = cpu_cores()
        return self

    def __exit__(self, *exc):
        return self._lim.__exit__(*exc)


def run_reference(args, rank, world):
    """The oracle on the host cores, on this workload (bounded sample per step)."""
    if rank != 0:
        return None
    times = []
    desc = None
    with OracleThreads() as th:
        for _ in range(args.warmup):
            oracle_sample(1, 1)
        for _ in range(args.steps):
            full, desc = oracle_sample(1, 1)
            times.append(full)
    ms = 1e3 * statistics.median(times)
    return dict(ms=ms, desc=desc, cores=th.cores, affinity=th.affinity)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config", default="gpt2", choices=["gpt2"] + sorted(CONFIGS),
                    help="gpt2: the headline workload; the others time one larger configuration (1 GPU)")
    ap.add_argument("--tile", type=int, default=256, choices=[128, 256, 512], help="--config himuon8b: tile size T")
    ap.add_argument("--layers", type=int, default=32, help="--config himuon8b: layers of the 8B-width set")
    ap.add_argument("--optimizer", default="muonh", choices=["muonh", "adamh"],
                    help="muonh: the headline MuonH step; adamh: the AdamH step on the same matrices")
    ap.add_argument("--ncu", action="store_true",
                    help="profiling case: warm-up and `steps` steps only, no timing or report")
    args = ap.parse_args()
    if args.warmup < 3 and not args.ncu:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if world > 1 and rank != 0:
            return 0
        steps = min(args.steps, 20)
        args.steps = steps
        args.warmup = min(args.warmup, 3)
        r = run_reference(args, rank, world)
        line = {"metric": METRIC, "value": round(r["ms"], 3), "unit": "ms", "n_gpus": args.gpus, "steps": steps,
                "warmup": args.warmup, "ms_per_step": round(r["ms"], 3), "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference",
                "config": {"workload": WORKLOAD, "matrices": 72, "params": 84934656},
                "cpu_baseline": {"value": round(r["ms"], 3), "unit": "ms", "cores": r["cores"],
                                 "affinity_cores": r["affinity"], "kind": "oracle",
                                 "sample": r["desc"]},
                "e2e": {"value": round(r["ms"], 3), "unit": "ms", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))

    if args.config != "gpt2":
        if world > 1:
            print("--config runs on one GPU", file=sys.stderr)
            return 2
        r = run_config(args)
        print("ncu case done" if r is None else json.dumps(r), flush=True)
        return 0
    if args.optimizer == "adamh":
        if world > 1:
            print("--optimizer adamh runs on one GPU", file=sys.stderr)
            return 2
        r = run_adamh(args, rank, world, local_rank)
        if r is None:
            print("ncu case done", flush=True)
            return 0
        print(json.dumps(report_adamh(args, r, world)), flush=True)
        return 0
    r = run_cuda(args, rank, world, local_rank)
    if r is None:
        print("ncu case done", flush=True)
        return 0
    peaks, peak_src = load_peaks()
    shp = r["shp"]
    flops = ns_flops(shp)
    prof = r["prof"]
    kp = r["kp"]
    gemm_ms = sum(prof.get(k, (0.0, 0))[0] for k in ("gram", "poly", "update")) / kp
    gemm_launches = sum(prof.get(k, (0.0, 0))[1] for k in ("gram", "poly", "update")) / kp
    ns_tflops = flops / (gemm_ms * 1e-3) / 1e12 if gemm_ms > 0 else None
    n = r["n_params"]
    # Algorithmic HBM bytes of the fused streaming kernels: momentum 12 B/elem
    # (G 2 + M 4 + 4 + U 2), apply 6 B/elem (W 2 + 2, O 2).
    mom_ms = prof.get("momentum", (0.0, 0))[0] / kp
    apply_ms = prof.get("apply", (0.0, 0))[0] / kp
    red_ms = prof.get("reduce", (0.0, 0))[0] / kp
    fused_bytes = 18.0 * n
    fused_ms = mom_ms + apply_ms + red_ms
    fused_gbs = fused_bytes / (fused_ms * 1e-3) / 1e9 if fused_ms > 0 else None
    mom_gbs = 12.0 * n / (mom_ms * 1e-3) / 1e9 if mom_ms > 0 else None
    peak_tf = peaks.get("bf16_tflops", DEFAULT_PEAKS["bf16_tflops"])
    peak_bw = peaks.get("hbm_gbs", DEFAULT_PEAKS["hbm_gbs"])
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with OracleThreads() as th:
            full, desc = oracle_sample()
        cpu = {"value": round(full * 1e3, 3), "unit": "ms", "cores": th.cores, "affinity_cores": th.affinity,
               "kind": "oracle", "sample": desc}
    if rank != 0:
        return 0
    line = {
        "metric": METRIC,
        "value": round(r["ms"], 4),
        "unit": "ms",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(r["ms"], 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded W0 ~ N(0, 0.02^2), spiked Gaussian gradients; no dataset)",
        "config": {"workload": WORKLOAD, "matrices": len(shp), "params": n, "ns_steps": 5,
                   "optimizer": "MuonH (Nesterov 0.95, eta 0.02, rho = ||W0||)",
                   "l2": "inputs larger than L2 (W+G+M = 680 MB per step, 4 rotating gradient sets)",
                   "parallelism": f"replica per GPU x{world}"},
        "throughput": {"value": round(world * n / (r["ms"] * 1e-3), 1), "unit": "params/s"},
        "ns_tflops": None if ns_tflops is None else round(ns_tflops, 1),
        "ns_frac_of_bf16_peak": None if ns_tflops is None else round(ns_tflops / peak_tf, 4),
        "ns_tflops_dense_equiv": None if gemm_ms <= 0 else round(ns_flops(shp, dense=True) / (gemm_ms * 1e-3) / 1e12, 1),
        "fused_gbs": None if fused_gbs is None else round(fused_gbs, 1),
        "fused_frac_of_hbm": None if fused_gbs is None else round(fused_gbs / peak_bw, 4),
        "roofline": {"bound": "tensor", "kernel": "gemm_tc2_kernel (NS Gram / polynomial / update, CTA pairs)",
                     "achieved": None if ns_tflops is None else round(ns_tflops, 1),
                     "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": None if ns_tflops is None else round(ns_tflops / peak_tf, 4),
                     "frac_of_sustained": None if ns_tflops is None else round(
                         ns_tflops / peaks.get("bf16_tflops_sustained", DEFAULT_PEAKS["bf16_tflops_sustained"]), 4),
                     "traffic": gemm_traffic(),
                     "peak_source": f"{peak_src} bf16 burst (sustained {peaks.get('bf16_tflops_sustained')})",
                     "flops_per_launch": round(flops / max(gemm_launches, 1)),
                     "per_launch_ms": round(gemm_ms / max(gemm_launches, 1), 5)},
        "kernels_ms_per_step": {k: round(v[0] / kp, 5) for k, v in prof.items()},
        "momentum_gbs": None if mom_gbs is None else round(mom_gbs, 1),
        "gpu_launches": int(round(r["launches_per_step"] * args.steps)),
        "device_status": r["flags"],
        "clocks": r["clocks"],
        "e2e": {"value": round(r["e2e_ms"], 4), "unit": "ms", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"], "pipeline": E2E_PIPELINE},
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def run():
    """main(), then every rank releases its process group, whichever way main returned."""
    try:
        return main()
    finally:
        if "torch.distributed" in sys.modules:
            import torch.distributed as dist
            if dist.is_available() and dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(run())
