"""Benchmark of the Muon-Hyperball optimizer step on B200.

Default workload (one step = the whole hot path over one batch of synthetic input): the
Qwen3-style ~1.2B matrix set -- 28 layers x {Wq 2048x2048, Wk/Wv 1024x2048, Wo 2048x2048,
gate/up 6144x2048, down 2048x6144}, 196 matrices, 1,409,286,144 parameters -- with bf16
weights and gradients, fp32 momentum, Nesterov beta = 0.95, K = 5 quintic Newton-Schulz
iterations on the tensor cores (all 196 matrices in the same launches) and the Hyperball
rule with rho = ||W0||_F per matrix and eta = 0.02.  Gradients are seeded N(0, sigma^2)
noise plus a rank-8 spike of RMS 10 sigma, sigma log-uniform in [1e-4, 1e-2] per matrix,
drawn on the device; two gradient sets rotate.  W + G + M is 11 GB per step, far larger
than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--config qwen3|qwen3-brake|gpt2|gpt2-adamh|himuon8b|newton]

Other configurations: `gpt2` (GPT-2-small set, 72 matrices), `qwen3-brake` (the same
Qwen3-style set with the RadialBrake hook), `gpt2-adamh` (AdamH on the GPT-2 set),
`himuon8b` (Hierarchical Muon on the 8B-width set, --tile T), `newton` (Newton-Muon on the
GPT-2 set with 48 layer inputs of 8192 tokens).  Each prints the same line.

One JSON line is printed by rank 0.  Under torchrun (N > 1) every rank runs its own replica
of the matrix set on its own GPU (weak scaling, no collective on the data path); the time is
the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time
from dataclasses import dataclass, field

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Muon-H optimizer step ms; NS TFLOP/s (% bf16 peak); fused-kernel HBM GB/s"
ETA = 0.02
DEFAULT_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
E2E_PIPELINE = "H2D of step k+1 on a second stream during step k (2 device buffers)"

# DRAM read + write per launch of a kernel from an ncu capture, valid only for the kernel
# source it was taken on (keyed by a hash prefix of that source file).  `scale` turns the
# captured case into one launch of the benchmarked set (units processed), and `case`
# says what was captured.
CSRC = os.path.join(ROOT, "newton_schulz_hyperball_b200", "csrc")
TRAFFIC = {
    "gemm_qwen3": {"source": "ns_tc2.cu", "sha256_prefix": "04b0c7ee8b4b7441", "bytes_per_launch": 4470472531,
                   "case": "4 of the 28 Qwen3-style layers (28 matrices), one step's 15 launches: 9.58 GB "
                           "DRAM read + write, 0.639 GB per launch, x7 for the 28 identical layers"},
    "gemm_gpt2": {"source": "ns_tc2.cu", "sha256_prefix": "04b0c7ee8b4b7441", "bytes_per_launch": 260381952,
                  "case": "GPT-2-small set, 15 launches of one step averaged"},
    "adam_gpt2": {"source": "stream_kernels.cu", "sha256_prefix": "d01621941b46621c",
                  "bytes_per_launch": 1814333696, "case": "GPT-2-small set, one launch"},
}


def source_hash(name):
    import hashlib
    try:
        with open(os.path.join(CSRC, name), "rb") as f:
            return hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None


def traffic_for(key):
    rec = TRAFFIC.get(key)
    if rec is None:
        return None
    return rec["bytes_per_launch"] if source_hash(rec["source"]) == rec["sha256_prefix"] else None


# --------------------------------------------------------------------- workloads
@dataclass
class Workload:
    key: str
    desc: str                 # config.workload
    cfg: int                  # seed configuration id (workloads.CFG_*)
    named: list               # (name, rows, cols)
    step: str                 # hyperball | brake | himuon | newton | adamh
    draw: str                 # host | device: where the seeded inputs are drawn
    n_grad_sets: int
    metric: str = METRIC
    tile: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def shapes(self):
        return [(r, c) for _, r, c in self.named]

    @property
    def n_params(self):
        return sum(r * c for r, c in self.shapes)


def make_workload(args) -> Workload:
    from newton_schulz_hyperball_b200 import workloads as wl
    c = args.config
    if c in ("qwen3", "qwen3-brake"):
        named = wl.qwen3_1b_shapes(args.layers or 28)
        hook = "brake" if c == "qwen3-brake" else "hyperball"
        what = ("MuonH step (Hyperball, eta 0.02, rho = ||W0||)" if hook == "hyperball"
                else "Muon + RadialBrake step (lr 0.02, outward 0.5, inward 1.0)")
        return Workload(c, f"Qwen3-style ~1.2B matrix set ({len(named)} matrices of {len(named) // 7} layers: "
                           f"Wq/Wo 2048x2048, Wk/Wv 1024x2048, gate/up 6144x2048, down 2048x6144), {what}",
                        wl.CFG_QWEN3_1B, named, hook, "device", 2)
    if c == "gpt2":
        named = wl.gpt2_small_shapes(args.layers or 12)
        return Workload(c, f"GPT-2-small matrix set ({len(named)} matrices: Wq/Wk/Wv/Wo 768x768, W_fc 3072x768, "
                           "W_proj 768x3072), MuonH step (Hyperball, eta 0.02, rho = ||W0||)",
                        wl.CFG_GPT2_SMALL, named, "hyperball", "host", 4)
    if c == "gpt2-adamh":
        named = wl.gpt2_small_shapes(args.layers or 12)
        return Workload(c, f"GPT-2-small matrix set ({len(named)} matrices), AdamH step (Adam 0.9/0.999/1e-8 "
                           "moments in fp32, Hyperball eta 0.02, rho = ||W0||)",
                        wl.CFG_GPT2_SMALL, named, "adamh", "host", 4, metric="AdamH optimizer step ms; fused HBM GB/s")
    if c == "himuon8b":
        named = wl.width_8b_shapes(args.layers or 32)
        return Workload(c, f"8B-width matrix set ({len(named)} matrices: 4096x4096 x2, 1024x4096 x2, "
                           f"14336x4096 x2, 4096x14336 per layer), Hierarchical Muon T={args.tile} + Hyperball step",
                        wl.CFG_8B_WIDTH, named, "himuon", "device", 1, tile=args.tile,
                        metric="HiMuon-H optimizer step ms; tiled NS TFLOP/s (% bf16 peak)")
    if c == "newton":
        named = wl.gpt2_small_shapes(args.layers or 12)
        zi, zrows = wl.newton_gpt2_z_index(named)
        return Workload(c, f"GPT-2-small matrix set ({len(named)} matrices), Newton-Muon step with {len(zrows)} "
                           "layer inputs Z of 8192 tokens (ridge 1e-3 tr(ZZ^T)/d_in) + Hyperball",
                        wl.CFG_NEWTON_GPT2, named, "newton", "device", 1,
                        metric="Newton-Muon-H optimizer step ms; tensor-core TFLOP/s (% bf16 peak)",
                        extra={"z_index": zi, "z_rows": zrows, "n_tokens": 8192})
    raise ValueError(c)


def ns_flops(shp, K=5, dense=False):
    """Algorithmic NS work per step: K (3 r^2 s + r^3), symmetric products counted once;
    dense=True gives the dense-equivalent K (4 r^2 s + 2 r^3) of the full products."""
    tot = 0.0
    for r, c in shp:
        rr, ss = min(r, c), max(r, c)
        tot += K * ((4.0 * rr * rr * ss + 2.0 * rr ** 3) if dense else (3.0 * rr * rr * ss + rr ** 3))
    return tot


def himuon_flops(shp, T, K=5):
    """Tiled NS work: K (3 T^3 + T^3) per T x T tile, i.e. 4 K T H W = 20 H W T at K = 5."""
    return sum(4.0 * K * r * c * T for r, c in shp)


def syrk_flops(zrows, n_tok):
    """Z Z^T with the symmetric half counted once: d^2 n per layer input."""
    return sum(float(d) * d * n_tok for d in zrows)


def solve_flops(shp):
    """The two triangular solves of P = U L^-T L^-1 (m x d right-hand sides): 2 m d^2."""
    return sum(2.0 * r * c * c for r, c in shp)


def potrf_flops(zrows):
    return sum(d ** 3 / 3.0 for d in zrows)


def work_flops(w: Workload):
    """Algorithmic tensor-core work of one step (what the roofline's kernel computes)."""
    if w.step == "himuon":
        return himuon_flops(w.shapes, w.tile)
    if w.step == "newton":
        return ns_flops(w.shapes) + syrk_flops(w.extra["z_rows"], w.extra["n_tokens"])
    if w.step == "adamh":
        return 0.0
    return ns_flops(w.shapes)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(DEFAULT_PEAKS), "fallback"


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every 5 ms while the timed region
    runs."""

    PERIOD_S = 0.005

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
            time.sleep(self.PERIOD_S)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        med = statistics.median(self.samples) if self.ok and self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "period_ms": self.PERIOD_S * 1e3}


# ------------------------------------------------------------------ inputs
def host_set(w: Workload, n_sets: int):
    """Seeded host inputs (bf16 values in float32 arrays): W0 and n_sets gradient sets."""
    from newton_schulz_hyperball_b200 import workloads as wl
    W0 = [wl.init_weight(w.cfg, i, r, c, bf16=True) for i, (r, c) in enumerate(w.shapes)]
    G = [[wl.gradient(w.cfg, i, s, r, c, bf16=True) for i, (r, c) in enumerate(w.shapes)] for s in range(n_sets)]
    return W0, G


def device_set(w: Workload, dev, torch, n_sets: int):
    """W ~ N(0, 0.02^2) and n_sets gradient sets G = sigma (E + (10/sqrt 8) A B^T) drawn on
    the device with a seeded generator (sigma per matrix from the host recipe); bf16.  The
    spike factors A, B are fixed per matrix, E is fresh in every set."""
    from newton_schulz_hyperball_b200 import workloads as wl
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + w.cfg)
    W = [(0.02 * torch.randn(r, c, device=dev, generator=g)).to(torch.bfloat16) for r, c in w.shapes]
    G = [[] for _ in range(n_sets)]
    for i, (r, c) in enumerate(w.shapes):
        a = torch.randn(r, 8, device=dev, generator=g)
        b = torch.randn(c, 8, device=dev, generator=g)
        spike = (10 / 8 ** 0.5) * (a @ b.T)
        for s in range(n_sets):
            e = torch.randn(r, c, device=dev, generator=g)
            G[s].append((wl.grad_sigma(w.cfg, i) * (e + spike)).to(torch.bfloat16))
            del e
        del a, b, spike
    return W, G


def device_layer_inputs(w: Workload, dev, torch):
    """Z = diag(e^u) E (u ~ U(ln 0.1, ln 10), E ~ N(0, 1)), d_in x n_tokens, bf16, on the device."""
    import math
    g = torch.Generator(device=dev)
    g.manual_seed(2000 + w.cfg)
    Z = []
    for d in w.extra["z_rows"]:
        u = torch.empty(d, 1, device=dev).uniform_(math.log(0.1), math.log(10.0), generator=g)
        Z.append((torch.exp(u) * torch.randn(d, w.extra["n_tokens"], device=dev, generator=g)).to(torch.bfloat16))
    return Z


# ------------------------------------------------------------------ the GPU arm
class Stepper:
    """The step call of a workload through the library's public API."""

    def __init__(self, w: Workload, W, M, rho, dev, torch, nshb, Z=None):
        self.w, self.nshb, self.torch = w, nshb, torch
        self.W, self.M, self.Z = W, M, Z
        self.count = 0
        kw = {"eta": ETA, "rho": rho}
        if w.step == "himuon":
            kw["tile"] = w.tile
        if w.step == "brake":
            kw = {"lr": 0.02, "brake_out": 0.5, "brake_in": 1.0}
        if w.step == "newton":
            kw["ridge_rel"] = 1e-3
        self.p = nshb.params(**kw)
        self.V = [torch.zeros(x.shape, dtype=torch.float32, device=dev) for x in W] if w.step == "adamh" else None
        self.op = {"hyperball": nshb.NSHB_OP_HYPERBALL, "brake": nshb.NSHB_OP_RADIAL_BRAKE,
                   "himuon": nshb.NSHB_OP_HIMUON, "newton": nshb.NSHB_OP_NEWTON_MUON,
                   "adamh": nshb.NSHB_OP_ADAMH}[w.step]
        self.zi = w.extra.get("z_index")

    def mats(self, G):
        return self.nshb.matrices(self.W, G, self.M, z_index=self.zi)

    def workspace(self, mats, dev):
        if self.w.step == "newton":
            return self.nshb.workspace(mats, self.p, self.op, device=dev, z_rows=self.w.extra["z_rows"],
                                       n_tokens=self.w.extra["n_tokens"])
        return self.nshb.workspace(mats, self.p, self.op, device=dev)

    def __call__(self, mats, ws, stream, Z=None):
        nshb, s = self.nshb, self.w.step
        if s == "hyperball":
            nshb.hyperball_step(mats, self.p, ws, stream)
        elif s == "brake":
            nshb.radial_brake_step(mats, self.p, ws, stream)
        elif s == "himuon":
            nshb.himuon_step(mats, self.p, ws, stream)
        elif s == "newton":
            nshb.newton_muon_step(mats, self.Z if Z is None else Z, self.w.extra["n_tokens"], self.p, ws, stream)
        else:
            self.count += 1
            nshb.adamh_step(mats, self.V, nshb.adam_params(step=self.count), self.p, ws, stream)


def timed_e2e(Gh, stepper, ws, stream, ke, torch, dev, Zh=None):
    """End to end through the public API with host buffers: every step's gradients (and, for
    Newton-Muon, its layer inputs Z) are copied host->device from pinned memory and the step's
    device status word is read back.  The copy of step k+1 runs on a second stream while step
    k computes (two device buffers, events in both directions), as an input pipeline would;
    all copies lie inside the timed region.
    Gh: list of pinned host gradient sets (used in turn); Zh: pinned host layer inputs."""
    bufs = [[torch.empty(g.shape, dtype=g.dtype, device=dev) for g in Gh[0]] for _ in range(2)]
    zbufs = [[torch.empty(z.shape, dtype=z.dtype, device=dev) for z in Zh] for _ in range(2)] if Zh else None
    mats_b = [stepper.mats(bufs[j]) for j in range(2)]
    st_host = torch.empty(1, dtype=torch.int32).pin_memory()
    h2d = sum(g.numel() * g.element_size() for g in Gh[0])
    if Zh:
        h2d += sum(z.numel() * z.element_size() for z in Zh)
    copy_stream = torch.cuda.Stream(device=dev)
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
            for d, s_ in zip(bufs[j], Gh[k % len(Gh)]):
                d.copy_(s_, non_blocking=True)
            if zbufs:
                for d, s_ in zip(zbufs[j], Zh):
                    d.copy_(s_, non_blocking=True)
            copied[j].record(copy_stream)

    issue_copy(0)
    for k in range(ke):
        if k + 1 < ke:
            issue_copy(k + 1)
        j = k % 2
        stream.wait_event(copied[j])
        stepper(mats_b[j], ws, stream, Z=zbufs[j] if zbufs else None)
        consumed[j].record(stream)
        st_host.copy_(ws[:4].view(torch.int32), non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / ke
    del bufs, zbufs, mats_b
    return ms, h2d


def run_cuda(args, rank, world, local_rank, w: Workload):
    import numpy as np
    import torch
    import newton_schulz_hyperball_b200 as nshb

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    Z = device_layer_inputs(w, dev, torch) if w.step == "newton" else None
    if w.draw == "host":
        W0, Gh = host_set(w, w.n_grad_sets)
        W = [torch.from_numpy(x).to(dev).to(torch.bfloat16) for x in W0]
        Gd = [[torch.from_numpy(g).to(dev).to(torch.bfloat16) for g in gs] for gs in Gh]
        rho = torch.tensor([float(np.linalg.norm(x.astype(np.float64))) for x in W0], dtype=torch.float32,
                           device=dev)
        del W0, Gh
    else:
        W, Gd = device_set(w, dev, torch, w.n_grad_sets)
        rho = torch.stack([x.float().norm() for x in W])
    M = [torch.zeros(x.shape, dtype=torch.float32, device=dev) for x in W]
    stepper = Stepper(w, W, M, rho, dev, torch, nshb, Z)
    mats = [stepper.mats(Gd[s]) for s in range(len(Gd))]
    ws = stepper.workspace(mats[0], dev)

    def step(k):
        stepper(mats[k % len(mats)], ws, stream)

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

    # ---- per-kernel times: the same steps again with an event pair around every launch
    nshb.profile_enable(True)
    nshb.profile_read()
    kp = max(3, min(args.steps, 20))
    for k in range(kp):
        step(k)
    torch.cuda.synchronize()
    prof = nshb.profile_read()
    nshb.profile_enable(False)
    launches_per_step = sum(c for _, c in prof.values()) / kp

    # ---- end to end through the public API with host buffers (see timed_e2e)
    e2e_ms, h2d = None, 0
    if not args.no_e2e:
        n_host = min(2, len(Gd))
        Gh = []
        for s in range(n_host):
            hs = []
            for g in Gd[s]:
                h = torch.empty(g.shape, dtype=g.dtype, pin_memory=True)
                h.copy_(g)
                hs.append(h)
            Gh.append(hs)
        Zh = None
        if Z is not None:
            # a training step's layer inputs arrive with its gradients
            Zh = []
            for z in Z:
                h = torch.empty(z.shape, dtype=z.dtype, pin_memory=True)
                h.copy_(z)
                Zh.append(h)
        del Gd, mats
        torch.cuda.empty_cache()
        ke = max(5, min(args.steps, 20))
        barrier()
        e2e_one, h2d = timed_e2e(Gh, stepper, ws, stream, ke, torch, dev, Zh)
        barrier()
        e2e_ms = max_over_ranks(e2e_one)
        del Gh
    return dict(ms=ms, prof=prof, kp=kp, launches_per_step=launches_per_step, flags=flags,
                clocks=clk.summary(), e2e_ms=e2e_ms, h2d=h2d, d2h=4, n_params=w.n_params, shp=w.shapes)


def run_sharded(args, rank, world, local_rank, w: Workload):
    """Data-parallel step over the ranks (strong scaling: the matrix set is fixed, the ranks
    share it).  Every rank holds the same weights and its own gradients of every matrix;
    one step = reduce-scatter of the gradients onto the owners (mean), the library's step
    on the owned matrices (LPT by NS work), all-gather of the updated weights over NCCL."""
    import torch
    from newton_schulz_hyperball_b200 import sharding
    import newton_schulz_hyperball_b200 as nshb
    if w.step not in ("hyperball", "brake", "himuon"):
        raise ValueError("--sharded runs the MuonH, RadialBrake and HiMuon steps")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    W, _ = device_set(w, dev, torch, 0)                  # identical weights on every rank
    wr = Workload(w.key, w.desc, w.cfg + 100 * (rank + 1), w.named, w.step, w.draw, 1)
    _, Gs = device_set(wr, dev, torch, 1)                 # this rank's own gradients
    G = Gs[0]
    rho = torch.stack([x.float().norm() for x in W])
    kw = {"eta": ETA}
    if w.step == "himuon":
        kw["tile"] = w.tile
    if w.step == "brake":
        kw = {"lr": 0.02, "brake_out": 0.5, "brake_in": 1.0}
    plan = sharding.make_plan(w.shapes, world, rank)
    opt = sharding.ShardedOptimizer(W, rho, plan, w.step, **kw)

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

    for _ in range(args.warmup):
        opt.step(G, stream)
    torch.cuda.synchronize()
    flags = opt.device_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            opt.step(G, stream)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1)) / args.steps
    # the library's step alone on this rank's matrices (no collectives)
    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0.record(stream)
    for _ in range(args.steps):
        opt.local_step(stream)
    l1.record(stream)
    torch.cuda.synchronize()
    local_ms = max_over_ranks(l0.elapsed_time(l1)) / args.steps
    # end to end: this rank's gradients copied from pinned host memory every step
    Gh = []
    for g in G:
        h = torch.empty(g.shape, dtype=g.dtype, pin_memory=True)
        h.copy_(g)
        Gh.append(h)
    st_host = torch.empty(1, dtype=torch.int32).pin_memory()
    ke = max(3, min(args.steps, 10))
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(ke):
        for d, h in zip(G, Gh):
            d.copy_(h, non_blocking=True)
        opt.step(G, stream)
        if opt.mats is not None:
            st_host.copy_(opt.ws[:4].view(torch.int32), non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / ke)
    h2d = sum(g.numel() * g.element_size() for g in G)
    return dict(ms=ms, local_ms=local_ms, e2e_ms=e2e_ms, h2d=h2d, flags=flags, clocks=clk.summary(),
                owned=len(plan.local), loads=plan.loads([sharding.ns_cost(r, c) for r, c in w.shapes]))


def report_sharded(args, w: Workload, r, world):
    line = common_line(args, w, world, r["ms"], r["ms"])
    n = w.n_params
    flops = work_flops(w)
    line.update({
        "scaling": "strong",
        "dtype": "bf16",
        "data": "synthetic (seeded on the device: identical weights, per-rank spiked Gaussian gradients)",
        "config": {"workload": w.desc + "; data-parallel sharded step", "matrices": len(w.shapes), "params": n,
                   "parallelism": f"dp{world}: reduce-scatter gradients -> step on owned matrices (LPT by NS "
                                  f"work) -> all-gather weights (NCCL)",
                   **({"tile": w.tile} if w.tile else {})},
        "throughput": {"value": round(n / (r["ms"] * 1e-3), 1), "unit": "params/s"},
        "step_tflops": round(flops / (r["ms"] * 1e-3) / 1e12, 1),
        "local_step_ms_max_over_ranks": round(r["local_ms"], 4),
        "ns_work_balance": round(max(r["loads"]) / (sum(r["loads"]) / world), 4),
        "device_status": r["flags"], "clocks": r["clocks"],
        "e2e": {"value": round(r["e2e_ms"], 4), "unit": "ms", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": 4,
                "pipeline": "copy of this rank's gradients, then the step (same stream)"},
        "cpu_baseline": None,
        "gpu_launches": None,
    })
    return line


# --------------------------------------------------------------- the oracle
def oracle_matrix(w: Workload, i: int, step: int = 0, state=None):
    """One matrix of the workload through the oracle's step on host-seeded inputs (bf16
    values upcast to fp64).  Returns (seconds of oracle work, state for the next step).
    Input generation is not timed."""
    import numpy as np
    from newton_schulz_hyperball_b200 import workloads as wl
    from oracle import nshb_oracle as o
    r, c = w.shapes[i]
    if state is None:
        W = wl.init_weight(w.cfg, i, r, c, bf16=True).astype(np.float64)
        state = {"W": W, "M": np.zeros_like(W), "V": np.zeros_like(W), "rho": o.fro(W)}
    G = wl.gradient(w.cfg, i, step, r, c, bf16=True).astype(np.float64)
    Zh = None
    if w.step == "newton":
        j = w.extra["z_index"][i]
        Zh = wl.layer_input(w.cfg, j, w.extra["z_rows"][j], w.extra["n_tokens"]).astype(np.float64)
    t0 = time.perf_counter()
    if w.step == "hyperball":
        state["W"], state["M"], _, _ = o.hyperball_step(state["W"], G, state["M"], eta=ETA, rho=state["rho"])
    elif w.step == "brake":
        state["W"], state["M"], _ = o.radial_brake_step(state["W"], G, state["M"], lr=0.02, outward=0.5, inward=1.0)
    elif w.step == "himuon":
        state["W"], state["M"], _, _ = o.himuon_step(state["W"], G, state["M"], tile=w.tile, eta=ETA,
                                                     rho=state["rho"])
    elif w.step == "newton":
        state["W"], state["M"], _, _ = o.newton_muon_step(state["W"], G, state["M"], Zh, ridge_rel=1e-3, eta=ETA,
                                                          rho=state["rho"])
    else:
        state["W"], state["M"], state["V"], _, _ = o.adamh_step(state["W"], G, state["M"], state["V"], t=step + 1,
                                                                eta=ETA, rho=state["rho"])
    return time.perf_counter() - t0, state


def unit_cost(w: Workload, i: int):
    """Work of matrix i in the unit used to extrapolate a sample to the whole set: the
    algorithmic flops of its step (elements for AdamH, which has no matrix products)."""
    r, c = w.shapes[i]
    if w.step == "himuon":
        return himuon_flops([(r, c)], w.tile)
    if w.step == "adamh":
        return float(r * c)
    f = ns_flops([(r, c)])
    if w.step == "newton":
        j = w.extra["z_index"][i]
        d = w.extra["z_rows"][j]
        share = sum(1 for z in w.extra["z_index"] if z == j)
        f += (syrk_flops([d], w.extra["n_tokens"]) + potrf_flops([d])) / share + solve_flops([(r, c)])
    return f


def cpu_sample_plan(w: Workload):
    """(matrix indices, steps) the cpu_baseline leg times: about 10-30 s of fp64 work on
    16 host cores."""
    if w.key in ("gpt2", "gpt2-adamh"):
        return list(range(len(w.shapes))), (2 if w.step == "hyperball" else 5)
    if w.key.startswith("qwen3"):
        return list(range(7)), 1                 # layer 0: every shape of the set once
    if w.step == "himuon":
        return [0, 2, 4], 1                      # 4096^2, 1024x4096, 14336x4096 of layer 0
    return list(range(6)), 1                     # newton: GPT-2 layer 0 with its four Z


def oracle_sample(w: Workload):
    """Times the oracle on the cpu_sample_plan matrices and extrapolates to one step of the
    whole set by the work of the matrices timed.  Returns (ms per full step, description)."""
    idx, steps = cpu_sample_plan(w)
    timed = 0.0
    for i in idx:
        st = None
        for s in range(steps):
            t, st = oracle_matrix(w, i, s, st)
            timed += t
    full = sum(unit_cost(w, i) for i in range(len(w.shapes)))
    part = sum(unit_cost(w, i) for i in idx)
    ms = 1e3 * timed / steps * full / part
    what = f"{len(idx)} of {len(w.shapes)} matrices ({', '.join(w.named[i][0] for i in idx[:7])}" + \
           (", ..." if len(idx) > 7 else "") + f"), {steps} step(s), {timed:.1f} s of oracle work timed"
    if len(idx) < len(w.shapes):
        unit = "elements" if w.step == "adamh" else "algorithmic flops"
        what += f"; extrapolated to the {len(w.shapes)}-matrix step by {unit} (x{full / part:.2f})"
    return ms, what


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


def run_reference(args, w: Workload):
    """The oracle on the host cores as the reference arm.  One step = the oracle's step of ONE
    matrix of the set (the matrices are taken in turn, each from its own seeded inputs), so that
    a `--steps K --warmup W` run ends within minutes.  Returns the measured seconds per timed
    step and the full-step value extrapolated by the work of the matrices timed."""
    n = len(w.shapes)
    times, work = [], []
    with OracleThreads() as th:
        for k in range(args.warmup + args.steps):
            i = k % n
            t, _ = oracle_matrix(w, i, 0)
            if k >= args.warmup:
                times.append(t)
                work.append(unit_cost(w, i))
    full = sum(unit_cost(w, i) for i in range(n))
    value_ms = 1e3 * sum(times) * full / sum(work)
    return dict(ms_per_step=1e3 * sum(times) / len(times), value_ms=value_ms, factor=full * len(times) / sum(work),
                timed_s=sum(times), cores=th.cores, affinity=th.affinity,
                matrices=sorted({w.named[k % n][0] for k in range(args.warmup, args.warmup + args.steps)}))


# ------------------------------------------------------------------ the report
def common_line(args, w: Workload, world, value, ms_per_step):
    return {
        "metric": w.metric,
        "value": round(value, 4),
        "unit": "ms",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
    }


def report(args, w: Workload, r, world, cpu):
    peaks, peak_src = load_peaks()
    prof, kp, n = r["prof"], r["kp"], r["n_params"]

    def kms(*kinds):
        return sum(prof.get(k, (0.0, 0))[0] for k in kinds) / kp

    def klaunch(*kinds):
        return sum(prof.get(k, (0.0, 0))[1] for k in kinds) / kp

    step_s = r["ms"] * 1e-3 * args.steps
    # A kernel timed inside a step whose timed region runs for longer than a second runs at
    # the power-capped clock: its peak is the sustained one, else the burst one.
    sustained = step_s >= 0.5
    peak_tf = peaks.get("bf16_tflops_sustained" if sustained else "bf16_tflops",
                        DEFAULT_PEAKS["bf16_tflops_sustained" if sustained else "bf16_tflops"])
    peak_bw = peaks.get("hbm_gbs", DEFAULT_PEAKS["hbm_gbs"])
    line = common_line(args, w, world, r["ms"], r["ms"])
    line.update({
        "dtype": "bf16" if w.step != "adamh" else "f32 (bf16 storage)",
        "data": "synthetic (seeded W0 ~ N(0, 0.02^2), Gaussian gradients with a rank-8 spike; no dataset)",
        "config": {"workload": w.desc, "matrices": len(w.shapes), "params": n,
                   "ns_steps": 0 if w.step == "adamh" else 5, "inputs": f"drawn on the {w.draw}",
                   "gradient_sets": w.n_grad_sets,
                   "l2": f"no flush: inputs larger than L2 (W + G + M = {n * 8 / 1e9:.2f} GB per step)",
                   "parallelism": f"replica per GPU x{world}"},
        "throughput": {"value": round(world * n / (r["ms"] * 1e-3), 1), "unit": "params/s"},
    })
    if w.tile:
        line["config"]["tile"] = w.tile
    # Streaming kernels: algorithmic HBM bytes momentum 14 B/elem (G 2 + M 4 + 4 + U 4: the NS
    # input X0 is written as a bf16 hi + lo pair, the compensated chain's fp32-accurate start),
    # apply 6 B/elem (W 2 + 2, O 2); reduce (fp32 weights only) re-reads W and O.
    mom_ms, apply_ms, red_ms = kms("momentum"), kms("apply"), kms("reduce")
    if w.step == "adamh":
        adam_ms = kms("adam")
        fused_ms = adam_ms + apply_ms
        fused = 28.0 * n / (fused_ms * 1e-3) / 1e9 if fused_ms > 0 else None
        ach = 22.0 * n / (adam_ms * 1e-3) / 1e9 if adam_ms > 0 else None
        line["roofline"] = {"bound": "hbm", "kernel": "adam_kernel (moments, U~, partials)",
                            "achieved": None if ach is None else round(ach, 1), "peak": peak_bw, "unit": "GB/s",
                            "frac": None if ach is None else round(ach / peak_bw, 4),
                            "traffic": traffic_for("adam_gpt2") if w.key == "gpt2-adamh" and not args.layers else None,
                            "algorithmic_bytes_per_launch": 22 * n,
                            "peak_source": f"{peak_src} copy bandwidth"}
        line["fused_gbs"] = None if fused is None else round(fused, 1)
    else:
        fused_ms = mom_ms + apply_ms + red_ms
        fused = 20.0 * n / (fused_ms * 1e-3) / 1e9 if fused_ms > 0 else None
        line["fused_gbs"] = None if fused is None else round(fused, 1)
        line["fused_frac_of_hbm"] = None if fused is None else round(fused / peak_bw, 4)
        line["momentum_gbs"] = round(14.0 * n / (mom_ms * 1e-3) / 1e9, 1) if mom_ms > 0 else None
        line["apply_gbs"] = round(6.0 * n / (apply_ms * 1e-3) / 1e9, 1) if apply_ms > 0 else None
        flops = work_flops(w)
        if w.step == "himuon" and w.tile in (128, 256):
            kinds, kname = ("gram",), f"himuon_tile{'128' if w.tile == 128 else ''}_kernel (tile-resident NS, T={w.tile})"
        elif w.step == "newton":
            kinds, kname = ("gram", "poly", "update"), "gemm_tc2_kernel (NS Gram / polynomial / update)"
            flops = ns_flops(w.shapes)
        else:
            kinds, kname = ("gram", "poly", "update"), "gemm_tc2_kernel (NS Gram / polynomial / update, CTA pairs)"
        g_ms, g_n = kms(*kinds), klaunch(*kinds)
        tf = flops / (g_ms * 1e-3) / 1e12 if g_ms > 0 else None
        traffic = None
        if not args.layers and w.key in ("gpt2", "qwen3", "qwen3-brake"):
            traffic = traffic_for("gemm_gpt2" if w.key == "gpt2" else "gemm_qwen3")
        line["ns_tflops"] = None if tf is None else round(tf, 1)
        line["ns_frac_of_bf16_peak"] = None if tf is None else round(tf / peak_tf, 4)
        if w.step != "himuon" and g_ms > 0:
            line["ns_tflops_dense_equiv"] = round(ns_flops(w.shapes, dense=True) / (g_ms * 1e-3) / 1e12, 1)
        line["roofline"] = {
            "bound": "tensor", "kernel": kname,
            "achieved": None if tf is None else round(tf, 1), "peak": peak_tf, "unit": "TFLOP/s",
            "frac": None if tf is None else round(tf / peak_tf, 4),
            "traffic": traffic,
            "peak_source": f"{peak_src} bf16 {'sustained' if sustained else 'burst'} "
                           f"(timed region {step_s:.2f} s; burst {peaks.get('bf16_tflops')}, "
                           f"sustained {peaks.get('bf16_tflops_sustained')})",
            "frac_of_burst": None if tf is None else round(tf / peaks.get("bf16_tflops", 1590.0), 4),
            "flops_per_launch": round(flops / max(g_n, 1)),
            "per_launch_ms": round(g_ms / max(g_n, 1), 5),
            "launches_per_step": g_n,
        }
        line["step_tflops"] = round(flops / (r["ms"] * 1e-3) / 1e12, 1)
        if w.step == "newton":
            pre_ms = kms("newton")
            line["precondition_ms"] = round(pre_ms, 4)
            line["syrk_tflop"] = round(syrk_flops(w.extra["z_rows"], w.extra["n_tokens"]) / 1e12, 4)
    line["kernels_ms_per_step"] = {k: round(v[0] / kp, 5) for k, v in prof.items()}
    line["launches_per_step"] = {k: round(v[1] / kp, 2) for k, v in prof.items()}
    line["gpu_launches"] = int(round(r["launches_per_step"] * args.steps))
    line["device_status"] = r["flags"]
    line["clocks"] = r["clocks"]
    if r["e2e_ms"] is not None:
        line["e2e"] = {"value": round(r["e2e_ms"], 4), "unit": "ms", "h2d_bytes_per_step": r["h2d"],
                       "d2h_bytes_per_step": r["d2h"], "pipeline": E2E_PIPELINE}
    else:
        line["e2e"] = {"value": None, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
                       "skipped": "--no-e2e"}
    line["cpu_baseline"] = cpu
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--config", default="qwen3",
                    choices=["qwen3", "qwen3-brake", "gpt2", "gpt2-adamh", "himuon8b", "newton"],
                    help="qwen3: the headline workload (the largest MuonH set on one GPU)")
    ap.add_argument("--optimizer", default=None, choices=["muonh", "adamh"],
                    help="adamh: shorthand for --config gpt2-adamh")
    ap.add_argument("--tile", type=int, default=256, choices=[128, 256, 512], help="--config himuon8b: tile size T")
    ap.add_argument("--layers", type=int, default=0, help="fewer layers of the set (profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sharded", action="store_true",
                    help="data-parallel sharded step over the ranks (reduce-scatter, owned step, all-gather)")
    ap.add_argument("--ncu", action="store_true",
                    help="profiling case: warm-up and `steps` steps only, no timing or report")
    args = ap.parse_args()
    if args.optimizer == "adamh":
        args.config = "gpt2-adamh"
    if args.warmup < 3 and not args.ncu:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = make_workload(args)

    if args.impl == "reference":
        if world > 1 and rank != 0:
            return 0
        r = run_reference(args, w)
        line = common_line(args, w, args.gpus, r["value_ms"], r["ms_per_step"])
        sample = (f"one matrix of the {len(w.shapes)}-matrix set per step, the matrices in turn "
                  f"({', '.join(r['matrices'])}); {args.steps} timed steps = {r['timed_s']:.1f} s of oracle work; "
                  f"value = the timed work extrapolated to one step of the whole set by "
                  f"{'elements' if w.step == 'adamh' else 'algorithmic flops'} (x{r['factor']:.2f})")
        line.update({
            "dtype": "f64", "data": "synthetic (the same seeded inputs, drawn on the host)", "impl": "reference",
            "config": {"workload": w.desc, "matrices": len(w.shapes), "params": w.n_params,
                       "sample_per_step": "one matrix (the oracle's step of that matrix)",
                       **({"tile": w.tile} if w.tile else {})},
            "extrapolated": True,
            "cpu_baseline": {"value": line["value"], "unit": "ms", "cores": r["cores"],
                             "affinity_cores": r["affinity"], "kind": "oracle", "sample": sample},
            "e2e": {"value": line["value"], "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        })
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))

    if args.sharded:
        r = run_sharded(args, rank, world, local_rank, w)
        if rank == 0:
            print(json.dumps(report_sharded(args, w, r, world)), flush=True)
        return 0
    r = run_cuda(args, rank, world, local_rank, w)
    if r is None:
        print("ncu case done", flush=True)
        return 0
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with OracleThreads() as th:
            ms, desc = oracle_sample(w)
        cpu = {"value": round(ms, 3), "unit": "ms", "cores": th.cores, "affinity_cores": th.affinity,
               "kind": "oracle", "sample": desc}
    if rank != 0:
        return 0
    print(json.dumps(report(args, w, r, world, cpu)), flush=True)
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
