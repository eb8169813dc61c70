#!/usr/bin/env python
"""Throughput benchmark for the B200 causal linear attention library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-secondary]

One JSON line on stdout (rank 0).  The headline workload is the elu(x)+1 bf16
chunked prefill, B=4 H=8 N=4096 D=64 (one step = one la_forward over the
batch); value = prefill tokens/s (B*N per step, all ranks).  The same line
carries, under "workloads", the BASED Taylor bf16 prefill (B=8 H=16 N=2048
d'=16), the elu bf16 training step (forward+backward, B=2 H=16 N=16384
D=128) and the BASED Taylor fp32 decode (256 sequences x 16 heads, 1024
one-token steps per graph replay), each with its own roofline.

Timing: W untimed warm-up steps, then exactly K steps replayed from a CUDA
graph, bracketed by a barrier and a device synchronisation, timed with CUDA
events on the launching stream; the max over ranks is reported.  Inputs that
fit in L2 rotate through enough copies that every step reads data last
touched more than L2's capacity ago.  With --gpus N > 1 each rank runs an
independent replica on its own GPU (the path needs no collective), so
scaling is weak.

--impl reference times the fp64 CPU oracle on this host's cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- utilities

def rank_env():
    """(world size, rank, local rank) from the torchrun environment; (1, 0, 0)
    when launched alone."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x, dist_on, device=None):
    """The largest of every rank's x.  Every rank calls it at the same point."""
    if not dist_on:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_seed(w, rank):
    """Each replica draws its own inputs: the workload's seed, offset by rank."""
    return w.index + 1000 * rank


def metric_name(w):
    return ("decode tokens/s" if w.decode_steps else
            "training tokens/s" if w.backward else "prefill tokens/s")


def base_config(w, world):
    """The config keys both arms report for workload w on `world` replicas."""
    return {"workload": w.describe(), "parallelism": f"replicas{world}"}


def whole_job_rate(units_per_rank, world, ms):
    """Units per second over all ranks for a step of `ms` milliseconds (the
    max over ranks): every replica processes the same number of units."""
    return units_per_rank * world / (ms * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text):
    """C/CUDA source with comments removed and whitespace runs collapsed, so
    that an edit to comments alone keeps a kernel's hash (string literals,
    such as inline PTX, are kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] in "\"'":
            q, j = text[i], i + 1
            while j < n and text[j] != q:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    return " ".join("".join(out).split())


def source_hash(*names):
    """Hash of the code (comments and layout aside) of kernel sources."""
    h = hashlib.sha256()
    for n in names:
        text = open(os.path.join(ROOT, "causal_kernelized_sequence_b200", "csrc", n), encoding="utf-8").read()
        h.update(_code_only(text).encode())
    return h.hexdigest()[:16]


def load_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel
    source is unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d:
        return None
    try:
        if source_hash(*d["sources"]) != d["source_hash"]:
            return None
    except OSError:
        return None
    return d["bytes_per_launch"]


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, device_index, period_s=0.005):
        self.dev = device_index
        self.period = period_s
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
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
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
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for n, bit in names.items():
                    if mask & bit:
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------- workloads

class Prefill:
    """One step = la_forward over the whole batch (o only)."""

    def __init__(self, w: W.Workload, dev, seed_offset=0):
        import causal_kernelized_sequence_b200 as la
        self.la, self.w, self.dev = la, w, dev
        g = torch.Generator(device=dev)
        g.manual_seed(replica_seed(w, seed_offset))
        set_bytes = w.B * w.H * w.N * (2 * w.dqk + 2 * w.dv) * 2
        self.nsets = max(1, math.ceil(2 * L2_BYTES / set_bytes) + 1) if set_bytes < 2 * L2_BYTES else 1
        mk = lambda d: (torch.randn(w.B, w.H, w.N, d, device=dev, generator=g) * w.scale).to(w.torch_dtype)
        self.sets = [(mk(w.dqk), mk(w.dqk), mk(w.dv), torch.empty(w.B, w.H, w.N, w.dv, device=dev, dtype=w.torch_dtype))
                     for _ in range(self.nsets)]
        # gated form: one log gate per head-token (fp32), one tensor per set
        self.gates = [W.make_gates(w, device=dev, seed=replica_seed(w, seed_offset) + i) for i in range(self.nsets)] \
            if w.decay else None
        self.tokens = w.B * w.N
        esz = 2 if w.dtype == W.BF16 else 4
        self.alg_bytes = w.B * w.H * w.N * ((2 * w.dqk + 2 * w.dv) * esz + (4 if w.decay else 0))
        F = w.feature_dim
        self.alg_flops = 4.0 * F * (w.dv + 1) * w.B * w.H * w.N
        wsb = (la.load_library().la_forward_decay_workspace_bytes if w.decay else la.la_forward_workspace_bytes)(
            w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
        self.ws = torch.empty(wsb, dtype=torch.uint8, device=dev) if wsb else None

    def step(self, i):
        q, k, v, o = self.sets[i % self.nsets]
        if self.gates is not None:
            self.la.la_forward(q, k, v, self.w.fmap, out=o, log_decay=self.gates[i % self.nsets], workspace=self.ws)
        else:
            self.la.la_forward(q, k, v, self.w.fmap, out=o, workspace=self.ws)

    def l2_note(self):
        return (f"{self.nsets} rotating input/output sets of "
                f"{self.alg_bytes / 1e6:.1f} MB (> 126 MB L2 between reuses)" if self.nsets > 1
                else f"inputs {self.alg_bytes / 1e6:.0f} MB > 126 MB L2")


class VarlenPrefill:
    """One step = la_forward_varlen over a packed batch of mixed-length
    sequences (o only)."""

    def __init__(self, w: W.Workload, dev, seed_offset=0):
        import causal_kernelized_sequence_b200 as la
        self.la, self.w, self.dev = la, w, dev
        lens = W.varlen_lengths(w)
        self.T = T = sum(lens)
        self.max_len = max(lens)
        g = torch.Generator(device=dev)
        g.manual_seed(replica_seed(w, seed_offset))
        set_bytes = w.H * T * (2 * w.dqk + 2 * w.dv) * 2
        self.nsets = max(1, math.ceil(2 * L2_BYTES / set_bytes) + 1) if set_bytes < 2 * L2_BYTES else 1
        mk = lambda d: (torch.randn(w.H, T, d, device=dev, generator=g) * w.scale).to(w.torch_dtype)
        self.sets = [(mk(w.dqk), mk(w.dqk), mk(w.dv), torch.empty(w.H, T, w.dv, device=dev, dtype=w.torch_dtype))
                     for _ in range(self.nsets)]
        self.cu = torch.tensor([0] + torch.tensor(lens).cumsum(0).tolist(), dtype=torch.int32, device=dev)
        self.tokens = T
        esz = 2 if w.dtype == W.BF16 else 4
        self.alg_bytes = w.H * T * (2 * w.dqk + 2 * w.dv) * esz
        self.alg_flops = 4.0 * w.feature_dim * (w.dv + 1) * w.H * T
        wsb = la.la_forward_varlen_workspace_bytes(w.B, w.H, self.max_len, w.dqk, w.dv, w.fmap, w.dtype)
        self.ws = torch.empty(wsb, dtype=torch.uint8, device=dev) if wsb else None

    def step(self, i):
        q, k, v, o = self.sets[i % self.nsets]
        self.la.la_forward_varlen(q, k, v, self.cu, self.max_len, self.w.fmap, out=o, workspace=self.ws)

    def l2_note(self):
        return (f"{self.nsets} rotating input/output sets of "
                f"{self.alg_bytes / 1e6:.1f} MB (> 126 MB L2 between reuses)")


class Train:
    """One step = la_forward (o, den) + la_backward (dq, dk, dv); for a gated
    workload la_forward_decay + la_backward_decay (also dL/dg)."""

    def __init__(self, w, dev, seed_offset=0):
        import causal_kernelized_sequence_b200 as la
        self.la, self.w, self.dev = la, w, dev
        g = torch.Generator(device=dev)
        g.manual_seed(replica_seed(w, seed_offset))
        mk = lambda d: (torch.randn(w.B, w.H, w.N, d, device=dev, generator=g) * w.scale).to(w.torch_dtype)
        self.q, self.k, self.v, self.do = mk(w.dqk), mk(w.dqk), mk(w.dv), mk(w.dv)
        self.o = torch.empty_like(self.v)
        self.den = torch.empty(w.B, w.H, w.N, device=dev)
        self.dq, self.dk, self.dvv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        lib = la.load_library()
        if w.decay:
            self.gate = W.make_gates(w, device=dev, seed=replica_seed(w, seed_offset))
            self.dgate = torch.empty_like(self.gate)
            self.fws_bytes = lib.la_forward_decay_workspace_bytes(w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
            self.bws_bytes = lib.la_backward_decay_workspace_bytes(w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
        else:
            self.fws_bytes = la.la_forward_workspace_bytes(w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
            self.bws_bytes = la.la_backward_workspace_bytes(w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
        self.fws = torch.empty(max(1, self.fws_bytes), dtype=torch.uint8, device=dev)
        self.bws = torch.empty(max(1, self.bws_bytes), dtype=torch.uint8, device=dev)
        self.tokens = w.B * w.N
        e = 2
        BHN = w.B * w.H * w.N
        gb = 4 if w.decay else 0   # the gate, read by each pass; dL/dg written by the backward
        self.fwd_bytes = BHN * (2 * w.dqk + 2 * w.dv) * e + BHN * 4 + BHN * gb
        self.bwd_bytes = BHN * (2 * w.dqk + 2 * w.dv) * e + BHN * (2 * w.dqk + w.dv) * e + 2 * BHN * gb
        self.alg_bytes = self.fwd_bytes + self.bwd_bytes
        F = w.feature_dim
        self.alg_flops = (4.0 * F * (w.dv + 1) + 10.0 * F * w.dv + 6.0 * F) * BHN

    def step(self, i):
        la = self.la
        w = self.w
        lib = la.load_library()
        import ctypes
        P = lambda t: ctypes.c_void_p(t.data_ptr())
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        if w.decay:
            r = lib.la_forward_decay(P(self.q), P(self.k), P(self.v), P(self.gate), P(self.o), None, None, None, None,
                                     P(self.den), P(self.fws), self.fws_bytes, w.B, w.H, w.N, w.dqk, w.dv, w.fmap,
                                     w.dtype, st)
            assert r == 0, r
            r = lib.la_backward_decay(P(self.q), P(self.k), P(self.v), P(self.gate), P(self.do), P(self.dq),
                                      P(self.dk), P(self.dvv), P(self.dgate), P(self.bws), self.bws_bytes,
                                      w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype, st)
            assert r == 0, r
            return
        r = lib.la_forward(P(self.q), P(self.k), P(self.v), P(self.o), None, None, P(self.den), P(self.fws),
                           self.fws_bytes, w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype, st)
        assert r == 0, r
        r = lib.la_backward(P(self.q), P(self.k), P(self.v), P(self.do), P(self.dq), P(self.dk), P(self.dvv),
                            P(self.bws), self.bws_bytes, w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype, st)
        assert r == 0, r

    def l2_note(self):
        return f"inputs {self.alg_bytes / 1e6:.0f} MB > 126 MB L2"


class Decode:
    """One step = 1024 one-token la_decode_step calls (one new token for each
    of the B*H heads per call), replayed from a CUDA graph as on the BASED
    page's generation benchmark."""

    def __init__(self, w, dev, seed_offset=0, steps=None):
        import causal_kernelized_sequence_b200 as la
        self.la, self.w, self.dev = la, w, dev
        T = w.decode_steps if steps is None else steps
        self.T = T
        g = torch.Generator(device=dev)
        g.manual_seed(replica_seed(w, seed_offset))
        mk = lambda *s: torch.randn(*s, device=dev, generator=g).to(w.torch_dtype)
        q, k, v = mk(w.B, w.H, w.N, w.dqk), mk(w.B, w.H, w.N, w.dqk), mk(w.B, w.H, w.N, w.dv)
        r = la.la_forward(q, k, v, w.fmap, state=True)
        self.s, self.z = r["s"], r["z"]
        del q, k, v, r
        self.sq, self.sk, self.sv = mk(T, w.B, w.H, w.dqk), mk(T, w.B, w.H, w.dqk), mk(T, w.B, w.H, w.dv)
        self.y = torch.empty(T, w.B, w.H, w.dv, device=dev, dtype=w.torch_dtype)
        self.tokens = w.B * T
        F = w.feature_dim
        esz = 4 if w.dtype == W.F32 else 2
        self.bytes_per_call = w.B * w.H * (2 * (F * w.dv + F) * 4 + (2 * w.dqk + 2 * w.dv) * esz)
        self.alg_bytes = self.bytes_per_call * T
        self.alg_flops = 4.0 * F * (w.dv + 1) * w.B * w.H * T

    def step(self, i):
        for t in range(self.T):
            self.la.la_decode_step(self.sq[t], self.sk[t], self.sv[t], self.s, self.z, self.w.fmap, y=self.y[t])

    def l2_note(self):
        return f"state {self.s.numel() * 4 / 1e6:.0f} MB > 126 MB L2"


class SwaPrefill:
    """One step = la_swa_forward over the whole batch (o only)."""

    def __init__(self, w: W.Workload, dev, seed_offset=0):
        import causal_kernelized_sequence_b200 as la
        self.la, self.w, self.dev = la, w, dev
        g = torch.Generator(device=dev)
        g.manual_seed(replica_seed(w, seed_offset))
        set_bytes = w.B * w.H * w.N * (2 * w.dqk + 2 * w.dv) * 2
        self.nsets = max(1, math.ceil(2 * L2_BYTES / set_bytes) + 1) if set_bytes < 2 * L2_BYTES else 1
        mk = lambda d: (torch.randn(w.B, w.H, w.N, d, device=dev, generator=g) * w.scale).to(w.torch_dtype)
        self.sets = [(mk(w.dqk), mk(w.dqk), mk(w.dv), torch.empty(w.B, w.H, w.N, w.dv, device=dev, dtype=w.torch_dtype))
                     for _ in range(self.nsets)]
        self.tokens = w.B * w.N
        self.alg_bytes = w.B * w.H * w.N * (2 * w.dqk + 2 * w.dv) * 2
        # flops of the band only: 2 w (dqk + dv) per head-token (QK^T and PV)
        self.alg_flops = 2.0 * w.window * (w.dqk + w.dv) * w.B * w.H * w.N

    def step(self, i):
        q, k, v, o = self.sets[i % self.nsets]
        self.la.la_swa_forward(q, k, v, self.w.window, out=o)

    def l2_note(self):
        return (f"{self.nsets} rotating input/output sets of "
                f"{self.alg_bytes / 1e6:.1f} MB (> 126 MB L2 between reuses)")


class SwaDecode:
    """One step = 1024 sliding-window decode steps (one token for each of the
    B*H heads per call) on w-token caches filled from an N-token prompt."""

    def __init__(self, w, dev, seed_offset=0, steps=None):
        import causal_kernelized_sequence_b200 as la
        self.la, self.w, self.dev = la, w, dev
        T = w.decode_steps if steps is None else steps
        self.T = T
        g = torch.Generator(device=dev)
        g.manual_seed(replica_seed(w, seed_offset))
        mk = lambda *s: torch.randn(*s, device=dev, generator=g).to(w.torch_dtype)
        k, v = mk(w.B, w.H, w.N, w.dqk), mk(w.B, w.H, w.N, w.dv)
        self.kc, self.vc = la.la_swa_cache_fill(k, v, w.window)
        del k, v
        self.sq, self.sk, self.sv = mk(T, w.B, w.H, w.dqk), mk(T, w.B, w.H, w.dqk), mk(T, w.B, w.H, w.dv)
        self.y = torch.empty(T, w.B, w.H, w.dv, device=dev, dtype=w.torch_dtype)
        # positions per step, precomputed so a step launches only the decode kernels
        self.pos = (w.N + torch.arange(T, device=dev, dtype=torch.int32))[:, None].expand(T, w.B).contiguous()
        self.tokens = w.B * T
        esz = 2 if w.dtype == W.BF16 else 4
        per_head = (w.window * (w.dqk + w.dv) + (w.dqk + w.dv) + 2 * w.dqk + 2 * w.dv) * esz
        self.alg_bytes = per_head * w.B * w.H * T
        self.alg_flops = 2.0 * w.window * (w.dqk + w.dv) * w.B * w.H * T

    def step(self, i):
        for t in range(self.T):
            self.la.la_swa_decode_step(self.sq[t], self.sk[t], self.sv[t], self.kc, self.vc, self.pos[t],
                                       self.w.window, y=self.y[t])

    def l2_note(self):
        return f"caches {(self.kc.numel() + self.vc.numel()) * self.kc.element_size() / 1e6:.0f} MB > 126 MB L2"


def make_run(w, dev, seed_offset):
    if w.window and w.decode_steps:
        return SwaDecode(w, dev, seed_offset)
    if w.window:
        return SwaPrefill(w, dev, seed_offset)
    if w.decode_steps:
        return Decode(w, dev, seed_offset)
    if w.backward:
        return Train(w, dev, seed_offset)
    if w.varlen:
        return VarlenPrefill(w, dev, seed_offset)
    return Prefill(w, dev, seed_offset)


def capture(run, nsteps, stream):
    """CUDA graph of `nsteps` consecutive steps."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(nsteps):
            run.step(i)
    return g


def timed(run, steps, warmup, dist_on, device_index, graph_len=None, repeats=1):
    """Run warm-up, then `repeats` timed regions of exactly `steps` steps each,
    replayed from CUDA graphs, each bracketed by a barrier and a device
    synchronisation and timed with CUDA events on the launching stream (max
    over ranks).  Returns (median ms per step, [min, mean, max] ms per step
    over the repeats, clocks sampled over all of them)."""
    stream = torch.cuda.Stream()
    # eager warm-up: also configures kernels before any capture
    with torch.cuda.stream(stream):
        for i in range(max(1, warmup)):
            run.step(i)
    torch.cuda.synchronize()
    G = graph_len or min(steps, 100)
    full, rem = divmod(steps, G)
    g = capture(run, G, stream) if full else None
    gr = capture(run, rem, stream) if rem else None
    # graph warm-up
    for _ in range(max(1, warmup // G)):
        (g or gr).replay()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    per_step = []
    with ClockSampler(device_index) as clk:
        for _ in range(max(1, repeats)):
            if dist_on:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            with torch.cuda.stream(stream):
                start.record(stream)
                for _ in range(full):
                    g.replay()
                if gr is not None:
                    gr.replay()
                end.record(stream)
            torch.cuda.synchronize()
            if dist_on:
                torch.distributed.barrier()
            per_step.append(max_over_ranks(start.elapsed_time(end), dist_on, "cuda") / steps)
    del g, gr
    return statistics.median(per_step), [min(per_step), statistics.fmean(per_step), max(per_step)], clk.summary()


def _e2e_buffers(w, dev, rank, nsets):
    """Pinned host q, k, v (the step's inputs) and o (its result), and `nsets`
    device buffer sets plus the forward's workspace."""
    import causal_kernelized_sequence_b200 as la
    g = torch.Generator()
    g.manual_seed(replica_seed(w, rank))
    mk = lambda d: (torch.randn(w.B, w.H, w.N, d, generator=g) * w.scale).to(w.torch_dtype).pin_memory()
    hq, hk, hv = mk(w.dqk), mk(w.dqk), mk(w.dv)
    ho = torch.empty(w.B, w.H, w.N, w.dv, dtype=w.torch_dtype).pin_memory()
    sets = [tuple(torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (hq, hk, hv, ho)) for _ in range(nsets)]
    wsb = la.la_forward_workspace_bytes(w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev) if wsb else None
    return (hq, hk, hv, ho), sets, ws


def _e2e_serial(w, dev, steps, warmup, dist_on, rank):
    """Every step on one stream: copy q, k, v in, forward, copy o out."""
    import causal_kernelized_sequence_b200 as la
    (hq, hk, hv, ho), [(dq_, dk_, dv_, do_)], ws = _e2e_buffers(w, dev, rank, 1)
    stream = torch.cuda.Stream()

    def one():
        dq_.copy_(hq, non_blocking=True)
        dk_.copy_(hk, non_blocking=True)
        dv_.copy_(hv, non_blocking=True)
        la.la_forward(dq_, dk_, dv_, w.fmap, out=do_, workspace=ws)
        ho.copy_(do_, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(1, warmup)):
            one()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        s.record(stream)
        for _ in range(steps):
            one()
        e.record(stream)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    ms = max_over_ranks(s.elapsed_time(e) / steps, dist_on, "cuda")
    return ms, (hq, hk, hv, ho)


def _e2e_pipelined(w, dev, steps, warmup, dist_on, rank):
    """The same steps on three streams with two device buffer sets: step t's
    inputs are copied in while step t-1 computes and step t-2's output is
    copied out, as a serving loop would run them.  Every step still copies all
    of its inputs in and its whole result out inside the timed region.  Also
    checks that the result copied out last is that step's forward."""
    import causal_kernelized_sequence_b200 as la
    (hq, hk, hv, ho), sets, ws = _e2e_buffers(w, dev, rank, 2)
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: [torch.cuda.Event() for _ in range(2)]
    copied_in, computed, copied_out = ev(), ev(), ev()
    used = [False, False]

    def step(t):
        b = t & 1
        dq_, dk_, dv_, do_ = sets[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(computed[b])        # step t-2 has read this set's inputs
            dq_.copy_(hq, non_blocking=True)
            dk_.copy_(hk, non_blocking=True)
            dv_.copy_(hv, non_blocking=True)
            copied_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(copied_in[b])
            if used[b]:
                s_comp.wait_event(copied_out[b])    # step t-2's output has left this set
            la.la_forward(dq_, dk_, dv_, w.fmap, out=do_, workspace=ws)
            computed[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            ho.copy_(do_, non_blocking=True)
            copied_out[b].record(s_out)
        used[b] = True

    for t in range(max(1, warmup)):
        step(t)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record(s_in)
    for t in range(steps):
        step(t)
    end.record(s_out)   # after the last output copy, which follows every other step's work
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    ms = max_over_ranks(start.elapsed_time(end) / steps, dist_on, "cuda")
    last = sets[(steps - 1) & 1]
    ok = torch.equal(ho, last[3].cpu())
    return ms, (hq, hk, hv, ho), ok


def e2e_prefill(w, dev, steps, warmup, dist_on=False, rank=0):
    """Same metric through the public API with host buffers: pinned host q,k,v
    copied in and o copied out inside the timed region, every step.  Runs the
    pipelined loop; the serial one-stream loop is the fallback if the pipelined
    one fails or its last output does not check out.  Returns (ms per step, max
    over ranks; h2d bytes; d2h bytes; mode)."""
    mode = "pipelined: copy-in, forward and copy-out on three streams, two buffer sets"
    if dist_on:
        # Every rank must take the same collective steps: an exception here
        # ends the job rather than leaving the ranks at different barriers,
        # and a failed check falls back on all ranks together.
        ms, host, ok = _e2e_pipelined(w, dev, steps, warmup, dist_on, rank)
        if max_over_ranks(0.0 if ok else 1.0, dist_on, "cuda") > 0:
            mode = "serial: one stream (the pipelined loop's last output did not check out on some rank)"
            ms, host = _e2e_serial(w, dev, steps, warmup, dist_on, rank)
    else:
        try:
            ms, host, ok = _e2e_pipelined(w, dev, steps, warmup, dist_on, rank)
            if not ok:
                raise RuntimeError("last output copied out differs from the device result")
        except Exception as exc:   # noqa: BLE001 - any failure falls back to the serial loop
            mode = f"serial: one stream (pipelined loop failed: {exc})"
            ms, host = _e2e_serial(w, dev, steps, warmup, dist_on, rank)
    hq, hk, hv, ho = host
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size()
    return ms, h2d, d2h, mode


# ----------------------------------------------------------------- CPU oracle

class OracleSample:
    """The fp64 oracle on a bounded sample of workload w: every one of the
    B*H heads (so OpenMP has all of them to share out, as on the full
    workload) for the first `positions` tokens (decode: that many one-token
    steps from a zero state).  The recurrence's cost per head-token does not
    depend on the position, so tokens/s scales to the full workload by the
    head-token count."""

    def __init__(self, w, positions):
        from oracle import oracle as orc
        orc.build()
        self.orc, self.w = orc, w
        self.full_positions = w.decode_steps if w.decode_steps else w.N
        self.Ns = max(1, min(int(positions), self.full_positions))
        Hs = w.B * w.H
        g = torch.Generator()
        g.manual_seed(w.index)
        mk = lambda d: (torch.randn(1, Hs, self.Ns, d, generator=g) * w.scale).to(w.torch_dtype)
        self.q, self.k, self.v = mk(w.dqk), mk(w.dqk), mk(w.dv)
        self.do = mk(w.dv) if w.backward else None

    def once(self):
        orc, w = self.orc, self.w
        q, k, v = self.q, self.k, self.v
        if w.backward:
            orc.forward_recurrent(w.fmap, q, k, v)
            orc.backward_recurrent(w.fmap, q, k, v, self.do)
        elif w.decode_steps:
            import numpy as np
            s = np.zeros((w.B * w.H, w.feature_dim, w.dv))
            z = np.zeros((w.B * w.H, w.feature_dim))
            for t in range(self.Ns):
                orc.decode_step(w.fmap, q[0, :, t], k[0, :, t], v[0, :, t], s, z)
        else:
            orc.forward_recurrent(w.fmap, q, k, v)

    def tokens_per_s(self, seconds_per_run):
        """Tokens/s of the full workload (B sequences x all positions) at
        this sample's speed."""
        return self.w.B * self.Ns / seconds_per_run

    def describe(self):
        w = self.w
        what = "decode steps" if w.decode_steps else "recurrent form" + (" + backward" if w.backward else "")
        unit = "steps" if w.decode_steps else "positions"
        return (f"fp64 oracle ({what}) on all {w.B * w.H} heads x {self.Ns} of {self.full_positions} {unit}; "
                f"tokens/s scaled to the full workload by head-token count")


def sized_oracle_sample(w, seconds):
    """An OracleSample whose one run takes about `seconds` of wall time on
    this host (at most the full workload), sized from a 32-position probe."""
    probe = OracleSample(w, 32)
    t0 = time.perf_counter()
    probe.once()
    dt = max(time.perf_counter() - t0, 1e-6)
    return OracleSample(w, int(32 * seconds / dt))


def oracle_baseline(w, min_cpu_s):
    """(tokens/s, wall seconds, description): the full-workload oracle run
    (or a sample of about 3 s wall per run) repeated until it has used about
    `min_cpu_s` of CPU time."""
    smp = sized_oracle_sample(w, 3.0)
    reps = 0
    t0 = time.perf_counter()
    c0 = time.process_time()
    while True:
        smp.once()
        reps += 1
        if time.process_time() - c0 >= min_cpu_s or time.perf_counter() - t0 >= 60:
            break
    wall = time.perf_counter() - t0
    cpu_s = time.process_time() - c0
    desc = smp.describe() + f"; {reps} runs, {cpu_s:.1f} s of CPU time over the oracle's threads"
    return smp.tokens_per_s(wall / reps), wall, desc


def omp_threads():
    try:
        return int(os.environ.get("OMP_NUM_THREADS", "")) or os.cpu_count()
    except ValueError:
        return os.cpu_count()


# ----------------------------------------------------------------- main

def roofline_entry(bound, achieved, peak, unit, traffic):
    return {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic}


def run_reference(args):
    """The oracle arm: rank 0 alone times the fp64 oracle; other ranks exit.
    Each step is one run of the same all-head sample the other arm's
    cpu_baseline uses (the full workload when one run of it takes a few
    seconds at most), sized so that warm-up and steps together take about
    two minutes."""
    _, rank, _ = rank_env()
    if rank != 0:
        return 0
    w = W.BY_NAME[args.workload]
    per_step_s = min(3.0, 120.0 / (args.warmup + args.steps))
    smp = sized_oracle_sample(w, per_step_s)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        smp.once()
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = statistics.median(times)
    value = smp.tokens_per_s(sec)
    desc = smp.describe() + ", one run per step, median over the steps"
    line = {
        "impl": "reference", "metric": metric_name(w), "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sum(times) / len(times) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": base_config(w, args.gpus), "timing": "host wall clock, fp64 oracle",
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": omp_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="elu_bf16_fwd", choices=list(W.BY_NAME))
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed regions of --steps steps each; the line reports their median")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="run this many untimed steps of --workload and exit (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        return run_reference(args)

    world, rank, local = rank_env()
    dist_on = world > 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist_on:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)

    import causal_kernelized_sequence_b200 as la
    la.load_library()
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])

    w = W.BY_NAME[args.workload]
    run = make_run(w, dev, rank)
    if args.profile_calls:
        for i in range(args.profile_calls):
            run.step(i)
        torch.cuda.synchronize()
        la.la_get_device_status()
        print(json.dumps({"profile_calls": args.profile_calls, "workload": w.describe(),
                          "kernels": la.kernel_plan(w)["kernels"]}), flush=True)
        return 0
    ms, spread, clocks = timed(run, args.steps, args.warmup, dist_on, local, repeats=args.repeats)
    value = whole_job_rate(run.tokens, world, ms)
    achieved = run.alg_bytes / (ms * 1e-3) / 1e9
    from causal_kernelized_sequence_b200 import kernel_plan
    kp = kernel_plan(w)
    line = {
        "metric": metric_name(w),
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == W.BF16 else "f32", "data": "synthetic",
        "config": base_config(w, world),
        "repeats": args.repeats, "ms_per_step_min_max": [round(spread[0], 6), round(spread[2], 6)],
        "ms_per_step_mean": round(spread[1], 6),
        "timing": f"median of {args.repeats} timed regions of {args.steps} steps (CUDA graphs, CUDA events)",
        "l2": run.l2_note(),
        "roofline": dict(roofline_entry("hbm", achieved, hbm, "GB/s", load_traffic("forward:" + w.name)),
                         peak_source=peak_kind, alg_bytes_per_step=run.alg_bytes,
                         launches_per_step=kp["launches_per_step"]),
        "clocks": clocks,
        "gpu_launches": kp["launches_per_step"] * args.steps * args.repeats,
        "kernels": kp["kernels"],
    }
    # e2e through the public API with host buffers
    if not w.decode_steps and not w.backward:
        e_ms, h2d, d2h, e_mode = e2e_prefill(w, dev, min(args.steps, 50), 3, dist_on, rank)
        line["e2e"] = {"value": round(whole_job_rate(run.tokens, world, e_ms), 1), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "mode": e_mode}

    if rank == 0 and world == 1 and not args.no_cpu:
        v, dt, desc = oracle_baseline(w, min_cpu_s=15.0)
        line["cpu_baseline"] = {"value": round(v, 1), "unit": "tokens/s", "cores": omp_threads(),
                                "kind": "oracle", "sample": desc + f" ({dt:.1f} s wall)"}

    if not args.no_secondary and world == 1:
        # The other workloads, each with its own roofline.  Compact keys, and
        # the configs with a published target last, so that a reader keeping
        # only the end of the line still has them: v = tokens/s, ms = per step,
        # hbm = fraction of measured HBM bandwidth on the algorithmic bytes,
        # tc = fraction of measured dense bf16 peak on the algorithmic FLOPs,
        # dram_x = DRAM bytes over algorithmic bytes (recorded ncu capture of
        # the current code, else absent).
        sec = {}
        for name in ("elu_bf16_varlen", "elu_bf16_decay_fwd", "elu_bf16_decay_train", "swa_bf16_fwd",
                     "swa_bf16_decode", "taylor_decode_sym", "taylor_bf16_train", "taylor_decode", "elu_bf16_train",
                     "taylor_bf16_fwd"):
            ws = W.BY_NAME[name]
            r2 = make_run(ws, dev, 0)
            st = 3 if ws.decode_steps else 50
            ms2, spread2, clk2 = timed(r2, st, 3, False, local, graph_len=1 if ws.decode_steps else None,
                                       repeats=3)
            ent = {"v": round(r2.tokens / (ms2 * 1e-3), 1), "ms": round(ms2, 4),
                   "hbm": round(r2.alg_bytes / (ms2 * 1e-3) / 1e9 / hbm, 4),
                   "tc": round(r2.alg_flops / (ms2 * 1e-3) / 1e12 / float(peaks["bf16_tflops"]), 4)}
            tr = load_traffic("step:" + name)
            if tr:
                ent["dram_x"] = round(tr / r2.alg_bytes, 3)
            sec[name] = ent
            print(f"[bench] {ws.describe()}: {ent['v'] / 1e6:.2f} M tokens/s, {ms2:.4f} ms/step "
                  f"(min {spread2[0]:.4f}, mean {spread2[1]:.4f}, max {spread2[2]:.4f}), {ent['hbm'] * 100:.1f} % HBM, "
                  f"{ent['tc'] * 100:.1f} % bf16 peak, clocks {clk2.get('sm_mhz')} MHz {clk2.get('reasons')}",
                  file=sys.stderr, flush=True)
            del r2
            torch.cuda.empty_cache()
        line["workloads"] = sec
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
