"""Seeded synthetic workloads for causal linear attention.

This module only describes shapes and draws random inputs. It holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from
it without sharing any computation.

The workloads, with the sizes used throughout the tests and the benchmark:

  elu_fp32_fwd       elu(x)+1 forward, fp32 I/O, B=1 H=1 N=256 D=32
  elu_bf16_fwd       elu(x)+1 chunked prefill, bf16 I/O, B=4 H=8 N=4096 D=64,
                     inputs N(0,1)/sqrt(64)
  taylor_bf16_fwd    BASED Taylor forward, bf16 I/O, B=8 H=16 N=2048 d'=16
                     (273 features), Dv=64, inputs N(0,1)
  elu_bf16_train     elu(x)+1 forward+backward, bf16 I/O, B=2 H=16 N=16384
                     D=128, inputs and upstream grad N(0,1)/sqrt(128)
  taylor_decode      BASED Taylor recurrent decode, fp32 I/O: 256 sequences,
                     H=16, d'=16, Dv=64, state from a 2048-token prefill, then
                     1024 one-token steps with fresh N(0,1) q/k/v
  taylor_decode_sym  the same with the folded 153-row Taylor state
  elu_bf16_varlen    16 packed prompts of seeded lengths in [1, 2048], H=8, D=64
  elu_bf16_decay_fwd the headline shape with per-token forget gates
  swa_bf16_fwd       sliding-window softmax attention, w=64, headline shape
  swa_bf16_decode    its decode: 1024 x 16 heads, 64-token caches, 1024 steps
  taylor_bf16_train  the Taylor forward's shape as a training step (forward +
                     backward), inputs and upstream grad N(0,1)
  elu_bf16_decay_train the gated form's training step on the headline shape

Random numbers come from torch's CPU Mersenne-Twister generator seeded with
the workload's index; tensors are drawn in the order Q, K, V, dO (decode: the
prefill's Q, K, V, then per step q, k, v), in fp32, then scaled, then rounded
to bf16 (round-to-nearest-even) for the bf16 workloads. The oracle receives
the rounded values, so it sees the same bytes as the GPU.

The BASED page ("Simple linear attention language models balance the
recall-throughput tradeoff") trains and evaluates on the Pile and MQAR; those
datasets are not used. The i.i.d. Gaussian inputs stand in for the projected
q/k/v of its kernel benchmarks (Knowl 5, Knowl 9).
"""
from __future__ import annotations

import dataclasses
import math

import torch

ELU1 = 0
TAYLOR2 = 1
TAYLOR2_SYM = 2
F32 = 0
BF16 = 1

_DT = {F32: torch.float32, BF16: torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int          # seed
    fmap: int
    dtype: int
    B: int
    H: int
    N: int
    dqk: int
    dv: int
    scale: float
    backward: bool = False
    decode_steps: int = 0
    varlen: bool = False   # B sequences of seeded lengths in [1, N], packed [H, T, *]
    decay: bool = False    # gated form: log forget gates g ~ U(-0.05, 0) per token
    window: int = 0        # sliding-window softmax attention with this window (no feature map)

    @property
    def torch_dtype(self):
        return _DT[self.dtype]

    @property
    def feature_dim(self) -> int:
        # ELU: one feature per input coordinate; Taylor: 1 + d' + d'^2; the
        # folded Taylor map: 1 + 2d' + d'(d'-1)/2.
        if self.fmap == ELU1:
            return self.dqk
        if self.fmap == TAYLOR2:
            return 1 + self.dqk + self.dqk * self.dqk
        return 1 + 2 * self.dqk + self.dqk * (self.dqk - 1) // 2

    def describe(self) -> str:
        fm = {ELU1: "elu1", TAYLOR2: "taylor2", TAYLOR2_SYM: "taylor2sym"}[self.fmap]
        if self.window:
            fm = f"sliding-window softmax w={self.window}"
        dt = "f32" if self.dtype == F32 else "bf16"
        s = f"{self.name}: {fm} {dt} B={self.B} H={self.H} N={self.N} dqk={self.dqk} dv={self.dv}"
        if self.decay:
            s += " gated (g ~ U(-0.05, 0))"
        if self.decode_steps:
            s += f" decode_steps={self.decode_steps}"
        if self.varlen:
            s = (f"{self.name}: {fm} {dt} {self.B} packed sequences of 1..{self.N} tokens "
                 f"(T={sum(varlen_lengths(self))}) H={self.H} dqk={self.dqk} dv={self.dv}")
        return s


WORKLOADS = [
    Workload("elu_fp32_fwd", 0, ELU1, F32, 1, 1, 256, 32, 32, 1.0),
    Workload("elu_bf16_fwd", 1, ELU1, BF16, 4, 8, 4096, 64, 64, 1.0 / math.sqrt(64)),
    Workload("taylor_bf16_fwd", 2, TAYLOR2, BF16, 8, 16, 2048, 16, 64, 1.0),
    Workload("elu_bf16_train", 3, ELU1, BF16, 2, 16, 16384, 128, 128, 1.0 / math.sqrt(128), backward=True),
    Workload("taylor_decode", 4, TAYLOR2, F32, 256, 16, 2048, 16, 64, 1.0, decode_steps=1024),
    # the same decode with the folded Taylor state (153 rows instead of 273)
    Workload("taylor_decode_sym", 4, TAYLOR2_SYM, F32, 256, 16, 2048, 16, 64, 1.0, decode_steps=1024),
    # a serving-style batch: 16 prompts of mixed lengths, elu d=64, packed
    Workload("elu_bf16_varlen", 5, ELU1, BF16, 16, 8, 2048, 64, 64, 1.0 / math.sqrt(64), varlen=True),
    # the headline shape with per-token forget gates
    Workload("elu_bf16_decay_fwd", 6, ELU1, BF16, 4, 8, 4096, 64, 64, 1.0 / math.sqrt(64), decay=True),
    # BASED's local mixer: sliding-window attention, w = 64, d = 64 (the width and head dimension
    # of the page's generation benchmark), on the headline shape; and its decode with a 64-token cache
    Workload("swa_bf16_fwd", 7, ELU1, BF16, 4, 8, 4096, 64, 64, 1.0, window=64),
    # (decode: 1024 sequences so that the 64-token bf16 caches, 268 MB, exceed L2; a 64-token
    # prompt fills each window, and a longer prompt would leave the same cache)
    Workload("swa_bf16_decode", 8, ELU1, BF16, 1024, 16, 64, 64, 64, 1.0, decode_steps=1024, window=64),
    # the BASED Taylor shape as a training step: forward + backward, inputs and
    # upstream gradient N(0,1)
    Workload("taylor_bf16_train", 9, TAYLOR2, BF16, 8, 16, 2048, 16, 64, 1.0, backward=True),
    # the gated form as a training step on the headline shape (gates as elu_bf16_decay_fwd's)
    Workload("elu_bf16_decay_train", 10, ELU1, BF16, 4, 8, 4096, 64, 64, 1.0 / math.sqrt(64), backward=True,
             decay=True),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def _draw(gen, shape, scale, dtype):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(dtype)


def make_inputs(w: Workload, *, B=None, H=None, N=None, seed=None, dtype=None):
    """Draw (q, k, v, dout) on the CPU for workload ``w``.

    Shapes may be shrunk (B, H, N) for small parity cases; the recipe (order,
    scale, rounding) stays the same. ``dout`` is None unless the workload has
    a backward pass. Returned tensors are CPU tensors in the I/O dtype.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    seed = w.index if seed is None else seed
    dt = w.torch_dtype if dtype is None else _DT[dtype]
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    q = _draw(gen, (B, H, N, w.dqk), w.scale, dt)
    k = _draw(gen, (B, H, N, w.dqk), w.scale, dt)
    v = _draw(gen, (B, H, N, w.dv), w.scale, dt)
    dout = _draw(gen, (B, H, N, w.dv), w.scale, dt) if w.backward else None
    return q, k, v, dout


def make_decode_inputs(w: Workload, *, B=None, H=None, prefill_N=None, steps=None, seed=None):
    """Prefill q/k/v [B,H,N,*] then per-step q/k/v stacked as [steps,B,H,*].

    Drawn from one generator in this order: prefill Q, K, V, then for each
    step q, k, v.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if prefill_N is None else prefill_N
    steps = w.decode_steps if steps is None else steps
    seed = w.index if seed is None else seed
    dt = w.torch_dtype
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    q = _draw(gen, (B, H, N, w.dqk), w.scale, dt)
    k = _draw(gen, (B, H, N, w.dqk), w.scale, dt)
    v = _draw(gen, (B, H, N, w.dv), w.scale, dt)
    sq = torch.empty(steps, B, H, w.dqk, dtype=dt)
    sk = torch.empty(steps, B, H, w.dqk, dtype=dt)
    sv = torch.empty(steps, B, H, w.dv, dtype=dt)
    for t in range(steps):
        sq[t] = _draw(gen, (B, H, w.dqk), w.scale, dt)
        sk[t] = _draw(gen, (B, H, w.dqk), w.scale, dt)
        sv[t] = _draw(gen, (B, H, w.dv), w.scale, dt)
    return (q, k, v), (sq, sk, sv)


def varlen_lengths(w: Workload) -> list:
    """Sequence lengths of a packed workload: B integers drawn uniformly from
    [1, N] by a generator seeded with the workload's seed + 1000."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.index + 1000)
    return [int(x) for x in torch.randint(1, w.N + 1, (w.B,), generator=gen)]


def make_varlen_inputs(w: Workload, dtype=None):
    """Packed q, k [H, T, dqk], v [H, T, dv] and cu_seqlens [B+1] (int32) on the
    CPU, drawn in the order q, k, v like make_inputs."""
    lens = varlen_lengths(w)
    T = sum(lens)
    dt = w.torch_dtype if dtype is None else _DT[dtype]
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.index)
    q = _draw(gen, (w.H, T, w.dqk), w.scale, dt)
    k = _draw(gen, (w.H, T, w.dqk), w.scale, dt)
    v = _draw(gen, (w.H, T, w.dv), w.scale, dt)
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32)
    return q, k, v, cu


def make_gates(w: Workload, B=None, H=None, N=None, device="cpu", seed=None):
    """Log forget gates [B, H, N] fp32, uniform on [-0.05, 0), from a generator
    seeded with the workload's seed + 2000 (decay about 2.5 % per token)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    N = w.N if N is None else N
    gen = torch.Generator(device=device)
    gen.manual_seed((w.index if seed is None else seed) + 2000)
    return -0.05 * torch.rand(B, H, N, generator=gen, device=device)


def random_qkv(seed, B, H, N, dqk, dv, *, fmap=ELU1, dtype=F32, scale=1.0, with_dout=False):
    """Free-form seeded draw for edge-case tests (same order and recipe)."""
    w = Workload("adhoc", seed, fmap, dtype, B, H, N, dqk, dv, scale, backward=with_dout)
    return make_inputs(w)
