"""Seeded synthetic inputs for the SSD layer (workload table + generators).

This module holds the input recipe only -- none of the layer's arithmetic.
Both the GPU path (tests, bench) and the CPU oracle draw their inputs from
here, on the same seed; tensors generated on one device are copied to the
other so that both sides see bit-identical values.

Workloads are the Mamba-2 mixer shapes of the Video-Ma2mba backbones
(0.3B / 1.3B / 2.7B, model card "Model Variants" table) at long context
(model card "Max context": up to ~1M tokens), plus one tiny fp32 case.
Distributions:
  u (pre-conv x|B|C stream), or x, B, C directly   ~ N(0, 1)
  dt = clamp(softplus(z + bias_h), dt_min, dt_max),  z ~ N(0, 0.5^2) per (t, h),
       bias_h = inverse softplus of dt0_h,  dt0_h ~ logU[dt_min, dt_max]
  A_h = -exp(U[log 1, log 16]),  D_h ~ N(0, 1),  conv w ~ U(-0.5, 0.5), conv bias 0
  h0 = 0 and zero conv tail unless a test asks for random ones.
  backward: dy ~ N(0, 1) in the I/O dtype, dh_final ~ N(0, 1).
"""
from dataclasses import dataclass, field
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    b: int
    L: int
    H: int
    P: int
    N: int
    G: int
    Q: int
    s: int
    dtype: str                 # "f32" or "bf16": the I/O dtype of x/B/C/u/v/y
    dt_min: float = 1e-3
    dt_max: float = 1e-1
    segments: int = 1          # the sequence is processed as this many resumed calls
    seed: int = 0

    @property
    def d_inner(self) -> int:
        return self.H * self.P

    @property
    def cch(self) -> int:
        return self.H * self.P + 2 * self.G * self.N

    @property
    def seg_len(self) -> int:
        return self.L // self.segments

    @property
    def tokens(self) -> int:
        return self.b * self.L


WORKLOADS = [
    Workload("tiny-f32-L256", b=1, L=256, H=2, P=16, N=16, G=1, Q=32, s=64, dtype="f32", seed=0),
    Workload("mamba2-0.3b-L16k", b=1, L=16384, H=32, P=64, N=128, G=1, Q=128, s=1024,
             dtype="bf16", seed=1),
    Workload("mamba2-0.3b-L1M-stream8", b=1, L=1048576, H=32, P=64, N=128, G=1, Q=128,
             s=4096, dtype="bf16", segments=8, seed=2),
    Workload("mamba2-1.3b-b2-L256k", b=2, L=262144, H=64, P=64, N=128, G=1, Q=128, s=2048,
             dtype="bf16", seed=3),
    Workload("mamba2-2.7b-b4-L64k", b=4, L=65536, H=80, P=64, N=128, G=1, Q=128, s=1024,
             dtype="bf16", dt_min=1e-2, dt_max=5e-1, seed=4),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_params(wl: Workload, device="cpu", seed=None):
    """Per-head and per-channel parameters: A, D, conv w, conv bias, dt bias."""
    g = _gen(wl.seed if seed is None else seed, device)
    H = wl.H
    logA = torch.empty(H, device=device, dtype=torch.float64).uniform_(0.0, math.log(16.0), generator=g)
    A = (-torch.exp(logA)).to(torch.float32)
    D = torch.randn(H, device=device, dtype=torch.float32, generator=g)
    w = torch.empty(wl.cch, 4, device=device, dtype=torch.float32).uniform_(-0.5, 0.5, generator=g)
    bias = torch.zeros(wl.cch, device=device, dtype=torch.float32)
    logdt0 = torch.empty(H, device=device, dtype=torch.float64).uniform_(
        math.log(wl.dt_min), math.log(wl.dt_max), generator=g)
    dt0 = torch.exp(logdt0)
    dt_bias = (dt0 + torch.log(-torch.expm1(-dt0))).to(torch.float32)
    return {"A": A, "D": D, "w": w, "bias": bias, "dt_bias": dt_bias}


def make_dt_raw(wl: Workload, L=None, b=None, device="cpu", seed=None):
    """The raw draws z ~ N(0, 0.5^2) [b, L, H] fp32 that make_dt turns into dt
    (for the entry points that take dt before its bias and softplus)."""
    L = wl.L if L is None else L
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 1000, device)
    return torch.randn(b, L, wl.H, device=device, dtype=torch.float32, generator=g) * 0.5


def make_dt(wl: Workload, dt_bias, L=None, b=None, device="cpu", seed=None):
    """dt [b, L, H] fp32 > 0 from the softplus recipe."""
    L = wl.L if L is None else L
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 1000, device)
    z = torch.randn(b, L, wl.H, device=device, dtype=torch.float32, generator=g) * 0.5
    dt = torch.nn.functional.softplus(z + dt_bias.to(device))
    return dt.clamp_(wl.dt_min, wl.dt_max)


def make_u(wl: Workload, L=None, b=None, device="cpu", seed=None, dtype=None):
    """Pre-conv packed stream u [b, L, H*P + 2GN] ~ N(0,1) in the I/O dtype."""
    L = wl.L if L is None else L
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 2000, device)
    dt_ = torch_dtype(wl.dtype) if dtype is None else dtype
    u = torch.empty(b, L, wl.cch, device=device, dtype=dt_)
    # draw in row blocks to bound the float32 temporaries at large L
    step = max(1, (1 << 26) // max(1, wl.cch))
    for bi in range(b):
        for t0 in range(0, L, step):
            t1 = min(L, t0 + step)
            u[bi, t0:t1] = torch.randn(t1 - t0, wl.cch, device=device, dtype=torch.float32,
                                       generator=g).to(dt_)
    return u


def make_xbc(wl: Workload, L=None, b=None, device="cpu", seed=None):
    """x [b,L,H*P], B [b,L,G*N], C [b,L,G*N] ~ N(0,1) drawn directly (standalone scan)."""
    L = wl.L if L is None else L
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 3000, device)
    dt_ = torch_dtype(wl.dtype)
    x = torch.randn(b, L, wl.d_inner, device=device, generator=g).to(dt_)
    Bm = torch.randn(b, L, wl.G * wl.N, device=device, generator=g).to(dt_)
    Cm = torch.randn(b, L, wl.G * wl.N, device=device, generator=g).to(dt_)
    return x, Bm, Cm


def make_h0(wl: Workload, b=None, device="cpu", seed=None, scale=1.0):
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 4000, device)
    return torch.randn(b, wl.H, wl.P, wl.N, device=device, generator=g) * scale


def make_tail(wl: Workload, b=None, device="cpu", seed=None):
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 5000, device)
    return torch.randn(b, 3, wl.cch, device=device, generator=g).to(torch_dtype(wl.dtype))


def make_grads(wl: Workload, L=None, b=None, device="cpu", seed=None):
    """Upstream gradients for the backward pass: dy [b, L, H*P] ~ N(0,1) in the
    I/O dtype and dh_final [b, H, P, N] ~ N(0,1) fp32."""
    L = wl.L if L is None else L
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 6000, device)
    dy = torch.randn(b, L, wl.d_inner, device=device, generator=g).to(torch_dtype(wl.dtype))
    dhf = torch.randn(b, wl.H, wl.P, wl.N, device=device, generator=g)
    return dy, dhf


def make_conv_grads(wl: Workload, b=None, device="cpu", seed=None):
    """The upstream gradient of the conv buffer a segment hands on: dtail_out [b, 3, C_ch]
    ~ N(0,1) fp32, and a conv bias ~ N(0, 0.3^2) [C_ch] fp32 for the gradient tests."""
    b = wl.b if b is None else b
    g = _gen((wl.seed if seed is None else seed) + 7000, device)
    dto = torch.randn(b, 3, wl.cch, device=device, generator=g)
    bias = torch.randn(wl.cch, device=device, generator=g) * 0.3
    return dto, bias


def scaled(wl: Workload, **changes) -> Workload:
    """A copy of a workload with some fields changed (e.g. a shorter L)."""
    d = dict(wl.__dict__)
    d.update(changes)
    return Workload(**d)
