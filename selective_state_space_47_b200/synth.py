"""Seeded synthetic inputs for the selective scan and the recurrent step.

This module only draws inputs; it holds none of the scan's arithmetic. The same
tensors (same bytes) feed the CUDA path and the float64 oracle.

Workloads (all A[d, n] = -(n + 1), the S4D-real initialisation; D ~ N(0, 1);
x, z, B, C ~ N(0, 1); dt_raw ~ N(0, 0.5^2); per channel dt log-uniform in
[1e-3, 0.1] and dt_bias = log(expm1(dt)), so softplus(dt_bias) = dt):

  tiny_f32        B=1  L=256     D=64   N=16  float32, gate on, final state out
  small_layer     B=4  L=2048    D=1536 N=16  bfloat16 tokens, float32 state
  mid_layer       B=8  L=4096    D=2048 N=16  bfloat16, gate on, final state out
  long_context    B=1  L=262144  D=5120 N=16  bfloat16 (sequence-parallel case)
  decode          B=256 D=5120 N=16, 1000 chained one-token steps, h ~ N(0, 1)

The chunked (Mamba-2) form with one scalar A per head, H heads of P = 64 channels
sharing the head's step size, N = 128 states (the Mamba-2 2.7B layer's head shape):

  ssd_layer       B=2  L=16384   H=80 (D=5120) P=64 N=128  bfloat16, gate on
  A[h] = -U[1, 16] (Mamba-2's initialisation range), dt per head as above, D ~ N(0, 1)
"""
from dataclasses import dataclass
import math

import torch

SEED_BASE = 20260


@dataclass(frozen=True)
class ScanWorkload:
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    dtype: torch.dtype
    gate: bool = True
    final_state: bool = False


@dataclass(frozen=True)
class SsdWorkload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    dtype: torch.dtype = torch.bfloat16


@dataclass(frozen=True)
class StepWorkload:
    name: str
    batch: int
    dim: int
    dstate: int
    steps: int
    dtype: torch.dtype = torch.bfloat16


WORKLOADS = {
    "tiny_f32": ScanWorkload("tiny_f32", 1, 256, 64, 16, torch.float32, True, True),
    "small_layer": ScanWorkload("small_layer", 4, 2048, 1536, 16, torch.bfloat16, True, True),
    "mid_layer": ScanWorkload("mid_layer", 8, 4096, 2048, 16, torch.bfloat16, True, True),
    "long_context": ScanWorkload("long_context", 1, 262144, 5120, 16, torch.bfloat16, True, True),
    # one sequence of long_context's length over a fifth of its channels: 32 channel groups,
    # too few to fill the GPU with one chain of segments each
    "long_narrow": ScanWorkload("long_narrow", 1, 262144, 1024, 16, torch.bfloat16, True, True),
    "decode": StepWorkload("decode", 256, 5120, 16, 1000),
    "ssd_layer": SsdWorkload("ssd_layer", 2, 16384, 80, 64, 128),
}
SEEDS = {"tiny_f32": SEED_BASE + 0, "small_layer": SEED_BASE + 1, "mid_layer": SEED_BASE + 2,
         "long_context": SEED_BASE + 3, "decode": SEED_BASE + 4, "ssd_layer": SEED_BASE + 5,
         "long_narrow": SEED_BASE + 6}


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def channel_params(dim, dstate, seed, device="cpu"):
    """A [D, N], D skip [D], dt_bias [D] as float32 (drawn on the CPU, then moved)."""
    g = _gen(seed + 7919, "cpu")
    A = -torch.arange(1, dstate + 1, dtype=torch.float32).repeat(dim, 1)
    Dskip = torch.randn(dim, generator=g, dtype=torch.float32)
    u = torch.rand(dim, generator=g, dtype=torch.float64)
    dt = torch.exp(math.log(1e-3) + u * (math.log(0.1) - math.log(1e-3)))
    dt_bias = torch.log(torch.expm1(dt)).to(torch.float32)
    return A.to(device), Dskip.to(device), dt_bias.to(device)


def _normal(shape, g, device, dtype, std=1.0):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def scan_inputs(batch, seqlen, dim, dstate, dtype=torch.float32, seed=SEED_BASE, device="cpu",
                gate=True, h0=False):
    """Tokens of one scan: x, dt, z [B, L, D]; B, C [B, L, N]; plus A, D, dt_bias, h0."""
    g = _gen(seed, device)
    x = _normal((batch, seqlen, dim), g, device, dtype)
    dt = _normal((batch, seqlen, dim), g, device, dtype, std=0.5)
    z = _normal((batch, seqlen, dim), g, device, dtype) if gate else None
    Bm = _normal((batch, seqlen, dstate), g, device, dtype)
    Cm = _normal((batch, seqlen, dstate), g, device, dtype)
    A, Dskip, dt_bias = channel_params(dim, dstate, seed, device)
    h = _normal((batch, dim, dstate), g, device, torch.float32) if h0 else None
    return dict(x=x, dt=dt, z=z, B=Bm, C=Cm, A=A, D=Dskip, dt_bias=dt_bias, h0=h)


def workload_inputs(name, device="cpu", h0=False):
    w = WORKLOADS[name]
    return scan_inputs(w.batch, w.seqlen, w.dim, w.dstate, w.dtype, SEEDS[name], device,
                       gate=w.gate, h0=h0)


def step_inputs(batch, dim, dstate, steps, dtype=torch.bfloat16, seed=SEED_BASE + 4, device="cpu",
                gate=True):
    """Decode: h [B, D, N] float32 ~ N(0, 1); per-step tokens x, dt, z [S, B, D] and B, C [S, B, N]."""
    g = _gen(seed, device)
    h = _normal((batch, dim, dstate), g, device, torch.float32)
    x = _normal((steps, batch, dim), g, device, dtype)
    dt = _normal((steps, batch, dim), g, device, dtype, std=0.5)
    z = _normal((steps, batch, dim), g, device, dtype) if gate else None
    Bm = _normal((steps, batch, dstate), g, device, dtype)
    Cm = _normal((steps, batch, dstate), g, device, dtype)
    A, Dskip, dt_bias = channel_params(dim, dstate, seed, device)
    return dict(h=h, x=x, dt=dt, z=z, B=Bm, C=Cm, A=A, D=Dskip, dt_bias=dt_bias)


def conv_params(dim, batch, dtype=torch.bfloat16, seed=SEED_BASE + 5, device="cpu", bias=True, prefix=True):
    """The block's short convolution: taps conv_w [D, 4] and bias conv_b [D] (float32,
    uniform in [-1/2, 1/2], the default initialisation of a depthwise Conv1d with fan-in
    4), and conv_x0 [B, 3, D], the three tokens before t = 0, ~ N(0, 1) in the token
    dtype. bias / prefix False give None for those."""
    g = _gen(seed + 104729, "cpu")
    w = torch.rand((dim, 4), generator=g, dtype=torch.float32) - 0.5
    b = torch.rand((dim,), generator=g, dtype=torch.float32) - 0.5
    x0 = _normal((batch, 3, dim), g, "cpu", dtype)
    return dict(conv_w=w.to(device), conv_b=b.to(device) if bias else None,
                conv_x0=x0.to(device) if prefix else None)


def to_numpy_storage(t):
    """A token tensor as numpy in its storage form: float32, or uint16 bfloat16 bit patterns."""
    if t is None:
        return None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(f"unsupported storage dtype {t.dtype}")


def ssd_inputs(batch, seqlen, nheads, headdim=64, dstate=128, dtype=torch.bfloat16, seed=SEED_BASE + 5,
               device="cpu", gate=True, h0=False):
    """Tokens of the chunked (one A per head) form: x, z [B, L, H, P]; dt [B, L, H]; B, C
    [B, L, N]; A, D, dt_bias [H] float32; h0 [B, H, P, N] float32 (or None)."""
    g = _gen(seed, device)
    x = _normal((batch, seqlen, nheads, headdim), g, device, dtype)
    dt = _normal((batch, seqlen, nheads), g, device, dtype, std=0.5)
    z = _normal((batch, seqlen, nheads, headdim), g, device, dtype) if gate else None
    Bm = _normal((batch, seqlen, dstate), g, device, dtype)
    Cm = _normal((batch, seqlen, dstate), g, device, dtype)
    gp = _gen(seed + 7919, "cpu")
    A = -(1.0 + 15.0 * torch.rand(nheads, generator=gp, dtype=torch.float32))
    Dskip = torch.randn(nheads, generator=gp, dtype=torch.float32)
    u = torch.rand(nheads, generator=gp, dtype=torch.float64)
    dtv = torch.exp(math.log(1e-3) + u * (math.log(0.1) - math.log(1e-3)))
    dt_bias = torch.log(torch.expm1(dtv)).to(torch.float32)
    h = _normal((batch, nheads, headdim, dstate), g, device, torch.float32) if h0 else None
    return dict(x=x, dt=dt, z=z, B=Bm, C=Cm, A=A.to(device), D=Dskip.to(device), dt_bias=dt_bias.to(device), h0=h)
