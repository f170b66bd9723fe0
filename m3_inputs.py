"""Seeded synthetic inputs for the Mamba-3 SSM forward.

This module only draws random tensors; it holds none of the method's
arithmetic, so both the fp64 oracle (tests) and the CUDA library (tests,
benchmark) can take their inputs from it without sharing any computation.

Distributions (the 1.5B-scale workloads' synthetic recipe):
  x ~ N(0, 1)                      [Bt, T, H, R, P]
  B, C ~ N(0, 1/N)                 [Bt, T, H, R, N]
  dt = softplus(N(-4, 1))          [Bt, T, H]
  A = -exp(U(0, ln 16))            [H]        (fp32, never rounded; or, with
                                               a_per_token, [Bt, T, H])
  lam = sigmoid(N(0, 1))           [Bt, T, H]
  theta ~ U(-pi, pi)               [Bt, T, H, N/2]   (one angle rate per state pair;
                                                      or, with theta_per_head, [H, N/2])
  D ~ N(0, 1)                      [H]        (fp32, never rounded)
Draw order is fixed (x, B, C, dt, A, lam, theta, D) from one torch.Generator
seeded with the workload's seed.  Tensors are drawn in fp32 and then rounded
to the I/O dtype (round-to-nearest-even); consumers see only the rounded
values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Shape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int   # P
    dstate: int    # N (even)
    rank: int      # R (MIMO rank; 1 = SISO)
    io: str        # "f32" or "bf16"
    seed: int = 0

    @property
    def torch_io(self):
        return torch.float32 if self.io == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Shape":
        return replace(self, **kw)


# The workloads the method is measured on (sizes of the pages' 1.5B-scale
# models), named by what they are.
WORKLOADS = {
    # small fp32-I/O SISO scan (oracle-sized)
    "siso_f32_b1_t256_h4_p64_n64": Shape(1, 256, 4, 64, 64, 1, "f32"),
    # SISO prefill, bf16 I/O, fp32 state
    "siso_bf16_b8_t4096_h32_p64_n128": Shape(8, 4096, 32, 64, 128, 1, "bf16"),
    # MIMO rank-4 prefill, halved state
    "mimo_bf16_b8_t4096_h32_p64_n64_r4": Shape(8, 4096, 32, 64, 64, 4, "bf16"),
    # decode: state from a 1024-token prefill, then single-token steps
    "decode_bf16_b256_h32_p64_n128_r1": Shape(256, 1024, 32, 64, 128, 1, "bf16"),
    "decode_bf16_b256_h32_p64_n128_r4": Shape(256, 1024, 32, 64, 128, 4, "bf16"),
    # long-context MIMO prefill
    "long_mimo_bf16_b1_t65536_h64_p64_n128_r4": Shape(1, 65536, 64, 64, 128, 4, "bf16"),
}
DECODE_STEPS = 1000
LONG_DECODE_STEPS = 256


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _draws(g, device, lead, H, R, P, N):
    """Draw the per-token tensors with leading dims `lead` (e.g. (Bt, T))."""
    f = dict(device=device, dtype=torch.float32, generator=g)
    x = torch.randn(*lead, H, R, P, **f)
    B = torch.randn(*lead, H, R, N, **f) / math.sqrt(N)
    C = torch.randn(*lead, H, R, N, **f) / math.sqrt(N)
    dt = torch.nn.functional.softplus(torch.randn(*lead, H, **f) - 4.0)
    return x, B, C, dt


def make_prefill(shape: Shape, device="cpu", seqlen: int | None = None, a_per_token: bool = False,
                 theta_per_head: bool = False):
    """Inputs of one prefill call.  Returns a dict of tensors on `device`.
    With a_per_token, A is drawn per token-head ([Bt, T, H], fp32) in A's
    place in the draw order; with theta_per_head, theta is drawn per head
    ([H, N/2], same distribution) in theta's place."""
    T = shape.seqlen if seqlen is None else seqlen
    Bt, H, R, P, N = shape.batch, shape.nheads, shape.rank, shape.headdim, shape.dstate
    g = _gen(shape.seed, device)
    f = dict(device=device, dtype=torch.float32, generator=g)
    x, B, C, dt = _draws(g, device, (Bt, T), H, R, P, N)
    A = -torch.exp(torch.rand(*((Bt, T, H) if a_per_token else (H,)), **f) * math.log(16.0))
    lam = torch.sigmoid(torch.randn(Bt, T, H, **f))
    theta = (torch.rand(*((H,) if theta_per_head else (Bt, T, H)), N // 2, **f) * 2.0 - 1.0) * math.pi
    D = torch.randn(H, **f)
    io = shape.torch_io
    return dict(x=x.to(io), B=B.to(io), C=C.to(io), dt=dt.to(io), lam=lam.to(io),
                theta=theta.to(io), A=A.contiguous(), D=D.contiguous())


def make_steps(shape: Shape, nsteps: int, device="cpu", seed_offset: int = 1, a_per_token: bool = False):
    """Per-step decode inputs, leading dim = step: x [S,Bt,H,R,P],
    B/C [S,Bt,H,R,N], dt/lam [S,Bt,H], theta [S,Bt,H,N/2].  A and D are the
    prefill's (same seed), so a prefill followed by these steps is one
    continuous sequence with per-head parameters; with a_per_token the steps
    also carry their own A [S,Bt,H] (fp32, drawn last)."""
    Bt, H, R, P, N = shape.batch, shape.nheads, shape.rank, shape.headdim, shape.dstate
    g = _gen(shape.seed + seed_offset, device)
    f = dict(device=device, dtype=torch.float32, generator=g)
    x, B, C, dt = _draws(g, device, (nsteps, Bt), H, R, P, N)
    lam = torch.sigmoid(torch.randn(nsteps, Bt, H, **f))
    theta = (torch.rand(nsteps, Bt, H, N // 2, **f) * 2.0 - 1.0) * math.pi
    io = shape.torch_io
    out = dict(x=x.to(io), B=B.to(io), C=C.to(io), dt=dt.to(io), lam=lam.to(io), theta=theta.to(io))
    if a_per_token:
        out["A"] = -torch.exp(torch.rand(nsteps, Bt, H, **f) * math.log(16.0))
    return out


def make_bcnorm(shape: Shape, device="cpu", seed_offset: int = 3):
    """Synthetic BC-norm parameters (fp32): RMS-norm weights wB, wC [N] ~
    (1 + 0.1 N(0,1)) / sqrt(N) and head-specific biases bB, bC [H, R, N] ~
    0.1 N(0,1) / sqrt(N), so the normalised rows keep the scale of the raw
    B, C draws (RMS about 1/sqrt(N))."""
    H, R, N = shape.nheads, shape.rank, shape.dstate
    g = _gen(shape.seed + seed_offset, device)
    f = dict(device=device, dtype=torch.float32, generator=g)
    wB = (1.0 + 0.1 * torch.randn(N, **f)) / math.sqrt(N)
    wC = (1.0 + 0.1 * torch.randn(N, **f)) / math.sqrt(N)
    bB = 0.1 * torch.randn(H, R, N, **f) / math.sqrt(N)
    bC = 0.1 * torch.randn(H, R, N, **f) / math.sqrt(N)
    return dict(wB=wB, wC=wC, bB=bB, bC=bC, eps=1e-6)


def make_proj(shape: Shape, device="cpu", seed_offset: int = 4):
    """Synthetic MIMO projection weights (fp32): wx [H, R, P], wB, wC [H, R, N]
    ~ N(0, 1), so that each widened column keeps the scale of the SISO draw,
    and wy [H, R, P] ~ N(0, 1) / sqrt(R), so that the sum over the R ranks
    keeps the scale of one."""
    H, R, P, N = shape.nheads, shape.rank, shape.headdim, shape.dstate
    g = _gen(shape.seed + seed_offset, device)
    f = dict(device=device, dtype=torch.float32, generator=g)
    wx = torch.randn(H, R, P, **f)
    wB = torch.randn(H, R, N, **f)
    wC = torch.randn(H, R, N, **f)
    wy = torch.randn(H, R, P, **f) / math.sqrt(R)
    return dict(wx=wx, wB=wB, wC=wC, wy=wy)


def make_prefill_proj(shape: Shape, device="cpu", **kw):
    """Inputs of one prefill call with the MIMO projections: the draws of
    make_prefill for this shape at rank 1, with x [Bt, T, H, P] and
    B, C [Bt, T, H, N] (the rank axis dropped); the rest unchanged."""
    d = make_prefill(shape.with_(rank=1), device=device, **kw)
    for k in ("x", "B", "C"):
        d[k] = d[k][:, :, :, 0].contiguous()
    return d


def make_steps_proj(shape: Shape, nsteps: int, device="cpu", **kw):
    """Decode-step inputs with the MIMO projections: make_steps at rank 1 with
    x [S, Bt, H, P] and B, C [S, Bt, H, N]."""
    d = make_steps(shape.with_(rank=1), nsteps, device=device, **kw)
    for k in ("x", "B", "C"):
        d[k] = d[k][:, :, :, 0].contiguous()
    return d


def make_state(shape: Shape, device="cpu", seed_offset: int = 2, scale: float = 1.0):
    """A random (h, b_prev, x_prev) state in fp32, for tests that start from a
    nonzero state."""
    Bt, H, R, P, N = shape.batch, shape.nheads, shape.rank, shape.headdim, shape.dstate
    g = _gen(shape.seed + seed_offset, device)
    f = dict(device=device, dtype=torch.float32, generator=g)
    h = torch.randn(Bt, H, N, P, **f) * scale
    bp = torch.randn(Bt, H, R, N, **f) / math.sqrt(N)
    xp = torch.randn(Bt, H, R, P, **f)
    return h, bp, xp
