"""fp64 CPU oracle for the Mamba-3 SSM forward -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never imports it and shares no code with it.

The arithmetic lives in ``m3_oracle.c`` (plain sequential recurrence, fp64,
one thread per (batch, head) slice); this module compiles it with gcc on first
use and marshals numpy arrays into it.  The recurrence it follows is the
three-term exponential-trapezoidal update displayed in "Знакомство с Mamba-3"
(section 1), with the complex state realised as 2x2 rotation blocks (same
page, section 2; "La dualità: Mamba-2 e Mamba-3", section "Mamba-3") and the
MIMO rank-R write and readout (same chapter, MIMO paragraph).

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, special-case reductions to Mamba-2, an explicit
complex-diagonal recurrence, a brute-force masked-attention dual, a
hand-derived worked example and a chunked restatement).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3_oracle.c")
_LIB = os.path.join(_HERE, "libm3_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64 = ctypes.c_int64
        dp = ctypes.c_void_p
        lib.m3o_scan.argtypes = ([i64] * 6 + [dp] * 8 + [dp] * 3 + [dp] * 4 + [ctypes.c_int] * 3 + [dp] * 4
                                 + [ctypes.c_double])
        lib.m3o_scan.restype = ctypes.c_int
        lib.m3o_step.argtypes = [i64] * 5 + [dp] * 8 + [dp] * 4 + [ctypes.c_int] * 2 + [dp] * 4 + [ctypes.c_double]
        lib.m3o_step.restype = ctypes.c_int
        lib.m3o_num_cores.argtypes = []
        lib.m3o_num_cores.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_cores() -> int:
    return int(_load().m3o_num_cores())


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


@dataclass
class BCNorm:
    """BC-norm prologue: RMS norm of every (token, head, rank) row of B and C
    over N, times w [N], plus the head-specific bias b [H, R, N]."""
    wB: np.ndarray
    wC: np.ndarray
    bB: np.ndarray
    bC: np.ndarray
    eps: float


def _bcn_args(bcn):
    if bcn is None:
        return [None] * 4 + [0.0]
    return [_f64(bcn.wB), _f64(bcn.wC), _f64(bcn.bB), _f64(bcn.bC), float(bcn.eps)]


@dataclass
class State:
    h: np.ndarray       # [Bt, H, N, P]
    b_prev: np.ndarray  # [Bt, H, R, N]
    x_prev: np.ndarray  # [Bt, H, R, P]


def scan(x, B, C, dt, lam, theta, A, D, init: State | None = None, nthreads: int = 0,
         bcnorm: BCNorm | None = None):
    """Full-sequence scan.  Shapes: x [Bt,T,H,R,P], B/C [Bt,T,H,R,N],
    dt/lam [Bt,T,H], theta [Bt,T,H,N/2] (or [H,N/2]: fixed per head), D [H],
    A [H] (per head) or [Bt,T,H] (per token); optional BC-norm prologue.
    Returns (y, State)."""
    x, B, C, dt, lam, theta, A, D = map(_f64, (x, B, C, dt, lam, theta, A, D))
    Bt, T, H, R, P = x.shape
    N = B.shape[-1]
    assert B.shape == (Bt, T, H, R, N) and C.shape == B.shape
    assert dt.shape == (Bt, T, H) and lam.shape == dt.shape
    assert theta.shape in ((Bt, T, H, N // 2), (H, N // 2)) and D.shape == (H,)
    th_head = int(theta.ndim == 2)
    assert A.shape in ((H,), (Bt, T, H))
    a_tok = int(A.shape == (Bt, T, H) and A.ndim == 3)
    h0 = bp0 = xp0 = None
    if init is not None:
        h0, bp0, xp0 = _f64(init.h), _f64(init.b_prev), _f64(init.x_prev)
        assert h0.shape == (Bt, H, N, P) and bp0.shape == (Bt, H, R, N) and xp0.shape == (Bt, H, R, P)
    y = np.zeros((Bt, T, H, R, P))
    hT = np.zeros((Bt, H, N, P))
    bpT = np.zeros((Bt, H, R, N))
    xpT = np.zeros((Bt, H, R, P))
    bn = _bcn_args(bcnorm)
    rc = _load().m3o_scan(Bt, T, H, P, N, R, *map(_ptr, (x, B, C, dt, lam, theta, A, D)),
                          _ptr(h0), _ptr(bp0), _ptr(xp0),
                          _ptr(y), _ptr(hT), _ptr(bpT), _ptr(xpT), int(nthreads), a_tok, th_head,
                          *map(_ptr, bn[:4]), bn[4])
    if rc != 0:
        raise ValueError("oracle scan rejected its arguments")
    return y, State(hT, bpT, xpT)


@dataclass
class MimoProj:
    """MIMO projections, as this build reads "Mamba-3, parte 1" (the
    architecture paragraph: the MIMO projections widen B and C to the shape
    the MIMO SSM needs) and "Знакомство с Mamba-3" (section 3: rank-R input
    and output projections, B_t in R^{N x R}, x_t in R^{P x R}): per head and
    rank, elementwise weights that widen the SISO-shaped x_t [P], B_t, C_t [N]
    of a token-head to rank R, and project the rank-R output back to P."""
    wx: np.ndarray  # [H, R, P]
    wB: np.ndarray  # [H, R, N]
    wC: np.ndarray  # [H, R, N]
    wy: np.ndarray  # [H, R, P]


def _widen(v, w):
    """v [..., H, K] (SISO-shaped), w [H, R, K] -> [..., H, R, K]: column r is w[h, r] * v."""
    return _f64(v)[..., :, None, :] * _f64(w)


def scan_proj(x, B, C, dt, lam, theta, A, D, proj: MimoProj, init: State | None = None, nthreads: int = 0):
    """Scan with the MIMO projections: x [Bt,T,H,P], B/C [Bt,T,H,N] are widened
    to rank R (X[..., r, :] = wx[h, r] * x, likewise B and C), the rank-R scan
    runs as `scan`, and y [Bt,T,H,P] = sum_r wy[h, r] * Y[..., r, :] (Y with its
    D term).  The state keeps the rank-R form (b_prev, x_prev widened)."""
    Y, st = scan(_widen(x, proj.wx), _widen(B, proj.wB), _widen(C, proj.wC), dt, lam, theta, A, D, init,
                 nthreads=nthreads)
    return (Y * _f64(proj.wy)).sum(axis=-2), st


def step_proj(x, B, C, dt, lam, theta, A, D, proj: MimoProj, state: State):
    """One decode step with the MIMO projections: x [Bt,H,P], B/C [Bt,H,N];
    returns (y [Bt,H,P], new State)."""
    Y, st = step(_widen(x, proj.wx), _widen(B, proj.wB), _widen(C, proj.wC), dt, lam, theta, A, D, state)
    return (Y * _f64(proj.wy)).sum(axis=-2), st


def step(x, B, C, dt, lam, theta, A, D, state: State, bcnorm: BCNorm | None = None):
    """One decode step for every (b,h).  x [Bt,H,R,P], B/C [Bt,H,R,N],
    dt/lam [Bt,H], theta [Bt,H,N/2], D [H], A [H] or [Bt,H] (per token).
    Returns (y, new State); the input state is not modified."""
    x, B, C, dt, lam, theta, A, D = map(_f64, (x, B, C, dt, lam, theta, A, D))
    Bt, H, R, P = x.shape
    N = B.shape[-1]
    h = _f64(state.h).copy()
    bp = _f64(state.b_prev).copy()
    xp = _f64(state.x_prev).copy()
    y = np.zeros((Bt, H, R, P))
    assert A.shape in ((H,), (Bt, H))
    assert theta.shape in ((Bt, H, N // 2), (H, N // 2))
    a_tok = int(A.ndim == 2)
    th_head = int(theta.ndim == 2)
    bn = _bcn_args(bcnorm)
    rc = _load().m3o_step(Bt, H, P, N, R, *map(_ptr, (x, B, C, dt, lam, theta, A, D)),
                          _ptr(h), _ptr(bp), _ptr(xp), _ptr(y), a_tok, th_head, *map(_ptr, bn[:4]), bn[4])
    if rc != 0:
        raise ValueError("oracle step rejected its arguments")
    return y, State(h, bp, xp)
