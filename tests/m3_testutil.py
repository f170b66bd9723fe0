"""Shared helpers for the parity tests: seeded inputs, oracle calls on host
copies, and the error metric (max over (batch, head) slices of the relative
L2 error over (t, r, p))."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# tolerances: fp32 I/O path and bf16 I/O path (fp32 state)
TOL_F32 = 1e-4
TOL_BF16 = 2e-2
KEYS = ("x", "B", "C", "dt", "lam", "theta", "A", "D")


def tol_for(io: str) -> float:
    return TOL_F32 if io == "f32" else TOL_BF16


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def max_rel_l2_y(y: np.ndarray, yref: np.ndarray) -> float:
    """y, yref [Bt, T, H, R, P]: per (b,h) slice ||y - yref|| / ||yref||, max."""
    if y.size == 0:
        return 0.0
    d = (y - yref).transpose(0, 2, 1, 3, 4).reshape(y.shape[0] * y.shape[2], -1)
    r = yref.transpose(0, 2, 1, 3, 4).reshape(d.shape)
    num = np.linalg.norm(d, axis=1)
    den = np.maximum(np.linalg.norm(r, axis=1), 1e-30)
    return float(np.max(num / den))


def max_rel_l2_state(h: np.ndarray, href: np.ndarray) -> float:
    """h, href [Bt, H, ...]: per (b,h) slice relative L2, max."""
    if h.size == 0:
        return 0.0
    d = (h - href).reshape(h.shape[0] * h.shape[1], -1)
    r = href.reshape(d.shape)
    return float(np.max(np.linalg.norm(d, axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-30)))


def oracle_scan_slices(inp: dict, bh_list, init=None):
    """Oracle on a subset of (b, h) slices: returns dict (b,h) -> (y [T,R,P], h, bp, xp)."""
    # stack the picked slices along the head axis so one oracle call runs them
    # on parallel threads (each slice keeps its own head's A and D)
    bh_list = list(bh_list)
    bi = [b for b, _ in bh_list]
    hi = [h for _, h in bh_list]
    sl = {k: np.ascontiguousarray(np.stack([host64(inp[k][b, :, h]) for b, h in bh_list], axis=1)[None])
          for k in KEYS if k not in ("A", "D")}
    A = host64(inp["A"])
    if A.ndim == 3:  # per-token A [Bt, T, H]: sliced like dt
        sl["A"] = np.ascontiguousarray(np.stack([A[b, :, h] for b, h in bh_list], axis=1)[None])
    else:
        sl["A"] = A[hi]
    sl["D"] = host64(inp["D"])[hi]
    st = None
    if init is not None:
        st = oracle.State(*(np.stack([host64(t[b, h]) for b, h in bh_list])[None] for t in init))
    y, fs = oracle.scan(*(sl[k] for k in KEYS), st)
    out = {}
    for j, key in enumerate(bh_list):
        out[key] = (y[0, :, j], fs.h[0, j], fs.b_prev[0, j], fs.x_prev[0, j])
    return out


def rel_l2(a: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-30))


def max_rel_l2_step(y: np.ndarray, yref: np.ndarray) -> float:
    """One decode step, y, yref [Bt, H, R, P]: per (b,h) slice relative L2
    over (r, p), max over slices (the same metric as the prefill's)."""
    if y.size == 0:
        return 0.0
    d = (y - yref).reshape(y.shape[0] * y.shape[1], -1)
    r = yref.reshape(d.shape)
    return float(np.max(np.linalg.norm(d, axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-30)))


# Worst per-slice errors of the parity tests that record them, printed at the
# end of the session (tests/conftest.py), so the margin against the bar is on
# record in every run's output: (test, worst error, bar).
MARGINS: list = []


def record_margin(name: str, err: float, tol: float):
    MARGINS.append((name, float(err), float(tol)))
