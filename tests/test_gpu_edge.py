"""GPU parity on the method's edge cases, every CUDA path against the fp64
oracle, slice by slice (max over (batch, head) slices of the relative L2
error over (t, r, p); bars 2e-2 for bf16 I/O, 1e-4 for fp32 I/O):

* deep decay -- A = -16 with dt near 0.5 in every token, so every chunk's
  total decay lies far beyond 2^-100 and the tensor-core kernel builds the
  decay mask element by element instead of as a row factor times a column
  factor (the condition is asserted on the inputs);
* mixed decay -- the same in every other chunk only, so one call takes both
  ways of building the mask;
* lam = 1, theta = 0 -- the Euler rule without rotation, the Mamba-2
  recurrence that "La dualità: Mamba-2 e Mamba-3" (section "Mamba-3",
  paragraph on the exponential-trapezoidal rule) names as the special case
  lam_t = 1 of the trapezoid;
* lam = 0 -- only the previous-token term of the trapezoid writes the state;
* large angles -- |theta| near pi and dt near 0.5 with a common sign per
  state pair, so the chunk-local cumulative angle reaches a few hundred
  radians (asserted on the inputs), with weak decay so the rotated state
  carries over many chunks.

Paths: the tensor-core prefill (N = 128 R = 1, N = 64 R = 4, and N = 128
R = 4 split into segments), the fp32 tensor-core prefill (N = 64, R = 1 and
2), the SIMT prefill (fp32 I/O), and the decode
kernels (one CTA per slice, the persistent rank >= 2 kernel with a full grid
and with few slices, bf16 and fp32 I/O)."""
import math

import numpy as np
import pytest
import torch

import oracle
from m3_inputs import Shape, make_prefill, make_state, make_steps
from m3_testutil import (KEYS, host64, max_rel_l2_state, max_rel_l2_step, max_rel_l2_y, record_margin,
                         tol_for)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:  # collected on CPU only to be deselected
    m3 = None
    DEV = "cpu"

KINDS = ["deep", "mixed", "euler", "lam0", "big_angle"]
LOG2E = 1.4426950408889634
STEP_KEYS = ("x", "B", "C", "dt", "lam", "theta")


def chunk_tokens(shape: Shape) -> int:
    """Tokens per chunk of the tensor-core prefill (128 rows of Q tokens x R ranks)."""
    return 128 // shape.rank


def edge_inputs(shape: Shape, kind: str, steps: int = 0):
    """The seeded inputs of `shape`, changed into the edge case `kind`; with
    steps > 0 also `steps` decode tokens changed the same way."""
    inp = make_prefill(shape)
    st = make_steps(shape, steps) if steps else None
    g = torch.Generator().manual_seed(7919 + shape.seed)
    io = shape.torch_io
    Bt, T, H, K2 = shape.batch, shape.seqlen, shape.nheads, shape.dstate // 2

    def big_dt(*lead):
        return (0.5 + 0.25 * torch.rand(*lead, generator=g)).to(io)

    if kind in ("deep", "mixed"):
        inp["A"] = torch.full((H,), -16.0)
        if kind == "deep":
            inp["dt"] = big_dt(Bt, T, H)
        else:
            deep = ((torch.arange(T) // chunk_tokens(shape)) % 2 == 0)[None, :, None]
            inp["dt"] = torch.where(deep, big_dt(Bt, T, H).float(), inp["dt"].float()).to(io)
        if st is not None:
            st["dt"] = big_dt(steps, Bt, H)
    elif kind == "euler":
        inp["lam"] = torch.ones_like(inp["lam"])
        inp["theta"] = torch.zeros_like(inp["theta"])
        if st is not None:
            st["lam"] = torch.ones_like(st["lam"])
            st["theta"] = torch.zeros_like(st["theta"])
    elif kind == "lam0":
        inp["lam"] = torch.zeros_like(inp["lam"])
        if st is not None:
            st["lam"] = torch.zeros_like(st["lam"])
    elif kind == "big_angle":
        sign = torch.where(torch.rand(Bt, 1, H, K2, generator=g) < 0.5, -1.0, 1.0)
        inp["theta"] = (sign * (math.pi - 0.3 * torch.rand(Bt, T, H, K2, generator=g))).to(io)
        inp["dt"] = (0.45 + 0.1 * torch.rand(Bt, T, H, generator=g)).to(io)
        inp["A"] = torch.full((H,), -0.02)
        if st is not None:
            st["theta"] = (sign[None, :, 0] * (math.pi - 0.3 * torch.rand(steps, Bt, H, K2, generator=g))).to(io)
            st["dt"] = (0.45 + 0.1 * torch.rand(steps, Bt, H, generator=g)).to(io)
    else:
        raise ValueError(kind)
    return inp, st


def chunk_decay_log2(inp, shape: Shape) -> np.ndarray:
    """Per (b, chunk, h): the decay from a chunk's first token to its last in
    log2 units, sum over s = c0+1 .. c0+Q-1 of dt_s |A_h| log2(e) -- the
    quantity the tensor-core kernel compares with 100 to choose how it builds
    the mask.  Full chunks only."""
    Q = chunk_tokens(shape)
    dt = host64(inp["dt"])
    A = host64(inp["A"])
    nfull = shape.seqlen // Q
    d = dt[:, :nfull * Q].reshape(shape.batch, nfull, Q, shape.nheads)[:, :, 1:]
    return d.sum(axis=2) * np.abs(A)[None, None, :] * LOG2E


def chunk_angles(inp, shape: Shape) -> np.ndarray:
    """Largest chunk-local cumulative angle |sum_{s in chunk} dt_s theta_s[k]|."""
    Q = chunk_tokens(shape)
    phi = host64(inp["dt"])[..., None] * host64(inp["theta"])
    nfull = shape.seqlen // Q
    return np.abs(phi[:, :nfull * Q].reshape(shape.batch, nfull, Q, shape.nheads, -1).cumsum(axis=2)).max()


def check_edge_inputs(inp, shape: Shape, kind: str):
    if kind == "deep":
        assert chunk_decay_log2(inp, shape).min() > 110.0, "every full chunk must decay beyond 2^-100"
    elif kind == "mixed":
        dec = chunk_decay_log2(inp, shape)
        assert dec.max() > 110.0 and dec.min() < 90.0, "both ways of building the mask must occur"
    elif kind == "big_angle":
        # about 0.5 * 3 rad per token of a common sign: ~190 rad over a 128-token chunk
        assert chunk_angles(inp, shape) > min(100.0, 1.2 * chunk_tokens(shape))


PREFILL_CASES = [
    ("tc_n128_r1", Shape(2, 300, 2, 64, 128, 1, "bf16", 61), "tc"),
    ("tc_n64_r4", Shape(1, 200, 3, 64, 64, 4, "bf16", 62), "tc"),
    ("tc_split_n128_r4", Shape(1, 600, 2, 64, 128, 4, "bf16", 63), "split"),
    ("simt_f32_n64_r2", Shape(1, 150, 2, 64, 64, 2, "f32", 64), "simt"),
    ("tc32_n64_r1", Shape(2, 300, 2, 64, 64, 1, "f32", 65), "tc"),
    ("tc32_n64_r2", Shape(1, 150, 2, 64, 64, 2, "f32", 66), "tc"),
]


def algo_of(path):
    return {"tc": m3.ALGO_TC, "split": m3.ALGO_TC_SEGMENTS(3), "simt": m3.ALGO_SIMT}[path]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("name,shape,path", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
def test_prefill_edge_case(name, shape, path, kind):
    inp, _ = edge_inputs(shape, kind)
    if path != "simt":
        check_edge_inputs(inp, shape, kind)
    dinp = {k: v.to(DEV) for k, v in inp.items()}
    init = m3.State(*(t.to(DEV) for t in make_state(shape)))
    y, fs = m3.scan_fwd(*(dinp[k] for k in KEYS), init, algo=algo_of(path))
    m3.stream_status()
    if path == "split":
        assert m3.scan_plan(m3.make_dims(*(getattr(shape, f) for f in
                                           ("batch", "seqlen", "nheads", "headdim", "dstate", "rank")),
                                         shape.torch_io), algo_of(path)).segments == 3
    yref, sref = oracle.scan(*(host64(dinp[k]) for k in KEYS), oracle.State(*(host64(t) for t in init)))
    tol = tol_for(shape.io)
    ey = max_rel_l2_y(host64(y), yref)
    eh = max_rel_l2_state(host64(fs.h), sref.h)
    record_margin(f"edge {kind} prefill {name}", max(ey, eh), tol)
    assert ey < tol, f"y rel-L2 {ey:.3e} >= {tol}"
    assert eh < tol, f"state rel-L2 {eh:.3e} >= {tol}"
    np.testing.assert_array_equal(host64(fs.b_prev), sref.b_prev)
    np.testing.assert_array_equal(host64(fs.x_prev), sref.x_prev)


DECODE_CASES = [
    ("tiled_n128_r1", Shape(5, 40, 32, 64, 128, 1, "bf16", 71)),       # one CTA per slice
    ("stream_n128_r4", Shape(5, 40, 32, 64, 128, 4, "bf16", 72)),      # the persistent kernel
    ("stream_few_n128_r4", Shape(1, 40, 16, 64, 128, 4, "bf16", 74)),  # 16 slices: dependent launch
    ("tiled_few_n64_r1", Shape(3, 40, 2, 64, 64, 1, "bf16", 75)),
    ("stream_f32_n64_r2", Shape(2, 40, 2, 64, 64, 2, "f32", 73)),
]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("name,shape", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_edge_case(name, shape, kind):
    """A prefill over the edge-case inputs, then decode steps with edge-case
    tokens, against the oracle's scan followed by its steps."""
    nsteps = 4
    inp, steps = edge_inputs(shape, kind, steps=nsteps)
    dinp = {k: v.to(DEV) for k, v in inp.items()}
    _, st = m3.scan_fwd(*(dinp[k] for k in KEYS), None)
    ys = []
    for i in range(nsteps):
        args = [steps[k][i].contiguous().to(DEV) for k in STEP_KEYS]
        ys.append(m3.step(*args, dinp["A"], dinp["D"], st).clone())
    m3.stream_status()
    _, ost = oracle.scan(*(host64(dinp[k]) for k in KEYS))
    tol = tol_for(shape.io)
    worst = 0.0
    for i in range(nsteps):
        yo, ost = oracle.step(*(host64(steps[k][i]) for k in STEP_KEYS), host64(dinp["A"]), host64(dinp["D"]), ost)
        e = max_rel_l2_step(host64(ys[i]), yo)
        worst = max(worst, e)
        assert e < tol, f"step {i}: y rel-L2 {e:.3e} (worst slice)"
    eh = max_rel_l2_state(host64(st.h), ost.h)
    record_margin(f"edge {kind} decode {name}", max(worst, eh), tol)
    assert eh < tol
    np.testing.assert_array_equal(host64(st.b_prev), ost.b_prev)
    np.testing.assert_array_equal(host64(st.x_prev), ost.x_prev)
