"""GPU tests of m3_scan_fwd_host, the scan over host-resident sequences with
pipelined copies: parity with the fp64 oracle, bit-exact agreement with the
same (group, slice) units run one by one through m3_scan_fwd on device
tensors (so a race between the copy streams and the kernels would show),
and the edge cases (empty sequence, empty batch, in-place resume, small
workspace, pageable host memory)."""
import numpy as np
import pytest
import torch

import oracle
from m3_inputs import Shape, make_bcnorm, make_prefill, make_state
from m3_testutil import KEYS, host64, max_rel_l2_state, max_rel_l2_y, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
else:
    m3 = None


def pinned(d):
    return {k: v.contiguous().pin_memory() for k, v in d.items()}


def host_state(shape, pin=True):
    st = make_state(shape)
    return m3.State(*(t.pin_memory() if pin else t.clone() for t in st))


def dims_of(shape, a_tok=False, th_head=False):
    return m3.make_dims(shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.rank,
                        shape.torch_io, a_per_token=a_tok, theta_per_head=th_head)


def by_units(inp, init, plan, shape, bcnorm=None):
    """The plan's units run one at a time on device tensors: each slice
    resumes from the previous slice's final state."""
    Bt, T = shape.batch, shape.seqlen
    y = torch.empty(inp["x"].shape, dtype=inp["x"].dtype)
    fin = [torch.empty_like(t) for t in make_state(shape)]
    per_tok = {"x", "B", "C", "dt", "lam"} | ({"theta"} if inp["theta"].dim() == 4 else set()) | \
        ({"A"} if inp["A"].dim() == 3 else set())
    for b0 in range(0, Bt, plan.group_batch):
        b1 = min(Bt, b0 + plan.group_batch)
        sl = plan.last_slice_tokens if b1 == Bt else plan.slice_tokens
        st = None if init is None else m3.State(*(t[b0:b1].cuda() for t in init))
        for t0 in range(0, max(T, 1), max(sl, 1)):
            t1 = min(T, t0 + sl)
            args = [(inp[k][b0:b1, t0:t1] if k in per_tok else inp[k]).contiguous().cuda() for k in KEYS]
            ys, st = m3.scan_fwd(*args, st, bcnorm=bcnorm)
            y[b0:b1, t0:t1] = ys.cpu()
        for f, s in zip(fin, st):
            f[b0:b1] = s.cpu()
    return y, m3.State(*fin)


CASES = [
    # (shape, per-token A, theta per head, with init)
    (Shape(2, 1000, 2, 64, 128, 1, "bf16", 301), False, False, True),    # 2 sequences x 4 slices, ragged last
    (Shape(2, 1000, 2, 64, 128, 1, "bf16", 302), False, False, False),
    (Shape(5, 300, 2, 64, 128, 2, "bf16", 303), False, False, True),     # 4 x 2 slices (256 + 44), last x 3
    (Shape(3, 300, 2, 64, 64, 4, "bf16", 304), True, True, True),        # MIMO, both optional features
    (Shape(16, 100, 2, 64, 64, 1, "f32", 305), False, False, True),      # 8 groups of 2, one slice each
    (Shape(12, 300, 1, 64, 64, 1, "bf16", 307), False, False, True),     # groups of 2 x 2-3 slices: strided copies
    (Shape(1, 2600, 1, 64, 128, 1, "bf16", 306), True, False, False),    # 7 slices of 384 tokens
]


@pytest.mark.parametrize("shape,a_tok,th_head,with_init", CASES,
                         ids=lambda v: f"b{v.batch}t{v.seqlen}n{v.dstate}r{v.rank}{v.io}"
                         if isinstance(v, Shape) else str(v))
def test_host_scan_matches_oracle_and_units(shape, a_tok, th_head, with_init):
    inp = pinned(make_prefill(shape, a_per_token=a_tok, theta_per_head=th_head))
    init = host_state(shape) if with_init else None
    plan = m3.scan_host_plan(dims_of(shape, a_tok, th_head))
    assert plan.units >= 1 and plan.workspace_bytes > 0
    y, fin = m3.scan_fwd_host(*(inp[k] for k in KEYS), init)
    torch.cuda.current_stream().synchronize()
    m3.stream_status()
    st = oracle.State(*(host64(t) for t in init)) if with_init else None
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), st)
    tol = tol_for(shape.io)
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fin.h), sr.h)
    assert ey < tol and eh < tol, f"y {ey:.3e} state {eh:.3e}"
    np.testing.assert_array_equal(host64(fin.b_prev), sr.b_prev)
    np.testing.assert_array_equal(host64(fin.x_prev), sr.x_prev)
    # the same units, one call at a time on device tensors: identical bits
    yu, fu = by_units(inp, init, plan, shape)
    assert torch.equal(y, yu)
    for a, b in zip(fin, fu):
        assert torch.equal(a, b)


@pytest.mark.parametrize("shape", [Shape(3, 700, 2, 64, 128, 1, "bf16", 320), Shape(2, 300, 2, 64, 64, 4, "bf16", 321)],
                         ids=lambda s: f"b{s.batch}t{s.seqlen}n{s.dstate}r{s.rank}")
def test_host_scan_bcnorm(shape):
    """The BC-norm prologue from host parameters: parity with the oracle and
    the same bits as the units run one by one with device parameters."""
    inp = pinned(make_prefill(shape))
    init = host_state(shape)
    p = make_bcnorm(shape)
    hb = m3.BCNorm(p["wB"], p["wC"], p["bB"], p["bC"], p["eps"])
    y, fin = m3.scan_fwd_host(*(inp[k] for k in KEYS), init, bcnorm=hb)
    torch.cuda.synchronize()
    m3.stream_status()
    ref = oracle.BCNorm(*(host64(p[k]) for k in ("wB", "wC", "bB", "bC")), p["eps"])
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), oracle.State(*(host64(t) for t in init)), bcnorm=ref)
    tol = tol_for(shape.io)
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fin.h), sr.h)
    assert ey < tol and eh < tol, f"y {ey:.3e} state {eh:.3e}"
    plan = m3.scan_host_plan(dims_of(shape), bcnorm=True)
    db = m3.BCNorm(*(t.cuda() for t in (p["wB"], p["wC"], p["bB"], p["bC"])), p["eps"])
    yu, fu = by_units(inp, init, plan, shape, bcnorm=db)
    assert torch.equal(y, yu)
    for a, c in zip(fin, fu):
        assert torch.equal(a, c)


def test_host_scan_agrees_with_device_scan():
    """Slices resume through the fp32 state at chunk boundaries: close to the
    single device call, far inside the bar against the oracle."""
    s = Shape(4, 2048, 4, 64, 128, 1, "bf16", 311)
    inp = pinned(make_prefill(s))
    init = host_state(s)
    y, fin = m3.scan_fwd_host(*(inp[k] for k in KEYS), init)
    yd, fd = m3.scan_fwd(*(inp[k].cuda() for k in KEYS), m3.State(*(t.cuda() for t in init)))
    torch.cuda.synchronize()
    m3.stream_status()
    assert max_rel_l2_y(host64(y), host64(yd)) < 5e-3
    assert max_rel_l2_state(host64(fin.h), host64(fd.h)) < 5e-3


def test_host_scan_repeatable_and_in_place():
    """Two back-to-back calls on another stream give the same bits; init and
    final_state may be the same host buffers."""
    s = Shape(3, 700, 2, 64, 128, 1, "bf16", 312)
    inp = pinned(make_prefill(s))
    init = host_state(s)
    ref_init = m3.State(*(t.clone().pin_memory() for t in init))
    stream = torch.cuda.Stream()
    ws = torch.empty(m3.scan_host_plan(dims_of(s)).workspace_bytes, dtype=torch.uint8, device="cuda")
    y1, f1 = m3.scan_fwd_host(*(inp[k] for k in KEYS), ref_init, workspace=ws, stream=stream)
    y2, f2 = m3.scan_fwd_host(*(inp[k] for k in KEYS), ref_init, workspace=ws, stream=stream)
    y3, f3 = m3.scan_fwd_host(*(inp[k] for k in KEYS), init, final=init, workspace=ws, stream=stream)
    stream.synchronize()
    m3.stream_status(stream)
    assert torch.equal(y1, y2) and torch.equal(y1, y3)
    for a, b, c in zip(f1, f2, f3):
        assert torch.equal(a, b) and torch.equal(a, c)
    assert f3.h.data_ptr() == init.h.data_ptr()


def test_host_scan_pageable_memory():
    """Pageable host tensors serialise the copies but give the same result."""
    s = Shape(2, 500, 2, 64, 64, 1, "bf16", 313)
    raw = make_prefill(s)
    yp, fp = m3.scan_fwd_host(*(pinned(raw)[k] for k in KEYS))
    y = torch.empty_like(raw["x"])
    fin = m3.State(*(torch.empty_like(t) for t in make_state(s)))
    m3.scan_fwd_host(*(raw[k] for k in KEYS), y=y, final=fin)
    torch.cuda.synchronize()
    assert torch.equal(y, yp)
    assert torch.equal(fin.h, fp.h)


def test_host_scan_empty_sequence_copies_init():
    s = Shape(3, 0, 2, 64, 64, 1, "bf16", 314)
    inp = pinned(make_prefill(s))
    init = host_state(s)
    y, fin = m3.scan_fwd_host(*(inp[k] for k in KEYS), init)
    torch.cuda.synchronize()
    assert y.numel() == 0
    for a, b in zip(fin, init):
        assert torch.equal(a, b)


def test_host_scan_empty_batch():
    s = Shape(0, 200, 2, 64, 128, 1, "bf16", 315)
    inp = pinned(make_prefill(s))
    assert m3.scan_host_plan(dims_of(s)).workspace_bytes == 0
    y, fin = m3.scan_fwd_host(*(inp[k] for k in KEYS), workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert y.numel() == 0


def test_host_scan_refuses_small_workspace_and_device_tensors():
    s = Shape(1, 300, 2, 64, 128, 1, "bf16", 316)
    inp = pinned(make_prefill(s))
    need = m3.scan_host_plan(dims_of(s)).workspace_bytes
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(m3.M3Error) as ei:
        m3.scan_fwd_host(*(inp[k] for k in KEYS), workspace=ws)
    assert ei.value.status == m3.M3_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        m3.scan_fwd_host(*(inp[k].cuda() for k in KEYS))
