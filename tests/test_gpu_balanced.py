"""The tensor-core prefill's balanced schedule: with more (batch, head)
slices than SMs, one CTA per SM takes an equal run of all chunks and a slice
cut between two CTAs is continued by the second from the state the first
publishes.  Checked against the fp64 oracle (per slice, 2e-2), and bit for
bit against the one-CTA-per-slice schedule (a call without a workspace),
which runs the same chunk arithmetic: a wrong hand-off, a chunk run twice or
skipped, or a race on a hand-off slot would all break the equality."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from m3_inputs import Shape, make_bcnorm, make_prefill, make_state
from m3_testutil import KEYS, host64, max_rel_l2_state, max_rel_l2_y, record_margin

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:  # collected on CPU only to be deselected
    m3 = None
    DEV = "cpu"


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def dims_of(s: Shape, **kw):
    return m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io, **kw)


def per_slice_call(inp, init, bcnorm=None):
    """The same call without a workspace: one CTA per (batch, head) slice."""
    x = inp["x"]
    Bt, T, H, R, P = x.shape
    N = inp["B"].shape[-1]
    dims = m3.make_dims(Bt, T, H, P, N, R, x.dtype, a_per_token=inp["A"].dim() == 3,
                        theta_per_head=inp["theta"].dim() == 2)
    assert m3.scan_plan_info(dims, flags=m3.PLAN_NO_WORKSPACE).balanced is False
    y = torch.empty_like(x)
    fin = m3.empty_state(Bt, H, N, P, R, device=DEV)
    st = None if init is None else ctypes.pointer(m3.CState(*(t.data_ptr() for t in init)))
    args = (*(ctypes.c_void_p(inp[k].data_ptr()) for k in KEYS), st, ctypes.c_void_p(y.data_ptr()),
            ctypes.pointer(m3.CState(*(t.data_ptr() for t in fin))), None, 0,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    lib = m3.get_lib()
    if bcnorm is None:
        st_ = lib.m3_scan_fwd_algo(m3.ALGO_AUTO, ctypes.byref(dims), *args)
    else:
        cb = m3.CBCNorm(*(t.data_ptr() for t in bcnorm[:4]), float(bcnorm.eps))
        st_ = lib.m3_scan_fwd_bcnorm(m3.ALGO_AUTO, ctypes.byref(dims), ctypes.byref(cb), *args)
    assert st_ == 0, lib.m3_last_error()
    return y, fin


BALANCED = [
    Shape(5, 300, 32, 64, 128, 1, "bf16", 81),   # 160 slices x 3 chunks: runs of 3.2 chunks
    Shape(2, 150, 80, 64, 64, 4, "bf16", 82),    # MIMO: 160 slices x 5 chunks of 32 tokens
    Shape(3, 200, 50, 64, 128, 2, "bf16", 83),   # 150 slices x 4 chunks (one more slice than SMs)
    Shape(1, 520, 300, 64, 128, 4, "bf16", 84),  # 300 slices x 17 chunks, ragged last chunk
]


def test_plan_of_the_balanced_schedule():
    s = Shape(8, 4096, 32, 64, 128, 1, "bf16")
    n = sms()
    info = m3.scan_plan_info(dims_of(s))
    assert info.kernel == m3.KERNEL_TC and info.balanced and info.ctas == n and info.launches == 1
    assert info.workspace_bytes == n * 128 * 64 * 4 + -(-n * 4 // 256) * 256
    assert m3.workspace_size(dims_of(s)) == info.workspace_bytes
    assert m3.scan_plan_info(dims_of(s), flags=m3.PLAN_STATIC).balanced
    w = m3.scan_plan_info(dims_of(s), flags=m3.PLAN_NO_WORKSPACE)
    assert not w.balanced and w.ctas == 8 * 32 and w.workspace_bytes == 0
    # no more slices than SMs (and too many to split): one CTA per slice
    few = m3.scan_plan_info(dims_of(s.with_(batch=4)))
    assert not few.balanced and few.ctas == 4 * 32 and few.workspace_bytes == 0


@pytest.mark.parametrize("shape", BALANCED, ids=lambda s: f"b{s.batch}t{s.seqlen}h{s.nheads}n{s.dstate}r{s.rank}")
def test_balanced_matches_oracle_and_per_slice(shape):
    assert shape.batch * shape.nheads > sms()
    assert m3.scan_plan_info(dims_of(shape)).balanced
    inp = {k: v.to(DEV) for k, v in make_prefill(shape).items()}
    init = m3.State(*(t.to(DEV) for t in make_state(shape)))
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init)
    m3.stream_status()
    y1, f1 = per_slice_call(inp, init)
    m3.stream_status()
    assert torch.equal(y, y1)
    for a, b in zip(fs, f1):
        assert torch.equal(a, b)
    yref, sref = oracle.scan(*(host64(inp[k]) for k in KEYS), oracle.State(*(host64(t) for t in init)))
    ey, eh = max_rel_l2_y(host64(y), yref), max_rel_l2_state(host64(fs.h), sref.h)
    record_margin(f"balanced prefill b{shape.batch}t{shape.seqlen}h{shape.nheads}n{shape.dstate}r{shape.rank}",
                  max(ey, eh), 2e-2)
    assert ey < 2e-2 and eh < 2e-2, (ey, eh)
    np.testing.assert_array_equal(host64(fs.b_prev), sref.b_prev)
    np.testing.assert_array_equal(host64(fs.x_prev), sref.x_prev)


def test_balanced_in_place_resume_and_repeat():
    """init and final_state the same buffers (a slice's state is read by the
    CTA that starts it and written by the one that ends it, after the hand-off),
    and the same call twice gives the same bits."""
    s = BALANCED[0]
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    st = m3.State(*(t.to(DEV) for t in make_state(s)))
    ref_init = m3.State(*(t.clone() for t in st))
    y_ref, f_ref = m3.scan_fwd(*(inp[k] for k in KEYS), ref_init)
    y, _ = m3.scan_fwd(*(inp[k] for k in KEYS), st, final=st)
    m3.stream_status()
    assert torch.equal(y, y_ref)
    for a, b in zip(st, f_ref):
        assert torch.equal(a, b)
    y2, f2 = m3.scan_fwd(*(inp[k] for k in KEYS), ref_init)
    assert torch.equal(y2, y_ref) and all(torch.equal(a, b) for a, b in zip(f2, f_ref))


@pytest.mark.parametrize("feature", ["a_per_token", "theta_per_head", "bcnorm"])
def test_balanced_optional_features_bit_exact(feature):
    """The optional features' instantiations under the balanced schedule: the
    per-head values (A, theta, BC-norm biases) change from slice to slice
    inside one CTA's run."""
    s = Shape(3, 260, 60, 64, 128, 1, "bf16", 85)
    kw = {} if feature == "bcnorm" else {feature: True}
    inp = {k: v.to(DEV) for k, v in make_prefill(s, **kw).items()}
    bcn = None
    if feature == "bcnorm":
        p = make_bcnorm(s, device=DEV)
        bcn = m3.BCNorm(p["wB"], p["wC"], p["bB"], p["bC"], p["eps"])
    assert m3.scan_plan_info(m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io,
                                          **kw)).balanced
    init = m3.State(*(t.to(DEV) for t in make_state(s)))
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, bcnorm=bcn)
    y1, f1 = per_slice_call(inp, init, bcnorm=bcn)
    m3.stream_status()
    assert torch.equal(y, y1)
    for a, b in zip(fs, f1):
        assert torch.equal(a, b)


def test_two_balanced_calls_on_two_streams():
    """Two balanced calls at once on two streams with their own workspaces
    (their CTAs compete for the SMs; each hand-off waits only on a CTA of its
    own grid with a lower index): same bits as one at a time."""
    s = BALANCED[1]
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    inp2 = {k: v.to(DEV) for k, v in make_prefill(s.with_(seed=86)).items()}
    ya, fa = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    yb, fb = m3.scan_fwd(*(inp2[k] for k in KEYS), None)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(3):
        outs.append(m3.scan_fwd(*(inp[k] for k in KEYS), None, stream=s1))
        outs.append(m3.scan_fwd(*(inp2[k] for k in KEYS), None, stream=s2))
    torch.cuda.synchronize()
    m3.stream_status(s1)
    m3.stream_status(s2)
    for i, (y, f) in enumerate(outs):
        yr, fr = (ya, fa) if i % 2 == 0 else (yb, fb)
        assert torch.equal(y, yr)
        assert all(torch.equal(a, b) for a, b in zip(f, fr))
