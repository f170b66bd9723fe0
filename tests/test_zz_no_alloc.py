"""The workspace-free prefill entry point (m3_scan_fwd_static: split
sequences keep their per-segment states in the library's own device scratch)
against the workspace entry point, on two different calls in a row.  Same
kernels and the same segment choice, so the results are identical."""
import pytest
import torch

from m3_inputs import Shape, make_prefill, make_state
from m3_testutil import KEYS

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:
    m3 = None
    DEV = "cpu"


def _dims(s):
    return m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io)


def test_static_scratch_matches_workspace_path_twice():
    shapes = [Shape(1, 8192, 2, 64, 128, 1, "bf16", 71), Shape(2, 3000, 1, 64, 64, 4, "bf16", 72)]
    for s in shapes:
        info = m3.scan_plan_info(_dims(s), flags=m3.PLAN_STATIC)
        assert info.segments > 1 and info.workspace_bytes > 0  # the scratch is really used
    for s in shapes:
        inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
        init = m3.State(*(t.to(DEV) for t in make_state(s)))
        y_ref, f_ref = m3.scan_fwd(*(inp[k] for k in KEYS), init)
        y, f = m3.scan_fwd_static(*(inp[k] for k in KEYS), init)
        m3.stream_status()
        assert torch.equal(y, y_ref)
        assert torch.equal(f.h, f_ref.h)
        assert torch.equal(f.b_prev, f_ref.b_prev) and torch.equal(f.x_prev, f_ref.x_prev)


def test_static_scratch_refuses_oversize():
    s = Shape(8, 384, 32, 64, 128, 1, "bf16", 73)  # 3 segments x 256 slices x 128 x 65 fp32 > 24 MiB
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    with pytest.raises(m3.M3Error) as e:
        m3.scan_fwd_static(*(inp[k] for k in KEYS), None, algo=m3.ALGO_TC_SEGMENTS(3))
    assert e.value.status == m3.M3_ERR_UNSUPPORTED
    assert "scratch" in str(e.value)
    # the library's own choice never exceeds the scratch
    y, _ = m3.scan_fwd_static(*(inp[k] for k in KEYS), None)
    y_ref, _ = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    m3.stream_status()
    assert torch.equal(y, y_ref)


def test_static_plan_reports_the_capped_segment_choice():
    """Where the workspace entry point's own segment choice would not fit the
    scratch, the static entry point splits into fewer segments; the plan
    query with M3_PLAN_STATIC says so, and both calls agree within the bf16
    bar (they differ only in where the sequence is cut)."""
    # 50 sequences of 1280 chunks: the free choice is 21 segments (33 MiB of
    # per-segment states), the scratch admits 9
    s = Shape(1, 40960, 50, 64, 128, 4, "bf16", 75)
    free = m3.scan_plan_info(_dims(s))
    capped = m3.scan_plan_info(_dims(s), flags=m3.PLAN_STATIC)
    assert free.workspace_bytes > 24 << 20 >= capped.workspace_bytes > 0
    assert 1 < capped.segments < free.segments
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    y_ref, f_ref = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    y, f = m3.scan_fwd_static(*(inp[k] for k in KEYS), None)
    m3.stream_status()
    ey = ((y.float() - y_ref.float()).norm() / y_ref.float().norm()).item()
    eh = ((f.h - f_ref.h).norm() / f_ref.h.norm()).item()
    assert ey < 1e-2 and eh < 1e-2, (ey, eh)
