"""Failure detection on the GPU without a fault: a bounded device wait that is
made to give up -- in the self-test kernel, and in the split prefill's
look-back on a segment flag that is never published -- must surface as
M3_ERR_TIMEOUT through m3_stream_status, be cleared by that call, and leave
the context usable."""
import pytest
import torch

from m3_inputs import Shape

from test_gpu_parity import check_scan

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3


def test_bounded_wait_timeout_is_reported_and_cleared():
    m3.stream_status()  # nothing pending
    m3.selftest_wait_timeout()
    with pytest.raises(m3.M3Error) as e:
        m3.stream_status()
    assert e.value.status == m3.M3_ERR_TIMEOUT
    assert "0x10" in str(e.value)  # the self-test's own code
    m3.stream_status()  # the record was cleared


def test_context_usable_after_timeout():
    s = torch.cuda.Stream()
    m3.selftest_wait_timeout(stream=s)
    with pytest.raises(m3.M3Error):
        m3.stream_status(stream=s)
    # every prefill kernel still runs and still matches the oracle
    check_scan(Shape(1, 300, 2, 64, 128, 1, "bf16", 81), m3.ALGO_TC, with_init=True)
    check_scan(Shape(1, 300, 2, 64, 64, 2, "f32", 83), m3.ALGO_TC, with_init=True)
    check_scan(Shape(1, 100, 2, 16, 32, 2, "f32", 82), m3.ALGO_SIMT, with_init=True)
    m3.stream_status()


@pytest.mark.parametrize("shape", [Shape(1, 600, 2, 64, 128, 1, "bf16", 84), Shape(1, 300, 2, 64, 64, 4, "bf16", 85)],
                         ids=["n128r1", "n64r4"])
def test_split_lookback_timeout_is_reported_and_the_context_stays_usable(shape):
    """The split prefill without its summary pass (a test-only entry point):
    the main pass's look-back in segments 1 and 2 waits on flags that are
    never published, gives up after its bounded wait, drains and returns;
    m3_stream_status reports M3_ERR_TIMEOUT with the segment code 0x8 and
    clears it.  Segment 0 needs no look-back, so its part of y is still
    right.  Afterwards the same split call with its summary pass matches the
    oracle on the same context."""
    import oracle
    from m3_inputs import make_prefill, make_state
    from m3_testutil import KEYS, TOL_BF16, host64, max_rel_l2_y
    s = shape
    inp = {k: v.cuda() for k, v in make_prefill(s).items()}
    init = m3.State(*(t.cuda() for t in make_state(s)))
    m3.stream_status()  # nothing pending
    y, _ = m3.selftest_segment_timeout(*(inp[k] for k in KEYS), segments=3, init=init)
    with pytest.raises(m3.M3Error) as e:
        m3.stream_status()
    assert e.value.status == m3.M3_ERR_TIMEOUT
    assert "0x8" in str(e.value)
    m3.stream_status()  # cleared
    Q = 128 // s.rank
    nch = -(-s.seqlen // Q)
    t0 = -(-nch // 3) * Q  # tokens of segment 0
    yr, _ = oracle.scan(*(host64(inp[k]) for k in KEYS), oracle.State(*(host64(t) for t in init)))
    assert max_rel_l2_y(host64(y)[:, :t0], yr[:, :t0]) < TOL_BF16
    check_scan(s, m3.ALGO_TC_SEGMENTS(3), with_init=True)
    m3.stream_status()
