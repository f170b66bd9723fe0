"""Failure detection on the GPU without a fault: a bounded device wait that is
made to give up must surface as M3_ERR_TIMEOUT through m3_stream_status, be
cleared by that call, and leave the context usable."""
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
