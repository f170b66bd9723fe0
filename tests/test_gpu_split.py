"""GPU parity of the tensor-core prefill with sequences split into segments
(summary pass, then the main pass with its look-back over the published
summaries) against the fp64 oracle, and against the same path unsplit."""
import pytest
import torch

from m3_inputs import WORKLOADS, Shape, make_prefill, make_state
from m3_testutil import KEYS, host64, max_rel_l2_state, max_rel_l2_y

from test_gpu_parity import check_scan, to_dev

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:
    m3 = None
    DEV = "cpu"

# (shape, forced segment counts): chunks of 128 / R tokens, ragged tails
SPLIT_CASES = [
    (Shape(1, 1100, 2, 64, 128, 1, "bf16", 61), (2, 3, 5)),   # 9 chunks
    (Shape(1, 640, 1, 64, 128, 1, "bf16", 62), (5,)),         # one chunk per segment
    (Shape(1, 300, 2, 64, 64, 4, "bf16", 63), (3, 4)),        # MIMO, 10 chunks of 32 tokens
    (Shape(2, 333, 1, 64, 128, 2, "bf16", 64), (2, 3)),       # rank 2, 6 chunks
    (Shape(1, 520, 2, 64, 64, 1, "bf16", 65), (2,)),          # N = 64, 5 chunks
    (Shape(1, 400, 1, 64, 128, 4, "bf16", 66), (13,)),        # N = 128 rank 4, 13 chunks
]
PARAMS = [(s, n) for s, ns in SPLIT_CASES for n in ns]


@pytest.mark.parametrize("shape,segs", PARAMS,
                         ids=lambda v: f"b{v.batch}t{v.seqlen}h{v.nheads}n{v.dstate}r{v.rank}" if isinstance(v, Shape) else f"s{v}")
@pytest.mark.parametrize("with_init", [False, True])
def test_split_prefill_matches_oracle(shape, segs, with_init):
    dims = m3.make_dims(shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.rank,
                        shape.torch_io)
    plan = m3.scan_plan(dims, m3.ALGO_TC_SEGMENTS(segs))
    assert plan.segments == segs and plan.launches == 2 and plan.workspace_bytes > 0
    check_scan(shape, m3.ALGO_TC_SEGMENTS(segs), with_init)
    m3.stream_status()


def test_split_agrees_with_unsplit():
    """Same arithmetic except where the state enters a segment (fp32 scan of
    fp32 summaries), so far tighter than the bar against the oracle."""
    s = Shape(2, 2000, 2, 64, 128, 1, "bf16", 67)
    inp = to_dev(make_prefill(s))
    init = m3.State(*(t.to(DEV) for t in make_state(s)))
    y1, f1 = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=m3.ALGO_TC_SEGMENTS(1))
    y4, f4 = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=m3.ALGO_TC_SEGMENTS(4))
    m3.stream_status()
    assert max_rel_l2_y(host64(y4), host64(y1)) < 5e-3
    assert max_rel_l2_state(host64(f4.h), host64(f1.h)) < 5e-3
    assert torch.equal(f4.b_prev, f1.b_prev) and torch.equal(f4.x_prev, f1.x_prev)


def test_split_in_place_resume():
    """init and final_state the same buffers: the first segment's summary and
    main-pass CTAs read the caller's state, and the last segment writes the
    final state only after both have (a flag, and the look-back on the first
    summary)."""
    s = Shape(1, 1000, 2, 64, 128, 1, "bf16", 68)
    inp = to_dev(make_prefill(s))
    st = m3.State(*(t.to(DEV) for t in make_state(s)))
    ref_init = m3.State(*(t.clone() for t in st))
    y_ref, f_ref = m3.scan_fwd(*(inp[k] for k in KEYS), ref_init, algo=m3.ALGO_TC_SEGMENTS(3))
    y, f = m3.scan_fwd(*(inp[k] for k in KEYS), st, final=st, algo=m3.ALGO_TC_SEGMENTS(3))
    m3.stream_status()
    assert f.h.data_ptr() == st.h.data_ptr()
    assert torch.equal(y, y_ref)
    assert torch.equal(st.h, f_ref.h)


def test_split_workspace_too_small_is_refused():
    s = Shape(1, 1100, 1, 64, 128, 1, "bf16", 69)
    inp = to_dev(make_prefill(s))
    dims = m3.make_dims(1, s.seqlen, 1, 64, 128, 1, s.torch_io)
    need = m3.workspace_size(dims, m3.ALGO_TC_SEGMENTS(3))
    ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(m3.M3Error) as e:
        m3.scan_fwd(*(inp[k] for k in KEYS), None, workspace=ws, algo=m3.ALGO_TC_SEGMENTS(3))
    assert e.value.status == m3.M3_ERR_INVALID_ARG


def test_auto_plan_splits_only_the_few_long_sequences():
    def plan(name):
        s = WORKLOADS[name]
        return m3.scan_plan(m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io))
    long_plan = plan("long_mimo_bf16_b1_t65536_h64_p64_n128_r4")
    assert long_plan.segments > 1 and long_plan.launches == 2
    assert plan("siso_bf16_b8_t4096_h32_p64_n128") == (0, 1, 1)
    assert plan("mimo_bf16_b8_t4096_h32_p64_n64_r4").segments == 1


@pytest.mark.parametrize("shape,segs", [
    (Shape(1, 1, 2, 64, 128, 1, "bf16", 151), 4),      # one token: the plan falls back to one segment
    (Shape(1, 256, 1, 64, 128, 1, "bf16", 152), 2),    # segment boundary at the last chunk boundary
    (Shape(1, 129, 1, 64, 128, 1, "bf16", 153), 2),    # second segment holds a single token
    (Shape(3, 520, 1, 64, 64, 2, "bf16", 154), 7),     # several sequences, many short segments
], ids=lambda v: f"t{v.seqlen}b{v.batch}r{v.rank}" if isinstance(v, Shape) else f"s{v}")
def test_split_edge_cases(shape, segs):
    dims = m3.make_dims(shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.rank,
                        shape.torch_io)
    plan = m3.scan_plan(dims, m3.ALGO_TC_SEGMENTS(segs))
    nch = -(-shape.seqlen // (128 // shape.rank))
    assert 1 <= plan.segments <= min(segs, nch)
    assert plan.launches == (2 if plan.segments > 1 else 1)
    check_scan(shape, m3.ALGO_TC_SEGMENTS(segs), with_init=True)
    m3.stream_status()


def test_split_zero_batch_is_noop():
    s = Shape(0, 1000, 2, 64, 128, 1, "bf16", 155)
    inp = to_dev(make_prefill(s))
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None, algo=m3.ALGO_TC_SEGMENTS(3))
    m3.stream_status()
    assert y.numel() == 0 and fs.h.numel() == 0


def test_split_calls_on_two_streams_at_once():
    """Two split calls queued on two streams, each with its own workspace
    (flags included), run at the same time: each equals the same call made
    alone (the look-back only ever reads its own call's flags and summaries)."""
    sa = Shape(1, 1500, 2, 64, 128, 1, "bf16", 161)
    sb = Shape(2, 900, 1, 64, 64, 4, "bf16", 162)
    ia, ib = to_dev(make_prefill(sa)), to_dev(make_prefill(sb))
    alg = m3.ALGO_TC_SEGMENTS(4)
    ya_ref, fa_ref = m3.scan_fwd(*(ia[k] for k in KEYS), None, algo=alg)
    yb_ref, fb_ref = m3.scan_fwd(*(ib[k] for k in KEYS), None, algo=alg)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(3):
        with torch.cuda.stream(s1):
            ya, fa = m3.scan_fwd(*(ia[k] for k in KEYS), None, algo=alg, stream=s1)
        with torch.cuda.stream(s2):
            yb, fb = m3.scan_fwd(*(ib[k] for k in KEYS), None, algo=alg, stream=s2)
        torch.cuda.synchronize()
        m3.stream_status()
        assert torch.equal(ya, ya_ref) and torch.equal(fa.h, fa_ref.h)
        assert torch.equal(yb, yb_ref) and torch.equal(fb.h, fb_ref.h)


@pytest.mark.parametrize("shape,segs", [
    (Shape(1, 256 * 128, 1, 64, 128, 1, "bf16", 171), 256),   # one chunk per segment: 255 summaries scanned by the last
    (Shape(1, 4096, 2, 64, 64, 4, "bf16", 172), 128),          # rank 4, 32-token chunks
], ids=["n128r1s256", "n64r4s128"])
def test_split_deep_lookback(shape, segs):
    """Many one-chunk segments: the main pass of the last segment combines
    every earlier segment's summary, and the summary grid runs in more than
    one wave before the main grid has taken every SM."""
    dims = m3.make_dims(shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.rank,
                        shape.torch_io)
    plan = m3.scan_plan(dims, m3.ALGO_TC_SEGMENTS(segs))
    assert plan.segments == segs and plan.launches == 2
    check_scan(shape, m3.ALGO_TC_SEGMENTS(segs), with_init=True)
    m3.stream_status()
