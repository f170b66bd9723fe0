"""GPU parity of the fp32 tensor-core prefill (fp32 I/O, headdim 64, dstate
64, rank 1, 2 or 4: every chunk product on tcgen05 with its operands split
into bf16 high and low halves) against the fp64 oracle at the fp32 bar
(max over (batch, head) slices of the relative L2 error over (t, r, p) below
1e-4), slice by slice, with and without an initial state; plus the kernel
choice (ALGO_AUTO and ALGO_TC take it for these sizes, m3_scan_plan_info names
it), its refusals, and the sizes it hands to the SIMT kernel."""
import numpy as np
import pytest
import torch

import oracle
from m3_inputs import WORKLOADS, Shape, make_bcnorm, make_prefill, make_state
from m3_testutil import (KEYS, TOL_F32, host64, max_rel_l2_state, max_rel_l2_y, oracle_scan_slices,
                         record_margin, rel_l2)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:  # collected on CPU only to be deselected
    m3 = None
    DEV = "cpu"


def dims_of(s: Shape):
    return m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io)


def run_and_check(shape: Shape, algo, with_init: bool, bcnorm: bool = False, name: str = ""):
    inp = {k: v.to(DEV) for k, v in make_prefill(shape).items()}
    init = m3.State(*(t.to(DEV) for t in make_state(shape))) if with_init else None
    bcn = bref = None
    if bcnorm:
        p = make_bcnorm(shape, device=DEV)
        bcn = m3.BCNorm(p["wB"], p["wC"], p["bB"], p["bC"], p["eps"])
        bref = oracle.BCNorm(host64(p["wB"]), host64(p["wC"]), host64(p["bB"]), host64(p["bC"]), p["eps"])
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=algo, bcnorm=bcn)
    m3.stream_status()
    st = oracle.State(*(host64(t) for t in init)) if with_init else None
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), st, bcnorm=bref)
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fs.h), sr.h)
    record_margin(f"tc32 {name or shape}", max(ey, eh), TOL_F32)
    assert ey < TOL_F32, f"y rel-L2 {ey:.3e}"
    assert eh < TOL_F32, f"state rel-L2 {eh:.3e}"
    if bcnorm:  # the normalised B of the last token, fp32 on both sides
        assert max_rel_l2_state(host64(fs.b_prev), sr.b_prev) < 1e-5
    else:  # copied, not computed
        np.testing.assert_array_equal(host64(fs.b_prev), sr.b_prev)
    np.testing.assert_array_equal(host64(fs.x_prev), sr.x_prev)
    return y, fs


CASES = [
    Shape(1, 1, 2, 64, 64, 1, "f32", 301),      # a single token
    Shape(2, 37, 3, 64, 64, 1, "f32", 302),     # one partial chunk
    Shape(1, 128, 2, 64, 64, 1, "f32", 303),    # exactly one chunk
    Shape(2, 300, 2, 64, 64, 1, "f32", 304),    # several chunks and a ragged tail
    Shape(1, 64, 1, 64, 64, 2, "f32", 305),     # exactly one chunk of rank 2
    Shape(1, 200, 3, 64, 64, 2, "f32", 306),
    Shape(2, 150, 2, 64, 64, 4, "f32", 307),
    Shape(1, 33, 2, 64, 64, 4, "f32", 308),     # one chunk of 32 tokens and a 1-token tail
]


@pytest.mark.parametrize("shape", CASES, ids=lambda s: f"b{s.batch}t{s.seqlen}h{s.nheads}r{s.rank}")
@pytest.mark.parametrize("with_init", [False, True])
def test_tc32_prefill_matches_oracle(shape, with_init):
    info = m3.scan_plan_info(dims_of(shape), m3.ALGO_TC)
    assert info == m3.PlanInfo(0, m3.KERNEL_TC32, 1, 1, shape.batch * shape.nheads)
    assert info.kernel_name == "prefill_tc32_kernel"
    run_and_check(shape, m3.ALGO_TC, with_init, name=f"t{shape.seqlen} r{shape.rank} init={with_init}")


@pytest.mark.parametrize("rank", [1, 4])
def test_tc32_bcnorm(rank):
    run_and_check(Shape(2, 170, 2, 64, 64, rank, "f32", 310 + rank), m3.ALGO_TC, True, bcnorm=True,
                  name=f"bcnorm r{rank}")


def test_tc32_many_slices_long_sequences():
    """More (batch, head) slices than SMs and 16 chunks per slice: one CTA per slice, many waves."""
    s = Shape(4, 2048, 40, 64, 64, 1, "f32", 320)
    run_and_check(s, m3.ALGO_TC, True, name="b4 t2048 h40 r1")


def test_tc32_rank4_long():
    s = Shape(2, 1000, 8, 64, 64, 4, "f32", 321)
    run_and_check(s, m3.ALGO_TC, True, name="b2 t1000 h8 r4")


def test_auto_takes_tc32_and_matches_explicit_choice():
    s = Shape(2, 300, 3, 64, 64, 2, "f32", 322)
    assert m3.scan_plan_info(dims_of(s)).kernel == m3.KERNEL_TC32
    assert m3.scan_plan_info(dims_of(s), flags=m3.PLAN_STATIC).kernel == m3.KERNEL_TC32
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    init = m3.State(*(t.to(DEV) for t in make_state(s)))
    y1, f1 = m3.scan_fwd(*(inp[k] for k in KEYS), init)
    y2, f2 = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=m3.ALGO_TC)
    y3, f3 = m3.scan_fwd_static(*(inp[k] for k in KEYS), init)
    torch.cuda.synchronize()
    for a, b, c in zip((y1, *f1), (y2, *f2), (y3, *f3)):
        assert torch.equal(a, b) and torch.equal(a, c)
    # and the SIMT kernel on the same inputs agrees within both kernels' error
    y4, f4 = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=m3.ALGO_SIMT)
    assert rel_l2(host64(y4), host64(y1)) < 2 * TOL_F32


def test_sizes_outside_tc32_run_simt_or_are_refused():
    for s in (Shape(1, 100, 2, 64, 128, 1, "f32"), Shape(1, 100, 2, 32, 64, 1, "f32"),
              Shape(1, 100, 2, 64, 64, 3, "f32")):
        assert m3.scan_plan_info(dims_of(s)).kernel == m3.KERNEL_SIMT
        with pytest.raises(m3.M3Error):
            m3.scan_plan_info(dims_of(s), m3.ALGO_TC)
    s = Shape(1, 600, 2, 64, 64, 1, "f32", 323)
    with pytest.raises(m3.M3Error):  # fp32 sequences are not split
        m3.scan_plan_info(dims_of(s), m3.ALGO_TC_SEGMENTS(2))
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    with pytest.raises(m3.M3Error):
        m3.scan_fwd(*(inp[k] for k in KEYS), None, algo=m3.ALGO_TC_SEGMENTS(2))


def test_tc32_small_workload_at_fp32_bar():
    """The fp32 SISO workload (batch 1, T = 256, 4 heads, P = N = 64) runs this kernel."""
    s = WORKLOADS["siso_f32_b1_t256_h4_p64_n64"]
    assert m3.scan_plan_info(dims_of(s)).kernel == m3.KERNEL_TC32
    run_and_check(s, m3.ALGO_AUTO, False, name="siso_f32_b1_t256_h4_p64_n64")


def test_tc32_resume_equals_one_call():
    """Two calls chained through the returned state equal one call over the whole sequence."""
    s = Shape(2, 384, 2, 64, 64, 2, "f32", 324)
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    y, _ = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    cut = 150  # inside a chunk

    def part(lo, hi):
        return [inp[k][:, lo:hi].contiguous() if inp[k].dim() >= 3 and k not in ("A", "D") else inp[k] for k in KEYS]

    ya, st = m3.scan_fwd(*part(0, cut), None)
    yb, _ = m3.scan_fwd(*part(cut, s.seqlen), st)
    torch.cuda.synchronize()
    assert rel_l2(host64(torch.cat([ya, yb], dim=1)), host64(y)) < TOL_F32


@pytest.mark.parametrize("rank", [1, 4])
def test_tc32_long_weak_decay_large_angles(rank):
    """16,384 tokens with almost no decay (A = -0.002) and large angle rates:
    the carried state is rotated once per chunk for 128 (rank 1) or 512 (rank
    4) chunks and keeps nearly all of its history, so errors of the chunk
    rotation and of the split products would compound; the result must stay
    within the fp32 bar."""
    s = Shape(1, 16384, 2, 64, 64, rank, "f32", 330 + rank)
    inp = make_prefill(s)
    inp["A"] = torch.full_like(inp["A"], -0.002)
    inp["theta"] = inp["theta"] * 3.0  # |theta| up to 3 pi
    inp = {k: v.to(DEV) for k, v in inp.items()}
    init = m3.State(*(t.to(DEV) for t in make_state(s)))
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=m3.ALGO_TC)
    m3.stream_status()
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), oracle.State(*(host64(t) for t in init)))
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fs.h), sr.h)
    record_margin(f"tc32 long weak decay r{rank}", max(ey, eh), TOL_F32)
    assert ey < TOL_F32, f"y rel-L2 {ey:.3e}"
    assert eh < TOL_F32, f"state rel-L2 {eh:.3e}"
