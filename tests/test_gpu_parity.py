"""GPU parity: the CUDA kernels (through the C ABI) against the fp64 oracle
on the same seeded inputs.  Metric: per (batch, head) slice, relative L2
error over (t, r, p); max over slices.  Bars: 1e-4 for fp32 I/O, 2e-2 for
bf16 I/O (fp32 state)."""
import numpy as np
import pytest
import torch

import oracle
from m3_inputs import WORKLOADS, Shape, make_prefill, make_state, make_steps
from m3_testutil import (KEYS, TOL_BF16, TOL_F32, host64, max_rel_l2_state, max_rel_l2_step, max_rel_l2_y,
                         oracle_scan_slices, record_margin, rel_l2, tol_for)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:  # collected on CPU only to be deselected
    m3 = None
    DEV = "cpu"


def to_dev(d):
    return {k: v.to(DEV) for k, v in d.items()}


def oracle_full(inp, init=None):
    st = None
    if init is not None:
        st = oracle.State(*(host64(t) for t in init))
    y, fs = oracle.scan(*(host64(inp[k]) for k in KEYS), st)
    return y, fs


def check_scan(shape: Shape, algo, with_init=True, tol=None):
    inp = to_dev(make_prefill(shape))
    init = m3.State(*(t.to(DEV) for t in make_state(shape))) if with_init else None
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=algo)
    torch.cuda.synchronize()
    yref, sref = oracle_full(inp, init)
    tol = tol or tol_for(shape.io)
    ey = max_rel_l2_y(host64(y), yref)
    eh = max_rel_l2_state(host64(fs.h), sref.h)
    assert ey < tol, f"y rel-L2 {ey:.3e} >= {tol}"
    assert eh < tol, f"state rel-L2 {eh:.3e} >= {tol}"
    # the pending inputs are copied, not computed: exact up to the io rounding
    np.testing.assert_array_equal(host64(fs.b_prev), sref.b_prev)
    np.testing.assert_array_equal(host64(fs.x_prev), sref.x_prev)
    return ey, eh


SMALL = [
    Shape(2, 37, 3, 8, 8, 1, "f32", 1),
    Shape(1, 100, 2, 16, 32, 2, "f32", 2),
    Shape(2, 130, 2, 64, 64, 1, "f32", 3),      # several chunks + ragged tail
    Shape(1, 70, 2, 64, 128, 4, "f32", 4),
    Shape(1, 1, 2, 64, 64, 1, "f32", 5),        # single token
    Shape(1, 65, 1, 64, 128, 1, "bf16", 6),
    Shape(2, 200, 2, 64, 64, 4, "bf16", 7),
    Shape(1, 33, 2, 128, 64, 2, "bf16", 8),
    Shape(1, 19, 1, 4, 256, 3, "f32", 9),       # largest state, odd rank
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: f"b{s.batch}t{s.seqlen}h{s.nheads}p{s.headdim}n{s.dstate}r{s.rank}{s.io}")
@pytest.mark.parametrize("with_init", [False, True])
def test_simt_prefill_matches_oracle(shape, with_init):
    check_scan(shape, m3.ALGO_SIMT, with_init)


def test_simt_prefill_siso_f32_workload():
    """The small fp32 SISO workload (batch 1, T=256, 4 heads, P=N=64) at 1e-4."""
    ey, eh = check_scan(WORKLOADS["siso_f32_b1_t256_h4_p64_n64"], m3.ALGO_AUTO, with_init=False, tol=TOL_F32)


def test_empty_sequence_copies_initial_state():
    s = Shape(2, 0, 3, 64, 64, 2, "bf16")
    inp = to_dev(make_prefill(s))
    init = m3.State(*(t.to(DEV) for t in make_state(s)))
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init)
    for a, b in zip(fs, init):
        assert torch.equal(a, b)
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    for a in fs:
        assert torch.count_nonzero(a) == 0


def test_zero_batch_is_noop():
    s = Shape(0, 16, 2, 64, 64, 1, "bf16")
    inp = to_dev(make_prefill(s))
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    assert y.numel() == 0


def test_in_place_resume():
    """init and final_state may be the very same buffers."""
    s = Shape(2, 50, 2, 64, 64, 1, "f32", 11)
    inp = to_dev(make_prefill(s))
    st = m3.State(*(t.to(DEV) for t in make_state(s)))
    ref_init = [t.clone() for t in st]
    y, _ = m3.scan_fwd(*(inp[k] for k in KEYS), st, final=st)
    yref, sref = oracle_full(inp, ref_init)
    assert max_rel_l2_y(host64(y), yref) < TOL_F32
    assert max_rel_l2_state(host64(st.h), sref.h) < TOL_F32


# ------------------------------------------------------------------ decode step
DECODE = [
    Shape(3, 1, 2, 64, 128, 1, "bf16", 21),
    Shape(3, 1, 2, 64, 128, 4, "bf16", 22),
    Shape(2, 1, 3, 64, 64, 2, "f32", 23),
    Shape(2, 1, 2, 128, 128, 1, "f32", 24),
    Shape(2, 1, 2, 64, 256, 4, "bf16", 25),
    Shape(5, 1, 32, 64, 64, 2, "f32", 28),      # 160 slices: the persistent kernel, fp32 I/O
    Shape(5, 1, 32, 64, 128, 1, "f32", 29),     # 160 slices: one CTA per slice, fp32 I/O
    Shape(1, 1, 1, 64, 128, 2, "bf16", 30),     # one slice: the persistent kernel, one CTA
    Shape(2, 1, 2, 12, 10, 3, "f32", 26),       # generic kernel
    Shape(1, 1, 2, 2, 6, 1, "f32", 27),         # generic kernel, tiny head
]


@pytest.mark.parametrize("shape", DECODE, ids=lambda s: f"b{s.batch}h{s.nheads}p{s.headdim}n{s.dstate}r{s.rank}{s.io}")
def test_decode_steps_match_oracle(shape):
    nsteps = 5
    st_host = make_state(shape)
    st = m3.State(*(t.to(DEV).clone() for t in st_host))
    steps = to_dev(make_steps(shape, nsteps))
    A = make_prefill(shape)["A"].to(DEV)
    D = make_prefill(shape)["D"].to(DEV)
    ost = oracle.State(*(host64(t) for t in st_host))
    tol = tol_for(shape.io)
    for i in range(nsteps):
        # fresh allocations: per-step slices of odd-sized tensors need not be 16-byte aligned
        args = [steps[k][i].clone() for k in ("x", "B", "C", "dt", "lam", "theta")]
        y = m3.step(*args, A, D, st)
        yref, ost = oracle.step(*(host64(a) for a in args), host64(A), host64(D), ost)
        torch.cuda.synchronize()
        e = max_rel_l2_step(host64(y), yref)
        assert e < tol, f"step {i}: y rel-L2 {e:.3e} (worst slice)"
    assert max_rel_l2_state(host64(st.h), ost.h) < tol
    np.testing.assert_array_equal(host64(st.b_prev), ost.b_prev)
    np.testing.assert_array_equal(host64(st.x_prev), ost.x_prev)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_prefill_then_decode_equals_full_scan(io):
    """scan(T1) then k decode steps equals one scan over T1 + k tokens."""
    s = Shape(2, 48, 2, 64, 64, 2, io, 31)
    full = to_dev(make_prefill(s))
    T1 = 40
    part = {k: (v[:, :T1].contiguous() if v.dim() >= 3 else v) for k, v in full.items()}
    yfull, sfull = m3.scan_fwd(*(full[k] for k in KEYS), None)
    y1, st = m3.scan_fwd(*(part[k] for k in KEYS), None)
    ys = [y1]
    for t in range(T1, s.seqlen):
        args = [full[k][:, t].contiguous() for k in ("x", "B", "C", "dt", "lam", "theta")]
        ys.append(m3.step(*args, full["A"], full["D"], st)[:, None])
    ycat = torch.cat(ys, 1)
    yref, sref = oracle_full(full)
    tol = tol_for(io)
    assert max_rel_l2_y(host64(ycat), yref) < tol
    assert max_rel_l2_y(host64(yfull), yref) < tol
    assert max_rel_l2_state(host64(st.h), sref.h) < tol
    assert max_rel_l2_state(host64(sfull.h), sref.h) < tol


# ------------------------------------------------------------------ full-size workloads, sampled
def sampled_slices(shape: Shape, n: int, seed: int = 0):
    rng = np.random.default_rng(seed)
    BH = shape.batch * shape.nheads
    picks = sorted(set([0, BH - 1] + list(rng.choice(BH, size=min(n, BH), replace=False))))
    return [(int(i) // shape.nheads, int(i) % shape.nheads) for i in picks][:n + 2]


def check_full_prefill(name, algo, nslices):
    shape = WORKLOADS[name]
    inp = make_prefill(shape, device=DEV)
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None, algo=algo)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    picks = sampled_slices(shape, nslices)
    ref = oracle_scan_slices(inp, picks)
    tol = tol_for(shape.io)
    worst = 0.0
    for (b, h), (yr, hr, bpr, xpr) in ref.items():
        ey = rel_l2(host64(y[b, :, h]), yr)
        eh = rel_l2(host64(fs.h[b, h]), hr)
        worst = max(worst, ey, eh)
        assert ey < tol and eh < tol, f"slice ({b},{h}): y {ey:.3e} state {eh:.3e}"
        np.testing.assert_array_equal(host64(fs.b_prev[b, h]), bpr)
    record_margin(f"full-size prefill {name} ({len(picks)} slices)", worst, tol)
    return worst


@pytest.mark.parametrize("name,nslices", [
    ("siso_bf16_b8_t4096_h32_p64_n128", 6),
    ("mimo_bf16_b8_t4096_h32_p64_n64_r4", 4),
    ("long_mimo_bf16_b1_t65536_h64_p64_n128_r4", 2),
])
def test_full_size_prefill_sampled(name, nslices):
    check_full_prefill(name, m3.ALGO_AUTO, nslices)


@pytest.mark.parametrize("name,nsteps,nslices", [
    ("decode_bf16_b256_h32_p64_n128_r1", 1000, 3),
    ("decode_bf16_b256_h32_p64_n128_r4", 1000, 3),
    ("long_mimo_bf16_b1_t65536_h64_p64_n128_r4", 256, 1),
])
def test_full_size_decode_sampled(name, nsteps, nslices):
    """The workload's prefill (1024 tokens; 65,536 for the long-context
    one), then its decode steps on every slice; sampled slices checked against
    the oracle's prefill + steps."""
    DECODE_STEPS = nsteps
    shape = WORKLOADS[name]
    inp = make_prefill(shape, device=DEV)
    _, st = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    steps = make_steps(shape, DECODE_STEPS, device=DEV)
    picks = sampled_slices(shape, nslices)
    bi = torch.tensor([b for b, _ in picks], device=DEV)
    hi = torch.tensor([h for _, h in picks], device=DEV)
    ys = []
    y = torch.empty(shape.batch, shape.nheads, shape.rank, shape.headdim, dtype=shape.torch_io, device=DEV)
    for i in range(DECODE_STEPS):
        m3.step(*(steps[k][i] for k in ("x", "B", "C", "dt", "lam", "theta")), inp["A"], inp["D"], st, y=y)
        ys.append(y[bi, hi].clone())
    torch.cuda.synchronize()
    ygpu = host64(torch.stack(ys, 1))  # [picks, steps, R, P]
    ref = oracle_scan_slices(inp, picks)
    tol = TOL_BF16
    worst = 0.0
    for j, (b, h) in enumerate(picks):
        _, hr, bpr, xpr = ref[(b, h)]
        ost = oracle.State(hr[None, None], bpr[None, None], xpr[None, None])
        yref = []
        for i in range(DECODE_STEPS):
            args = [host64(steps[k][i][b:b + 1, h:h + 1]) for k in ("x", "B", "C", "dt", "lam", "theta")]
            yo, ost = oracle.step(*args, host64(inp["A"][h:h + 1]), host64(inp["D"][h:h + 1]), ost)
            yref.append(yo[0, 0])
        e = rel_l2(ygpu[j], np.stack(yref))
        assert e < tol, f"slice ({b},{h}) decode y rel-L2 {e:.3e}"
        eh = rel_l2(host64(st.h[b, h]), ost.h[0, 0])
        assert eh < tol, f"slice ({b},{h}) state rel-L2 {eh:.3e}"
        worst = max(worst, e, eh)
    record_margin(f"full-size decode {name}, {nsteps} steps ({len(picks)} slices)", worst, tol)


# ------------------------------------------------------------------ tensor-core prefill
TC_SHAPES = [
    Shape(1, 128, 1, 64, 128, 1, "bf16", 41),   # exactly one chunk
    Shape(1, 300, 2, 64, 128, 1, "bf16", 42),   # three chunks, ragged tail
    Shape(2, 77, 2, 64, 64, 4, "bf16", 43),     # MIMO: 32 tokens x 4 ranks per chunk
    Shape(1, 200, 2, 64, 64, 1, "bf16", 44),
    Shape(1, 100, 2, 64, 128, 4, "bf16", 45),
    Shape(1, 150, 2, 64, 128, 2, "bf16", 46),
    Shape(1, 90, 1, 64, 64, 2, "bf16", 47),
    Shape(1, 1, 1, 64, 128, 1, "bf16", 48),     # single token
    Shape(3, 513, 3, 64, 128, 1, "bf16", 49),   # batch x heads grid, many chunks
]


@pytest.mark.parametrize("shape", TC_SHAPES, ids=lambda s: f"b{s.batch}t{s.seqlen}h{s.nheads}n{s.dstate}r{s.rank}")
@pytest.mark.parametrize("with_init", [False, True])
def test_tc_prefill_matches_oracle(shape, with_init):
    check_scan(shape, m3.ALGO_TC, with_init)
    m3.stream_status()


def test_tc_agrees_with_simt():
    """The two CUDA paths agree with each other far tighter than either's
    bar against the oracle (same algorithm, different operand precision)."""
    s = Shape(2, 700, 4, 64, 128, 1, "bf16", 50)
    inp = to_dev(make_prefill(s))
    init = m3.State(*(t.to(DEV) for t in make_state(s)))
    y1, f1 = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=m3.ALGO_TC)
    y2, f2 = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=m3.ALGO_SIMT)
    m3.stream_status()
    assert max_rel_l2_y(host64(y1), host64(y2)) < 1e-2
    assert max_rel_l2_state(host64(f1.h), host64(f2.h)) < 1e-2


def test_tc_is_the_default_for_bf16():
    s = WORKLOADS["siso_bf16_b8_t4096_h32_p64_n128"]
    dims = m3.make_dims(s.batch, 16, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io)
    inp = to_dev(make_prefill(s.with_(seqlen=16, batch=1)))
    y_auto, _ = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    y_tc, _ = m3.scan_fwd(*(inp[k] for k in KEYS), None, algo=m3.ALGO_TC)
    assert torch.equal(y_auto, y_tc)
