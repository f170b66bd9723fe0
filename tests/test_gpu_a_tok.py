"""GPU parity with a data-dependent A_t (one fp32 value per token-head,
M3_FLAG_A_PER_TOKEN) against the fp64 oracle: tensor-core and SIMT prefill,
split sequences, decode steps, and the full-size SISO workload sampled."""
import pytest
import torch

import oracle
from m3_inputs import WORKLOADS, Shape, make_prefill, make_state, make_steps
from m3_testutil import (max_rel_l2_step, KEYS, TOL_BF16, host64, max_rel_l2_state, max_rel_l2_y, oracle_scan_slices, rel_l2,
                         tol_for)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:
    m3 = None
    DEV = "cpu"


def check(shape, algo, with_init):
    inp = {k: v.to(DEV) for k, v in make_prefill(shape, a_per_token=True).items()}
    assert inp["A"].shape == (shape.batch, shape.seqlen, shape.nheads)
    init = m3.State(*(t.to(DEV) for t in make_state(shape))) if with_init else None
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=algo)
    m3.stream_status()
    st = oracle.State(*(host64(t) for t in init)) if with_init else None
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), st)
    tol = tol_for(shape.io)
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fs.h), sr.h)
    assert ey < tol and eh < tol, f"y {ey:.3e} state {eh:.3e}"
    return ey, eh


TC_CASES = [
    (Shape(1, 300, 2, 64, 128, 1, "bf16", 91), "tc"),
    (Shape(2, 77, 2, 64, 64, 4, "bf16", 92), "tc"),
    (Shape(1, 150, 2, 64, 128, 2, "bf16", 93), "tc"),
    (Shape(1, 1100, 2, 64, 128, 1, "bf16", 94), "split3"),
    (Shape(1, 300, 2, 64, 64, 4, "bf16", 95), "split4"),
    (Shape(1, 130, 2, 64, 64, 1, "f32", 96), "simt"),
    (Shape(1, 70, 2, 64, 128, 4, "f32", 97), "simt"),
    (Shape(1, 130, 2, 64, 64, 1, "f32", 96), "tc"),
    (Shape(2, 77, 2, 64, 64, 4, "f32", 99), "tc"),
]


@pytest.mark.parametrize("shape,path", TC_CASES, ids=lambda v: v if isinstance(v, str) else
                         f"t{v.seqlen}n{v.dstate}r{v.rank}{v.io}")
@pytest.mark.parametrize("with_init", [False, True])
def test_prefill_a_per_token(shape, path, with_init):
    algo = {"tc": m3.ALGO_TC, "simt": m3.ALGO_SIMT, "split3": m3.ALGO_TC_SEGMENTS(3),
            "split4": m3.ALGO_TC_SEGMENTS(4)}[path]
    check(shape, algo, with_init)


def test_a_per_token_constant_in_time_matches_per_head():
    """A_t = A_h for every token reproduces the per-head path bit for bit."""
    s = Shape(2, 300, 2, 64, 128, 1, "bf16", 98)
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    y1, f1 = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    inp["A"] = inp["A"][None, None, :].expand(s.batch, s.seqlen, s.nheads).contiguous()
    y2, f2 = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    m3.stream_status()
    assert torch.equal(y1, y2) and torch.equal(f1.h, f2.h)


@pytest.mark.parametrize("shape", [Shape(2, 1, 3, 64, 128, 1, "bf16", 99), Shape(2, 1, 2, 64, 128, 4, "bf16", 100),
                                   Shape(1, 1, 2, 32, 64, 2, "f32", 101)], ids=lambda s: f"n{s.dstate}r{s.rank}{s.io}")
def test_decode_a_per_token(shape):
    """Prefill with A_t, then decode steps with their own A_t: equals the
    oracle's scan followed by its steps."""
    pre = {k: v.to(DEV) for k, v in make_prefill(shape.with_(seqlen=40), a_per_token=True).items()}
    _, st = m3.scan_fwd(*(pre[k] for k in KEYS), None)
    steps = make_steps(shape, 6, device=DEV, a_per_token=True)
    ys = []
    for i in range(6):
        ys.append(m3.step(*(steps[k][i] for k in ("x", "B", "C", "dt", "lam", "theta")), steps["A"][i],
                          pre["D"], st).clone())
    m3.stream_status()
    _, ost = oracle.scan(*(host64(pre[k]) for k in KEYS))
    tol = tol_for(shape.io)
    for i in range(6):
        args = [host64(steps[k][i]) for k in ("x", "B", "C", "dt", "lam", "theta")]
        yo, ost = oracle.step(*args, host64(steps["A"][i]), host64(pre["D"]), ost)
        assert max_rel_l2_step(host64(ys[i]), yo) < tol, f"step {i} (worst slice)"
    assert max_rel_l2_state(host64(st.h), ost.h) < tol


def test_full_size_siso_a_per_token_sampled():
    shape = WORKLOADS["siso_bf16_b8_t4096_h32_p64_n128"]
    inp = make_prefill(shape, device=DEV, a_per_token=True)
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    m3.stream_status()
    picks = [(0, 0), (3, 17), (7, 31)]
    ref = oracle_scan_slices(inp, picks)
    for (b, h), (yr, hr, _, _) in ref.items():
        assert rel_l2(host64(y[b, :, h]), yr) < TOL_BF16
        assert rel_l2(host64(fs.h[b, h]), hr) < TOL_BF16
