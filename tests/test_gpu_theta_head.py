"""GPU parity with the angle rates fixed per head (theta [H, N/2],
M3_FLAG_THETA_PER_HEAD) against the fp64 oracle: tensor-core and SIMT
prefill, split sequences, decode steps, combined with a data-dependent A_t,
and the full-size SISO workload sampled."""
import pytest
import torch

import oracle
from m3_inputs import WORKLOADS, Shape, make_prefill, make_state, make_steps
from m3_testutil import max_rel_l2_step, KEYS, TOL_BF16, host64, max_rel_l2_state, max_rel_l2_y, oracle_scan_slices, rel_l2, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:
    m3 = None
    DEV = "cpu"


def check(shape, algo, with_init, a_per_token=False):
    inp = {k: v.to(DEV) for k, v in make_prefill(shape, a_per_token=a_per_token, theta_per_head=True).items()}
    assert inp["theta"].shape == (shape.nheads, shape.dstate // 2)
    init = m3.State(*(t.to(DEV) for t in make_state(shape))) if with_init else None
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=algo)
    m3.stream_status()
    st = oracle.State(*(host64(t) for t in init)) if with_init else None
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), st)
    tol = tol_for(shape.io)
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fs.h), sr.h)
    assert ey < tol and eh < tol, f"y {ey:.3e} state {eh:.3e}"


CASES = [
    (Shape(1, 300, 2, 64, 128, 1, "bf16", 111), "tc"),
    (Shape(2, 77, 2, 64, 64, 4, "bf16", 112), "tc"),
    (Shape(1, 150, 2, 64, 128, 2, "bf16", 113), "tc"),
    (Shape(1, 1100, 2, 64, 128, 1, "bf16", 114), "split3"),
    (Shape(1, 130, 2, 64, 64, 1, "f32", 115), "simt"),
    (Shape(1, 70, 2, 64, 128, 4, "f32", 116), "simt"),
    (Shape(1, 130, 2, 64, 64, 1, "f32", 115), "tc"),
    (Shape(2, 77, 2, 64, 64, 4, "f32", 119), "tc"),
]


@pytest.mark.parametrize("shape,path", CASES, ids=lambda v: v if isinstance(v, str) else
                         f"t{v.seqlen}n{v.dstate}r{v.rank}{v.io}")
@pytest.mark.parametrize("with_init", [False, True])
@pytest.mark.parametrize("a_per_token", [False, True], ids=["A_head", "A_tok"])
def test_prefill_theta_per_head(shape, path, with_init, a_per_token):
    algo = {"tc": m3.ALGO_TC, "simt": m3.ALGO_SIMT, "split3": m3.ALGO_TC_SEGMENTS(3)}[path]
    check(shape, algo, with_init, a_per_token)


def test_theta_per_head_close_to_broadcast_per_token():
    """Same method with theta repeated over tokens (angles summed per token
    instead of taken as theta_k times the cumulative dt): agreement far
    inside the bar against the oracle."""
    s = Shape(2, 700, 2, 64, 128, 1, "bf16", 117)
    inp = {k: v.to(DEV) for k, v in make_prefill(s, theta_per_head=True).items()}
    y1, f1 = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    inp["theta"] = inp["theta"][None, None].expand(s.batch, s.seqlen, s.nheads, s.dstate // 2).contiguous()
    y2, f2 = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    m3.stream_status()
    assert max_rel_l2_y(host64(y1), host64(y2)) < 5e-3
    assert max_rel_l2_state(host64(f1.h), host64(f2.h)) < 5e-3


@pytest.mark.parametrize("shape", [Shape(2, 1, 3, 64, 128, 1, "bf16", 118), Shape(2, 1, 2, 64, 128, 4, "bf16", 119),
                                   Shape(1, 1, 2, 32, 64, 2, "f32", 120)], ids=lambda s: f"n{s.dstate}r{s.rank}{s.io}")
def test_decode_theta_per_head(shape):
    pre = {k: v.to(DEV) for k, v in make_prefill(shape.with_(seqlen=40), theta_per_head=True).items()}
    _, st = m3.scan_fwd(*(pre[k] for k in KEYS), None)
    steps = make_steps(shape, 5, device=DEV)
    ys = [m3.step(*(steps[k][i] for k in ("x", "B", "C", "dt", "lam")), pre["theta"], pre["A"], pre["D"], st).clone()
          for i in range(5)]
    m3.stream_status()
    _, ost = oracle.scan(*(host64(pre[k]) for k in KEYS))
    tol = tol_for(shape.io)
    for i in range(5):
        args = [host64(steps[k][i]) for k in ("x", "B", "C", "dt", "lam")]
        yo, ost = oracle.step(*args, host64(pre["theta"]), host64(pre["A"]), host64(pre["D"]), ost)
        assert max_rel_l2_step(host64(ys[i]), yo) < tol, f"step {i} (worst slice)"
    assert max_rel_l2_state(host64(st.h), ost.h) < tol


def test_full_size_siso_theta_per_head_sampled():
    shape = WORKLOADS["siso_bf16_b8_t4096_h32_p64_n128"]
    inp = make_prefill(shape, device=DEV, theta_per_head=True)
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None)
    m3.stream_status()
    picks = [(0, 0), (4, 9), (7, 31)]
    sl = dict(inp)
    # the slice helper stacks per-token tensors; give it theta repeated over tokens
    sl["theta"] = inp["theta"][None, None].expand(shape.batch, shape.seqlen, shape.nheads, -1)
    ref = oracle_scan_slices(sl, picks)
    for (b, h), (yr, hr, _, _) in ref.items():
        assert rel_l2(host64(y[b, :, h]), yr) < TOL_BF16
        assert rel_l2(host64(fs.h[b, h]), hr) < TOL_BF16
