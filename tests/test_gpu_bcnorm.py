"""GPU parity of the fused BC-norm prologue (RMS norm of every (token, head,
rank) row of B and C, weights, head-specific biases) against the fp64
oracle: tensor-core and SIMT prefill, split sequences, decode steps through
the tiled and the generic kernels, and the full-size SISO workload sampled."""
import pytest
import torch

import oracle
from m3_inputs import WORKLOADS, Shape, make_bcnorm, make_prefill, make_state, make_steps
from m3_testutil import max_rel_l2_step, KEYS, TOL_BF16, host64, max_rel_l2_state, max_rel_l2_y, rel_l2, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:
    m3 = None
    DEV = "cpu"


def params(shape):
    p = make_bcnorm(shape, device=DEV)
    dev = m3.BCNorm(p["wB"], p["wC"], p["bB"], p["bC"], p["eps"])
    ref = oracle.BCNorm(host64(p["wB"]), host64(p["wC"]), host64(p["bB"]), host64(p["bC"]), p["eps"])
    return dev, ref


def check(shape, algo, with_init):
    inp = {k: v.to(DEV) for k, v in make_prefill(shape).items()}
    bcn, bref = params(shape)
    init = m3.State(*(t.to(DEV) for t in make_state(shape))) if with_init else None
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=algo, bcnorm=bcn)
    m3.stream_status()
    st = oracle.State(*(host64(t) for t in init)) if with_init else None
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), st, bcnorm=bref)
    tol = tol_for(shape.io)
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fs.h), sr.h)
    assert ey < tol and eh < tol, f"y {ey:.3e} state {eh:.3e}"
    # b_prev holds the normalised B of the last token (fp32 on both sides)
    assert max_rel_l2_state(host64(fs.b_prev), sr.b_prev) < 1e-5


CASES = [
    (Shape(1, 300, 2, 64, 128, 1, "bf16", 131), "tc"),
    (Shape(2, 77, 2, 64, 64, 4, "bf16", 132), "tc"),
    (Shape(1, 150, 2, 64, 128, 2, "bf16", 133), "tc"),
    (Shape(1, 100, 2, 64, 128, 4, "bf16", 134), "tc"),
    (Shape(1, 1100, 2, 64, 128, 1, "bf16", 135), "split3"),
    (Shape(1, 130, 2, 64, 64, 1, "f32", 136), "simt"),
    (Shape(1, 70, 2, 64, 128, 4, "f32", 137), "simt"),
    (Shape(2, 37, 3, 8, 8, 1, "f32", 138), "simt"),
    (Shape(1, 130, 2, 64, 64, 1, "f32", 136), "tc"),
    (Shape(2, 77, 2, 64, 64, 2, "f32", 143), "tc"),
]


@pytest.mark.parametrize("shape,path", CASES, ids=lambda v: v if isinstance(v, str) else
                         f"t{v.seqlen}p{v.headdim}n{v.dstate}r{v.rank}{v.io}")
@pytest.mark.parametrize("with_init", [False, True])
def test_prefill_bcnorm(shape, path, with_init):
    algo = {"tc": m3.ALGO_TC, "simt": m3.ALGO_SIMT, "split3": m3.ALGO_TC_SEGMENTS(3)}[path]
    check(shape, algo, with_init)


@pytest.mark.parametrize("shape", [Shape(2, 1, 3, 64, 128, 1, "bf16", 139), Shape(2, 1, 2, 64, 128, 4, "bf16", 140),
                                   Shape(1, 1, 2, 64, 64, 2, "f32", 141), Shape(1, 1, 2, 12, 16, 3, "f32", 142)],
                         ids=lambda s: f"p{s.headdim}n{s.dstate}r{s.rank}{s.io}")
def test_decode_bcnorm(shape):
    """Prefill then decode steps, both with the prologue: equals the oracle's
    scan followed by its steps (tiled kernel; the last shape runs the
    generic one)."""
    pre = {k: v.to(DEV) for k, v in make_prefill(shape.with_(seqlen=30)).items()}
    bcn, bref = params(shape)
    _, st = m3.scan_fwd(*(pre[k] for k in KEYS), None, bcnorm=bcn)
    steps = make_steps(shape, 5, device=DEV)
    ys = [m3.step(*(steps[k][i] for k in ("x", "B", "C", "dt", "lam", "theta")), pre["A"], pre["D"], st,
                  bcnorm=bcn).clone() for i in range(5)]
    m3.stream_status()
    _, ost = oracle.scan(*(host64(pre[k]) for k in KEYS), bcnorm=bref)
    tol = tol_for(shape.io)
    for i in range(5):
        args = [host64(steps[k][i]) for k in ("x", "B", "C", "dt", "lam", "theta")]
        yo, ost = oracle.step(*args, host64(pre["A"]), host64(pre["D"]), ost, bcnorm=bref)
        assert max_rel_l2_step(host64(ys[i]), yo) < tol, f"step {i} (worst slice)"
    assert max_rel_l2_state(host64(st.h), ost.h) < tol
    assert max_rel_l2_state(host64(st.b_prev), ost.b_prev) < 1e-5


def test_bcnorm_validation():
    s = Shape(1, 16, 1, 64, 128, 1, "bf16", 143)
    inp = {k: v.to(DEV) for k, v in make_prefill(s).items()}
    bcn, _ = params(s)
    with pytest.raises(m3.M3Error) as e:
        m3.scan_fwd(*(inp[k] for k in KEYS), None, bcnorm=bcn._replace(eps=0.0))
    assert e.value.status == m3.M3_ERR_INVALID_ARG


def test_full_size_siso_bcnorm_sampled():
    shape = WORKLOADS["siso_bf16_b8_t4096_h32_p64_n128"]
    inp = make_prefill(shape, device=DEV)
    bcn, bref = params(shape)
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None, bcnorm=bcn)
    m3.stream_status()
    for b, h in [(0, 0), (5, 13), (7, 31)]:
        sl = {k: host64(inp[k][b:b + 1, :, h:h + 1]) for k in KEYS if k not in ("A", "D")}
        sl["A"], sl["D"] = host64(inp["A"][h:h + 1]), host64(inp["D"][h:h + 1])
        hb = oracle.BCNorm(bref.wB, bref.wC, bref.bB[h:h + 1], bref.bC[h:h + 1], bref.eps)
        yr, sr = oracle.scan(*(sl[k] for k in KEYS), bcnorm=hb)
        assert rel_l2(host64(y[b, :, h]), yr[0, :, 0]) < TOL_BF16
        assert rel_l2(host64(fs.h[b, h]), sr.h[0, 0]) < TOL_BF16
