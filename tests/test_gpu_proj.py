"""GPU parity of the fused MIMO projections (m3_scan_fwd_proj, m3_step_proj)
against the fp64 oracle's scan_proj and step_proj, slice by slice at the
bf16 bar (max over (batch, head) slices of the relative L2 error below 2e-2):
x, B, C and y with one row per token-head, widened to rank R on chip by
per-head, per-rank weights; chunk sizes, ragged tails, initial states, split
sequences, the per-token A and per-head theta layouts, decode steps that
continue the prefill, and the refusals."""
import numpy as np
import pytest
import torch

import oracle
from m3_inputs import Shape, make_prefill_proj, make_proj, make_state, make_steps_proj
from m3_testutil import KEYS, TOL_BF16, host64, max_rel_l2_state, record_margin

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:  # collected on CPU only to be deselected
    m3 = None
    DEV = "cpu"

STEP_KEYS = ("x", "B", "C", "dt", "lam", "theta")


def rel_slices(y, yref):
    """y, yref [Bt, T, H, P] (or [Bt, H, P]): per (b, h) slice relative L2, max."""
    if y.ndim == 3:
        y, yref = y[:, None], yref[:, None]
    d = (y - yref).transpose(0, 2, 1, 3).reshape(y.shape[0] * y.shape[2], -1)
    r = yref.transpose(0, 2, 1, 3).reshape(d.shape)
    return float(np.max(np.linalg.norm(d, axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-30)))


def weights(s):
    w = make_proj(s, device=DEV)
    return m3.MimoProj(w["wx"], w["wB"], w["wC"], w["wy"]), oracle.MimoProj(*(host64(w[k]) for k in ("wx", "wB", "wC", "wy")))


def run_and_check(s, algo=None, with_init=True, a_tok=False, th_head=False, name=""):
    inp = {k: v.to(DEV) for k, v in make_prefill_proj(s, a_per_token=a_tok, theta_per_head=th_head).items()}
    pr, opr = weights(s)
    init = m3.State(*(t.to(DEV) for t in make_state(s))) if with_init else None
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=algo if algo is not None else m3.ALGO_AUTO, proj=pr)
    m3.stream_status()
    st = oracle.State(*(host64(t) for t in init)) if with_init else None
    yr, sr = oracle.scan_proj(*(host64(inp[k]) for k in KEYS), opr, st)
    assert y.shape == (s.batch, s.seqlen, s.nheads, s.headdim)
    ey, eh = rel_slices(host64(y), yr), max_rel_l2_state(host64(fs.h), sr.h)
    record_margin(f"proj {name or s}", max(ey, eh), TOL_BF16)
    assert ey < TOL_BF16, f"y rel-L2 {ey:.3e}"
    assert eh < TOL_BF16, f"state rel-L2 {eh:.3e}"
    # the pending term: the last token's row times the fp32 weights, in fp32
    assert max_rel_l2_state(host64(fs.b_prev), sr.b_prev) < 1e-6
    assert max_rel_l2_state(host64(fs.x_prev), sr.x_prev) < 1e-6
    return inp, pr, opr, fs, sr


CASES = [
    Shape(2, 100, 2, 64, 128, 4, "bf16", 501),   # 4 chunks of 32 tokens, ragged tail
    Shape(1, 300, 3, 64, 64, 4, "bf16", 502),
    Shape(2, 257, 2, 64, 128, 2, "bf16", 503),   # 64-token chunks, 1-token tail
    Shape(1, 33, 2, 64, 64, 2, "bf16", 504),     # one partial chunk
    Shape(1, 200, 2, 64, 128, 1, "bf16", 505),   # rank 1: the projections scale x, B, C and y
    Shape(2, 130, 2, 64, 64, 1, "bf16", 506),
    Shape(1, 1, 2, 64, 128, 4, "bf16", 507),     # a single token
]


@pytest.mark.parametrize("shape", CASES, ids=lambda s: f"b{s.batch}t{s.seqlen}h{s.nheads}n{s.dstate}r{s.rank}")
@pytest.mark.parametrize("with_init", [False, True])
def test_proj_prefill_matches_oracle(shape, with_init):
    info = m3.scan_plan_info(m3.make_dims(shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate,
                                          shape.rank, shape.torch_io))
    assert info.kernel == m3.KERNEL_TC
    run_and_check(shape, with_init=with_init, name=f"t{shape.seqlen} n{shape.dstate} r{shape.rank} init={with_init}")


@pytest.mark.parametrize("shape,segs", [(Shape(1, 1000, 2, 64, 128, 4, "bf16", 510), 3),
                                        (Shape(2, 700, 1, 64, 64, 2, "bf16", 511), 4)],
                         ids=["n128r4s3", "n64r2s4"])
def test_proj_split_sequences(shape, segs):
    run_and_check(shape, m3.ALGO_TC_SEGMENTS(segs), name=f"split s{segs} n{shape.dstate} r{shape.rank}")


@pytest.mark.parametrize("a_tok,th_head", [(True, False), (False, True)], ids=["a_tok", "theta_head"])
def test_proj_with_optional_layouts(a_tok, th_head):
    run_and_check(Shape(1, 160, 2, 64, 128, 4, "bf16", 512), a_tok=a_tok, th_head=th_head,
                  name=f"a_tok={a_tok} theta_head={th_head}")


@pytest.mark.parametrize("shape", [Shape(2, 70, 3, 64, 128, 4, "bf16", 520), Shape(1, 40, 2, 64, 64, 2, "bf16", 521)],
                         ids=["n128r4", "n64r2"])
def test_proj_decode_continues_the_prefill(shape):
    """Prefill with the projections, then 3 decode steps with them, against
    the oracle's scan_proj followed by step_proj."""
    inp, pr, opr, fs, sr = run_and_check(shape, with_init=True, name=f"decode base n{shape.dstate} r{shape.rank}")
    steps = make_steps_proj(shape, 3)
    ost = sr
    worst = 0.0
    for i in range(3):
        args = [steps[k][i].contiguous().to(DEV) for k in STEP_KEYS]
        yi = m3.step(*args, inp["A"], inp["D"], fs, proj=pr).clone()
        m3.stream_status()
        assert yi.shape == (shape.batch, shape.nheads, shape.headdim)
        yo, ost = oracle.step_proj(*(host64(a) for a in args), host64(inp["A"]), host64(inp["D"]), opr, ost)
        worst = max(worst, rel_slices(host64(yi), yo))
    record_margin(f"proj decode n{shape.dstate} r{shape.rank}", worst, TOL_BF16)
    assert worst < TOL_BF16, f"decode rel-L2 {worst:.3e}"
    assert max_rel_l2_state(host64(fs.h), ost.h) < TOL_BF16


def test_proj_decode_many_slices_streaming():
    """Rank 4 with more slices than the persistent streaming decode kernel has
    CTAs (each CTA walks several slices through its two-stage copy ring), from
    a random rank-4 state, two steps, against the oracle's step_proj."""
    s = Shape(96, 1, 8, 64, 128, 4, "bf16", 525)
    pr, opr = weights(s)
    st = m3.State(*(t.to(DEV) for t in make_state(s)))
    ost = oracle.State(*(host64(t) for t in st))
    pre = make_prefill_proj(s)
    A, D = pre["A"].to(DEV), pre["D"].to(DEV)
    steps = make_steps_proj(s, 2)
    worst = 0.0
    for i in range(2):
        args = [steps[k][i].contiguous().to(DEV) for k in STEP_KEYS]
        yi = m3.step(*args, A, D, st, proj=pr).clone()
        m3.stream_status()
        yo, ost = oracle.step_proj(*(host64(a) for a in args), host64(A), host64(D), opr, ost)
        worst = max(worst, rel_slices(host64(yi), yo))
    record_margin("proj decode 768 slices r4 (streaming)", worst, TOL_BF16)
    assert worst < TOL_BF16, f"decode rel-L2 {worst:.3e}"
    assert max_rel_l2_state(host64(st.h), ost.h) < TOL_BF16
    assert max_rel_l2_state(host64(st.b_prev), ost.b_prev) < 1e-6
    assert max_rel_l2_state(host64(st.x_prev), ost.x_prev) < 1e-6


def test_proj_full_size_sampled():
    """The MIMO workload's shape (batch 8, 4096 tokens, 32 heads, N 64, R 4)
    with the projections; the oracle recomputes two of its sequences' first
    two heads in full (the other slices are checked finite)."""
    s = Shape(8, 4096, 32, 64, 64, 4, "bf16", 530)
    inp = {k: v.to(DEV) for k, v in make_prefill_proj(s, device=DEV).items()}
    pr, opr = weights(s)
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), None, proj=pr)
    m3.stream_status()
    assert torch.isfinite(y.float()).all()
    for b in (0, 5):
        sub = {k: (v[b:b + 1, :, :2] if v.dim() >= 3 else v[:2]) for k, v in inp.items()}
        osub = oracle.MimoProj(*(w[:2] for w in (opr.wx, opr.wB, opr.wC, opr.wy)))
        yr, sr = oracle.scan_proj(*(host64(sub[k]) for k in KEYS), osub)
        ey = rel_slices(host64(y[b:b + 1, :, :2]), yr)
        eh = max_rel_l2_state(host64(fs.h[b:b + 1, :2]), sr.h)
        record_margin(f"proj full size b{b} h0-1", max(ey, eh), TOL_BF16)
        assert ey < TOL_BF16 and eh < TOL_BF16, (ey, eh)


def test_proj_refusals():
    s = Shape(1, 50, 2, 64, 64, 2, "bf16", 540)
    inp = {k: v.to(DEV) for k, v in make_prefill_proj(s).items()}
    pr, _ = weights(s)
    with pytest.raises(m3.M3Error) as e:  # the SIMT kernel has no projections
        m3.scan_fwd(*(inp[k] for k in KEYS), None, algo=m3.ALGO_SIMT, proj=pr)
    assert e.value.status == m3.M3_ERR_UNSUPPORTED
    f32 = {k: (v.float() if v.dtype == torch.bfloat16 else v) for k, v in inp.items()}
    with pytest.raises(m3.M3Error) as e:  # fp32 I/O
        m3.scan_fwd(*(f32[k] for k in KEYS), None, proj=pr)
    assert e.value.status == m3.M3_ERR_UNSUPPORTED
    bad = s.with_(headdim=32)  # the tensor-core prefill's sizes only
    inb = {k: v.to(DEV) for k, v in make_prefill_proj(bad).items()}
    prb, _ = weights(bad)
    with pytest.raises(m3.M3Error) as e:
        m3.scan_fwd(*(inb[k] for k in KEYS), None, proj=prb)
    assert e.value.status == m3.M3_ERR_UNSUPPORTED
    # decode: sizes outside the register-tiled kernel (dstate 32) are refused
    small = Shape(1, 8, 2, 64, 32, 2, "bf16", 541)
    prs, _ = weights(small)
    st = m3.State(*(t.to(DEV) for t in make_state(small)))
    steps = make_steps_proj(small, 1)
    args = [steps[k][0].contiguous().to(DEV) for k in STEP_KEYS]
    pre = make_prefill_proj(small)
    with pytest.raises(m3.M3Error) as e:
        m3.step(*args, pre["A"].to(DEV), pre["D"].to(DEV), st, proj=prs)
    assert e.value.status == m3.M3_ERR_UNSUPPORTED
    # BC-norm and the projections together are refused
    from m3_inputs import make_bcnorm
    b = make_bcnorm(s, device=DEV)
    with pytest.raises(m3.M3Error) as e:
        m3.scan_fwd(*(inp[k] for k in KEYS), None, proj=pr,
                    bcnorm=m3.BCNorm(b["wB"], b["wC"], b["bB"], b["bC"], b["eps"]))
    assert e.value.status == m3.M3_ERR_UNSUPPORTED
    m3.stream_status()
