"""GPU parity sweep: seeded random shapes across every prefill kernel (bf16
tensor-core, fp32 tensor-core, SIMT, split sequences) with random feature
combinations (initial state, data-dependent A_t, angle rates fixed per head,
BC-norm), each followed by decode steps, against the fp64 oracle slice by
slice (max over (batch, head) slices of the relative L2 error; 2e-2 for bf16
I/O, 1e-4 for fp32 I/O).  The shapes are drawn once from a fixed seed, so
the cases are the same on every run; the plan query names the kernel each
case runs, and the test checks it is the one the case is meant for."""
import random

import pytest
import torch

import oracle
from m3_inputs import Shape, make_bcnorm, make_prefill, make_state, make_steps
from m3_testutil import KEYS, host64, max_rel_l2_state, max_rel_l2_step, max_rel_l2_y, record_margin, tol_for

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import state_space_sequence_ssm_b200 as m3
    DEV = "cuda"
else:  # collected on CPU only to be deselected
    m3 = None
    DEV = "cpu"

STEP_KEYS = ("x", "B", "C", "dt", "lam", "theta")


def draw_cases(n_per_kind=4, seed=20261203):
    """(name, shape, kind, features) for the kinds tc (bf16 tensor-core), tc32
    (fp32 tensor-core), simt (fp32 at sizes the tensor-core kernels do not
    take) and split (bf16 tensor-core, sequences split into segments)."""
    rng = random.Random(seed)
    cases = []
    for kind in ("tc", "tc32", "simt", "split"):
        for i in range(n_per_kind):
            if kind in ("tc", "split"):
                N, R, io = rng.choice([64, 128]), rng.choice([1, 2, 4]), "bf16"
                P = 64
            elif kind == "tc32":
                N, R, io, P = 64, rng.choice([1, 2, 4]), "f32", 64
            else:
                P, N, R, io = rng.choice([16, 32, 64]), rng.choice([16, 32, 128]), rng.choice([1, 3]), "f32"
            T = rng.randint(600, 1400) if kind == "split" else rng.randint(1, 500)
            Bt, H = rng.randint(1, 3), rng.randint(1, 3)
            feats = {"init": rng.random() < 0.5, "a_tok": rng.random() < 0.3, "th_head": rng.random() < 0.3,
                     "bcnorm": rng.random() < 0.3}
            seed_i = 9000 + len(cases)
            cases.append((f"{kind}{i}", Shape(Bt, T, H, P, N, R, io, seed_i), kind, feats))
    return cases


CASES = draw_cases()


@pytest.mark.parametrize("name,shape,kind,feats", CASES, ids=[c[0] for c in CASES])
def test_sweep_prefill_then_decode(name, shape, kind, feats):
    s = shape
    inp = {k: v.to(DEV) for k, v in make_prefill(s, a_per_token=feats["a_tok"],
                                                  theta_per_head=feats["th_head"]).items()}
    init = m3.State(*(t.to(DEV) for t in make_state(s))) if feats["init"] else None
    bcn = bref = None
    if feats["bcnorm"]:
        p = make_bcnorm(s, device=DEV)
        bcn = m3.BCNorm(p["wB"], p["wC"], p["bB"], p["bC"], p["eps"])
        bref = oracle.BCNorm(host64(p["wB"]), host64(p["wC"]), host64(p["bB"]), host64(p["bC"]), p["eps"])
    algo = {"tc": m3.ALGO_TC, "tc32": m3.ALGO_TC, "simt": m3.ALGO_AUTO, "split": m3.ALGO_TC_SEGMENTS(3)}[kind]
    dims = m3.make_dims(s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.rank, s.torch_io,
                        a_per_token=feats["a_tok"], theta_per_head=feats["th_head"])
    want = {"tc": m3.KERNEL_TC, "tc32": m3.KERNEL_TC32, "simt": m3.KERNEL_SIMT, "split": m3.KERNEL_TC}[kind]
    assert m3.scan_plan_info(dims, algo).kernel == want
    y, fs = m3.scan_fwd(*(inp[k] for k in KEYS), init, algo=algo, bcnorm=bcn)
    m3.stream_status()
    st0 = oracle.State(*(host64(t) for t in init)) if init is not None else None
    yr, sr = oracle.scan(*(host64(inp[k]) for k in KEYS), st0, bcnorm=bref)
    tol = tol_for(s.io)
    ey, eh = max_rel_l2_y(host64(y), yr), max_rel_l2_state(host64(fs.h), sr.h)
    record_margin(f"sweep {name} {s.batch}x{s.seqlen}x{s.nheads} P{s.headdim} N{s.dstate} R{s.rank} {s.io} "
                  f"{'+'.join(k for k, v in feats.items() if v) or 'plain'}", max(ey, eh), tol)
    assert ey < tol, f"y rel-L2 {ey:.3e}"
    assert eh < tol, f"state rel-L2 {eh:.3e}"
    # decode steps from the returned state (decode A per head unless the
    # prefill's A was per token, then the steps draw their own)
    nsteps = 3
    steps = make_steps(s, nsteps, a_per_token=feats["a_tok"])
    ost = sr
    worst = 0.0
    for i in range(nsteps):
        args = [steps[k][i].contiguous().to(DEV) for k in STEP_KEYS[:5]]
        # angle rates fixed per head: the decode takes the prefill's [H, N/2]
        th_i = inp["theta"] if feats["th_head"] else steps["theta"][i].contiguous().to(DEV)
        Ai = steps["A"][i].contiguous().to(DEV) if feats["a_tok"] else inp["A"]
        yi = m3.step(*args, th_i, Ai, inp["D"], fs, bcnorm=bcn).clone()
        m3.stream_status()
        yo, ost = oracle.step(*(host64(a) for a in args), host64(th_i), host64(Ai), host64(inp["D"]), ost,
                              bcnorm=bref)
        worst = max(worst, max_rel_l2_step(host64(yi), yo))
    assert worst < tol, f"decode rel-L2 {worst:.3e}"
    assert max_rel_l2_state(host64(fs.h), ost.h) < tol
