"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a hand-derived worked example, a closed form, a special case that
reduces to the Mamba-2 recurrence, an explicit complex-diagonal recurrence,
the literal rotated-frame statement, the brute-force masked-attention dual,
and a chunked restatement.  Everything here is fp64 and CPU-only."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from m3_inputs import Shape, make_prefill, make_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
TOL = 1e-12


def rand_case(Bt=1, T=37, H=2, P=5, N=8, R=3, seed=0, init=True):
    s = Shape(Bt, T, H, P, N, R, "f32", seed)
    d = {k: v.double().numpy() for k, v in make_prefill(s).items()}
    st = None
    if init:
        h, bp, xp = (t.double().numpy() for t in make_state(s))
        st = oracle.State(h, bp, xp)
    return d, st


def run(d, st=None):
    return oracle.scan(d["x"], d["B"], d["C"], d["dt"], d["lam"], d["theta"], d["A"], d["D"], st)


def rel(a, b):
    return np.max(np.abs(a - b)) / max(1.0, np.max(np.abs(b)))


# ---------------------------------------------------------------- worked examples
@pytest.mark.parametrize("ex", json.load(open(GOLDEN))["examples"], ids=lambda e: e["name"])
def test_hand_worked_examples(ex):
    dm, inp, exp_ = ex["dims"], ex["inputs"], ex["expected"]
    T, N, P = dm["seqlen"], dm["dstate"], dm["headdim"]
    x = np.array(inp["x"]).reshape(1, T, 1, 1, P)
    B = np.array(inp["B"]).reshape(1, T, 1, 1, N)
    C = np.array(inp["C"]).reshape(1, T, 1, 1, N)
    dt = np.array(inp["dt"]).reshape(1, T, 1)
    lam = np.array(inp["lam"]).reshape(1, T, 1)
    th = np.array(inp["theta"]).reshape(1, T, 1, N // 2)
    A = np.array([inp["A"]])
    D = np.array([inp["D"]])
    st = None
    if "h0" in inp:
        st = oracle.State(np.array(inp["h0"]).reshape(1, 1, N, P),
                          np.array(inp["b_prev0"]).reshape(1, 1, 1, N),
                          np.array([inp["x_prev0"]]).reshape(1, 1, 1, P))
    y, fs = oracle.scan(x, B, C, dt, lam, th, A, D, st)
    np.testing.assert_allclose(y.reshape(-1), exp_["y"], atol=TOL, rtol=0)
    np.testing.assert_allclose(fs.h.reshape(N, P), np.array(exp_["h"]), atol=TOL, rtol=0)
    np.testing.assert_allclose(fs.b_prev.reshape(-1), exp_["b_prev"], atol=TOL, rtol=0)
    np.testing.assert_allclose(fs.x_prev.reshape(-1), [exp_["x_prev"]], atol=TOL, rtol=0)


# ---------------------------------------------------------------- closed forms
def test_single_token_closed_form():
    """T=1 from zero state: y_0 = lam_0 dt_0 (C_0^T B_0) x_0 + D x_0 (MIMO: the
    R x R block C_0^T B_0 mixes ranks)."""
    d, _ = rand_case(T=1, init=False)
    y, fs = run(d)
    gam = d["lam"] * d["dt"]                       # [1,1,H]
    CB = np.einsum("bthrn,bthsn->bthrs", d["C"], d["B"])
    ref = gam[..., None, None] * np.einsum("bthrs,bthsp->bthrp", CB, d["x"])
    ref += d["D"][None, None, :, None, None] * d["x"]
    assert rel(y, ref) < TOL
    # state after one token: gamma_0 B_0 x_0^T (the pending term of token 0 is zero)
    hs = gam[:, 0, :, None, None] * np.einsum("bhrn,bhrp->bhnp", d["B"][:, 0], d["x"][:, 0])
    assert rel(fs.h, hs) < TOL


def test_free_decay_closed_form():
    """x = 0 and no pending input: the state only decays and rotates, so
    h_t = exp(A sum dt) Rot(-sum dt*theta) h_0 in closed form."""
    d, st = rand_case(T=29)
    d["x"][:] = 0.0
    st.x_prev[:] = 0.0
    y, fs = run(d, st)
    cumdt = np.cumsum(d["dt"], axis=1)                          # [Bt,T,H]
    phi = np.cumsum(d["dt"][..., None] * d["theta"], axis=1)    # [Bt,T,H,N/2]
    decay = np.exp(cumdt * d["A"][None, None, :])
    h0 = st.h                                                   # [Bt,H,N,P]
    u, v = h0[:, None, :, 0::2, :], h0[:, None, :, 1::2, :]
    c, s = np.cos(phi)[..., None], np.sin(phi)[..., None]
    hu = decay[..., None, None] * (u * c + v * s)
    hv = decay[..., None, None] * (-u * s + v * c)
    ht = np.empty(hu.shape[:3] + (hu.shape[3] * 2, hu.shape[4]))
    ht[..., 0::2, :], ht[..., 1::2, :] = hu, hv
    ref = np.einsum("bthnp,bthrn->bthrp", ht, d["C"])
    assert rel(y, ref) < TOL
    assert rel(fs.h, ht[:, -1]) < TOL


def test_constant_input_fixed_point():
    """theta = 0 and constant (dt, lam, B, x): the state converges to
    (beta' a + gamma) B x^T / (1 - a) with a = exp(dt A)."""
    T, N, P = 400, 4, 3
    rng = np.random.default_rng(5)
    Bv, xv = rng.normal(size=N), rng.normal(size=P)
    dtv, lamv, A = 0.3, 0.3, np.array([-1.7])
    x = np.broadcast_to(xv, (1, T, 1, 1, P)).copy()
    B = np.broadcast_to(Bv, (1, T, 1, 1, N)).copy()
    C = rng.normal(size=(1, T, 1, 1, N))
    dt = np.full((1, T, 1), dtv)
    lam = np.full((1, T, 1), lamv)
    th = np.zeros((1, T, 1, N // 2))
    y, fs = oracle.scan(x, B, C, dt, lam, th, A, np.zeros(1))
    a = math.exp(dtv * A[0])
    hstar = ((1 - lamv) * dtv * a + lamv * dtv) * np.outer(Bv, xv) / (1 - a)
    assert rel(fs.h[0, 0], hstar) < 1e-10


# ---------------------------------------------------------------- special cases
def mamba2_reference(d):
    """Independent Mamba-2 (exponential-Euler, real, scalar decay) recurrence in
    the S in R^{P x N} orientation of the SSD chapter ('La dualità'):
    S_t = e^{dt A} S_{t-1} + dt x_t B_t^T, y_t = S_t C_t + D x_t."""
    x, B, C, dt, A, D = d["x"], d["B"], d["C"], d["dt"], d["A"], d["D"]
    Bt, T, H, R, P = x.shape
    N = B.shape[-1]
    y = np.zeros_like(x)
    for b in range(Bt):
        for h in range(H):
            S = np.zeros((P, N))
            for t in range(T):
                S = math.exp(dt[b, t, h] * A[h]) * S + dt[b, t, h] * x[b, t, h].T @ B[b, t, h]
                y[b, t, h] = (S @ C[b, t, h].T).T + D[h] * x[b, t, h]
    return y


@pytest.mark.parametrize("R", [1, 3])
def test_euler_real_reduces_to_mamba2(R):
    """lam = 1 (Euler) and theta = 0 (real) reduce the method to Mamba-2."""
    d, _ = rand_case(T=41, R=R, init=False)
    d["lam"][:] = 1.0
    d["theta"][:] = 0.0
    y, _ = run(d)
    assert rel(y, mamba2_reference(d)) < TOL


def test_trapezoid_half_is_average_of_endpoints():
    """lam = 1/2 is the classic trapezoid: the input integral is the average of
    the two endpoint writes, the older one carried through one decay."""
    d, _ = rand_case(T=23, R=1, init=False)
    d["lam"][:] = 0.5
    d["theta"][:] = 0.0
    y, _ = run(d)
    x, B, C, dt, A, D = d["x"], d["B"], d["C"], d["dt"], d["A"], d["D"]
    Bt, T, H, R, P = x.shape
    ref = np.zeros_like(y)
    for b in range(Bt):
        for h in range(H):
            S = np.zeros((P, B.shape[-1]))
            for t in range(T):
                a = math.exp(dt[b, t, h] * A[h])
                cur = np.outer(x[b, t, h, 0], B[b, t, h, 0])
                prev = np.outer(x[b, t - 1, h, 0], B[b, t - 1, h, 0]) if t else 0.0
                S = a * S + 0.5 * dt[b, t, h] * (a * prev + cur)
                ref[b, t, h, 0] = S @ C[b, t, h, 0] + D[h] * x[b, t, h, 0]
    assert rel(y, ref) < TOL


# ---------------------------------------------------------------- equivalent forms
def complex_diagonal_reference(d, st):
    """Complex SSM of state N/2: z_k = h_{2k} + i h_{2k+1}, transition
    exp(dt (A - i theta_k)), writes b_k x^T with b_k = B_{2k} + i B_{2k+1},
    readout Re(conj(c_k) z_k) summed over k."""
    x, B, C, dt, lam, th, A, D = (d[k] for k in ("x", "B", "C", "dt", "lam", "theta", "A", "D"))
    Bt, T, H, R, P = x.shape
    y = np.zeros_like(x)
    hT = np.zeros_like(st.h)
    for b in range(Bt):
        for h in range(H):
            z = st.h[b, h, 0::2] + 1j * st.h[b, h, 1::2]             # [N/2, P]
            bprev = st.b_prev[b, h, :, 0::2] + 1j * st.b_prev[b, h, :, 1::2]  # [R, N/2]
            xprev = st.x_prev[b, h]                                  # [R, P]
            for t in range(T):
                lt = np.exp(dt[b, t, h] * (A[h] - 1j * th[b, t, h]))  # [N/2]
                bt = B[b, t, h, :, 0::2] + 1j * B[b, t, h, :, 1::2]
                ct = C[b, t, h, :, 0::2] + 1j * C[b, t, h, :, 1::2]
                z = lt[:, None] * (z + (1 - lam[b, t, h]) * dt[b, t, h] * bprev.T @ xprev)
                z = z + lam[b, t, h] * dt[b, t, h] * bt.T @ x[b, t, h]
                y[b, t, h] = np.real(np.conj(ct) @ z) + D[h] * x[b, t, h]
                bprev, xprev = bt, x[b, t, h]
            hT[b, h, 0::2], hT[b, h, 1::2] = z.real, z.imag
    return y, hT


def test_equals_complex_diagonal_ssm():
    d, st = rand_case()
    y, fs = run(d, st)
    yc, hc = complex_diagonal_reference(d, st)
    assert rel(y, yc) < TOL and rel(fs.h, hc) < TOL


def rot(v, ang):
    """Rotate interleaved pairs (v[2k], v[2k+1]) of the last axis by +ang[k]."""
    out = np.empty_like(v)
    c, s = np.cos(ang), np.sin(ang)
    out[..., 0::2] = v[..., 0::2] * c - v[..., 1::2] * s
    out[..., 1::2] = v[..., 0::2] * s + v[..., 1::2] * c
    return out


def rotated_frame_reference(d, st):
    """The literal statement: B_t, C_t rotated pair-wise by the cumulative angle
    phi_t = sum_{s<=t} dt_s theta_s, and
    g_t = a_t g_{t-1} + (1-lam_t) dt_t a_t B~_{t-1} x_{t-1}^T + lam_t dt_t B~_t x_t^T,
    y_t = g_t^T C~_t + D x_t;  the plain-frame state is Rot(-phi_t) g_t."""
    x, B, C, dt, lam, th, A, D = (d[k] for k in ("x", "B", "C", "dt", "lam", "theta", "A", "D"))
    Bt, T, H, R, P = x.shape
    phi = np.cumsum(dt[..., None] * th, axis=1)
    Bn = rot(B, phi[:, :, :, None, :])
    Cn = rot(C, phi[:, :, :, None, :])
    y = np.zeros_like(x)
    hT = np.zeros_like(st.h)
    for b in range(Bt):
        for h in range(H):
            g = st.h[b, h].copy()
            bprev, xprev = st.b_prev[b, h], st.x_prev[b, h]
            for t in range(T):
                a = math.exp(dt[b, t, h] * A[h])
                g = (a * g + (1 - lam[b, t, h]) * dt[b, t, h] * a * bprev.T @ xprev
                     + lam[b, t, h] * dt[b, t, h] * Bn[b, t, h].T @ x[b, t, h])
                y[b, t, h] = (g.T @ Cn[b, t, h].T).T + D[h] * x[b, t, h]
                bprev, xprev = Bn[b, t, h], x[b, t, h]
            hT[b, h] = rot(g.T, -phi[b, T - 1, h]).T
    return y, hT


def test_equals_rotated_frame_statement():
    d, st = rand_case()
    y, fs = run(d, st)
    yr, hr = rotated_frame_reference(d, st)
    assert rel(y, yr) < TOL and rel(fs.h, hr) < TOL


def ssd_dual_reference(d, st):
    """Brute-force masked-attention ('dual') form: materialise the full
    (T R) x (T R) matrix M o (C~ B~^T) and multiply by X.  Weights:
    w(t,t) = gamma_t; w(t,s<t) = exp(A sum_{k=s+1..t} dt_k) (gamma_s + beta'_{s+1}),
    plus the initial state read out through the total decay since the start."""
    x, B, C, dt, lam, th, A, D = (d[k] for k in ("x", "B", "C", "dt", "lam", "theta", "A", "D"))
    Bt, T, H, R, P = x.shape
    phi = np.cumsum(dt[..., None] * th, axis=1)
    Bn = rot(B, phi[:, :, :, None, :])
    Cn = rot(C, phi[:, :, :, None, :])
    y = np.zeros_like(x)
    for b in range(Bt):
        for h in range(H):
            gam = lam[b, :, h] * dt[b, :, h]
            betap = (1 - lam[b, :, h]) * dt[b, :, h]
            cum = np.concatenate([[0.0], np.cumsum(dt[b, :, h] * A[h])])  # cum[t+1] = sum_{k<=t}
            W = np.zeros((T, T))
            for t in range(T):
                W[t, t] = gam[t]
                for s in range(t):
                    W[t, s] = math.exp(cum[t + 1] - cum[s + 1]) * (gam[s] + betap[s + 1])
            CB = np.einsum("trn,sqn->trsq", Cn[b, :, h], Bn[b, :, h])  # [T,R,T,R]
            Mfull = W[:, None, :, None] * CB
            Y = Mfull.reshape(T * R, T * R) @ x[b, :, h].reshape(T * R, P)
            h0 = st.h[b, h] + betap[0] * st.b_prev[b, h].T @ st.x_prev[b, h]
            for t in range(T):
                Y[t * R:(t + 1) * R] += math.exp(cum[t + 1]) * (Cn[b, t, h] @ h0)
            y[b, :, h] = Y.reshape(T, R, P) + D[h] * x[b, :, h]
    return y


@pytest.mark.parametrize("R", [1, 2])
def test_equals_ssd_dual_bruteforce(R):
    d, st = rand_case(T=24, R=R)
    y, _ = run(d, st)
    assert rel(y, ssd_dual_reference(d, st)) < TOL


# ---------------------------------------------------------------- chunked restatement
def chunked_reference(d, st, Q):
    """Chunked form of the recurrence: chunk-local cumulative angles and
    log-decays, a masked decay-weighted C~ B~^T block inside each chunk, a
    decay-weighted chunk state G = (w o B~)^T X, and a plain-frame carried state
    h*_c = Rot(-Phi_c)(exp(cA_end) h*_{c-1} + G_c) between chunks (the four
    pieces of the chunked SSD algorithm, extended with the trapezoid's pending
    term folded into gamma_hat_s = gamma_s + beta'_{s+1})."""
    x, B, C, dt, lam, th, A, D = (d[k] for k in ("x", "B", "C", "dt", "lam", "theta", "A", "D"))
    Bt, T, H, R, P = x.shape
    N = B.shape[-1]
    y = np.zeros_like(x)
    hT = np.zeros_like(st.h)
    for b in range(Bt):
        for h in range(H):
            gam = lam[b, :, h] * dt[b, :, h]
            betap = (1 - lam[b, :, h]) * dt[b, :, h]
            ghat = gam.copy()
            ghat[:-1] += betap[1:]
            hs = st.h[b, h] + betap[0] * st.b_prev[b, h].T @ st.x_prev[b, h] if T else st.h[b, h]
            for c0 in range(0, T, Q):
                sl = slice(c0, min(T, c0 + Q))
                L = sl.stop - sl.start
                cA = np.cumsum(dt[b, sl, h] * A[h])
                phi = np.cumsum(dt[b, sl, h][:, None] * th[b, sl, h], axis=0)   # [L, N/2]
                Bn = rot(B[b, sl, h], phi[:, None, :])                            # [L,R,N]
                Cn = rot(C[b, sl, h], phi[:, None, :])
                Wm = np.zeros((L, L))
                for i in range(L):
                    for s in range(i + 1):
                        coef = gam[c0 + i] if s == i else ghat[c0 + s]
                        Wm[i, s] = math.exp(cA[i] - cA[s]) * coef
                S = np.einsum("irn,sqn->irsq", Cn, Bn)
                Xc = x[b, sl, h]
                Yd = np.einsum("is,irsq,sqp->irp", Wm, S, Xc)
                Yo = np.exp(cA)[:, None, None] * np.einsum("irn,np->irp", Cn, hs)
                y[b, sl, h] = Yd + Yo + D[h] * Xc
                w = np.exp(cA[-1] - cA) * ghat[sl]
                if sl.stop == T:
                    w[-1] = gam[T - 1]
                G = np.einsum("s,sqn,sqp->np", w, Bn, Xc)
                inner = math.exp(cA[-1]) * hs + G
                hs = rot(inner.T, -phi[-1]).T
            hT[b, h] = hs
    return y, hT


@pytest.mark.parametrize("Q", [1, 4, 16, 64])
def test_chunked_form_matches(Q):
    d, st = rand_case(T=53, R=2)
    y, fs = run(d, st)
    yc, hc = chunked_reference(d, st, Q)
    assert rel(y, yc) < TOL and rel(fs.h, hc) < TOL


# ---------------------------------------------------------------- structure
def test_mimo_is_sum_of_rank_one_runs():
    """The rank-R write is a sum of R outer products on one shared state, so the
    MIMO output for output rank r equals the sum over input ranks q of SISO runs
    driven by (B[:,q], x[:,q]) and read out with C[:,r]."""
    d, _ = rand_case(T=31, R=3, init=False)
    y, _ = run(d)
    Bt, T, H, R, P = d["x"].shape
    ref = np.zeros_like(y)
    for r in range(R):
        for q in range(R):
            ys, _ = oracle.scan(d["x"][:, :, :, q:q + 1], d["B"][:, :, :, q:q + 1],
                                d["C"][:, :, :, r:r + 1], d["dt"], d["lam"], d["theta"],
                                d["A"], np.zeros_like(d["D"]))
            ref[:, :, :, r] += ys[:, :, :, 0]
        ref[:, :, :, r] += d["D"][None, None, :, None] * d["x"][:, :, :, r]
    assert rel(y, ref) < TOL


def test_prefill_then_decode_equals_full_scan():
    d, st = rand_case(T=40, R=2)
    yfull, sfull = run(d, st)
    T1 = 25
    part = {k: (v[:, :T1] if v.ndim >= 3 else v) for k, v in d.items()}
    y1, s = run(part, st)
    ys = [y1]
    for t in range(T1, 40):
        yt, s = oracle.step(d["x"][:, t], d["B"][:, t], d["C"][:, t], d["dt"][:, t],
                            d["lam"][:, t], d["theta"][:, t], d["A"], d["D"], s)
        ys.append(yt[:, None])
    np.testing.assert_allclose(np.concatenate(ys, axis=1), yfull, atol=1e-13, rtol=0)
    np.testing.assert_allclose(s.h, sfull.h, atol=1e-13, rtol=0)
    np.testing.assert_allclose(s.b_prev, sfull.b_prev, atol=0, rtol=0)
    np.testing.assert_allclose(s.x_prev, sfull.x_prev, atol=0, rtol=0)


def test_split_scan_resumes_exactly():
    """scan(T1) with its final state passed as the next call's initial state
    equals one scan over T1+T2 (the pending term crosses the call boundary)."""
    d, st = rand_case(T=30, R=1)
    yfull, sfull = run(d, st)
    a = {k: (v[:, :11] if v.ndim >= 3 else v) for k, v in d.items()}
    b = {k: (v[:, 11:] if v.ndim >= 3 else v) for k, v in d.items()}
    ya, sa = run(a, st)
    yb, sb = run(b, sa)
    np.testing.assert_allclose(np.concatenate([ya, yb], 1), yfull, atol=1e-13, rtol=0)
    np.testing.assert_allclose(sb.h, sfull.h, atol=1e-13, rtol=0)


def test_empty_sequence_returns_initial_state():
    d, st = rand_case(T=0)
    y, fs = run(d, st)
    assert y.shape[1] == 0
    np.testing.assert_array_equal(fs.h, st.h)
    np.testing.assert_array_equal(fs.b_prev, st.b_prev)
    np.testing.assert_array_equal(fs.x_prev, st.x_prev)


def test_threading_is_deterministic():
    d, st = rand_case(Bt=3, H=3, T=17)
    y1, s1 = oracle.scan(*(d[k] for k in ("x", "B", "C", "dt", "lam", "theta", "A", "D")), st, nthreads=1)
    y4, s4 = oracle.scan(*(d[k] for k in ("x", "B", "C", "dt", "lam", "theta", "A", "D")), st, nthreads=4)
    np.testing.assert_array_equal(y1, y4)
    np.testing.assert_array_equal(s1.h, s4.h)


# ---------------------------------------------------------------- per-token A
def per_token_case(T=31, R=2, seed=11):
    s = Shape(2, T, 2, 5, 8, R, "f32", seed)
    d = {k: v.double().numpy() for k, v in make_prefill(s, a_per_token=True).items()}
    h, bp, xp = (t.double().numpy() for t in make_state(s))
    return d, oracle.State(h, bp, xp)


def test_per_token_A_constant_in_time_equals_per_head():
    """A_t held fixed per head is the per-head method: same arithmetic, so the
    results agree to the last bit."""
    d, st = rand_case(T=29)
    Bt, T, H = d["dt"].shape
    y1, f1 = run(d, st)
    d2 = dict(d, A=np.ascontiguousarray(np.broadcast_to(d["A"], (Bt, T, H))))
    y2, f2 = run(d2, st)
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(f1.h, f2.h)


def test_per_token_A_free_decay_closed_form():
    """x = 0, no pending input, A varying per token: the state decays by
    exp(sum_t dt_t A_t) and rotates by sum_t dt_t theta_t."""
    d, st = per_token_case(T=27)
    d["x"][:] = 0.0
    st.x_prev[:] = 0.0
    y, fs = run(d, st)
    ldec = np.cumsum(d["dt"] * d["A"], axis=1)                    # [Bt,T,H]
    phi = np.cumsum(d["dt"][..., None] * d["theta"], axis=1)
    u, v = st.h[:, None, :, 0::2, :], st.h[:, None, :, 1::2, :]
    c, s = np.cos(phi)[..., None], np.sin(phi)[..., None]
    e = np.exp(ldec)[..., None, None]
    ht = np.empty(u.shape[:1] + (phi.shape[1],) + u.shape[2:3] + (u.shape[3] * 2, u.shape[4]))
    ht[..., 0::2, :], ht[..., 1::2, :] = e * (u * c + v * s), e * (-u * s + v * c)
    ref = np.einsum("bthnp,bthrn->bthrp", ht, d["C"])
    assert rel(y, ref) < TOL
    assert rel(fs.h, ht[:, -1]) < TOL


def test_per_token_A_ssd_dual_bruteforce():
    """The masked-attention dual with the decay between s and t taken as
    exp(sum_{k=s+1..t} dt_k A_k)."""
    d, st = per_token_case(T=19, R=2)
    y, _ = run(d, st)
    x, B, C, dt, lam, th, A, D = (d[k] for k in ("x", "B", "C", "dt", "lam", "theta", "A", "D"))
    Bt, T, H, R, P = x.shape
    phi = np.cumsum(dt[..., None] * th, axis=1)
    Bn, Cn = rot(B, phi[:, :, :, None, :]), rot(C, phi[:, :, :, None, :])
    ref = np.zeros_like(x)
    for b in range(Bt):
        for h in range(H):
            gam, betap = lam[b, :, h] * dt[b, :, h], (1 - lam[b, :, h]) * dt[b, :, h]
            cum = np.concatenate([[0.0], np.cumsum(dt[b, :, h] * A[b, :, h])])
            Y = np.zeros((T, R, P))
            h0 = st.h[b, h] + betap[0] * st.b_prev[b, h].T @ st.x_prev[b, h]
            for t in range(T):
                acc = math.exp(cum[t + 1]) * (Cn[b, t, h] @ h0)
                for s_ in range(t + 1):
                    w = gam[t] if s_ == t else math.exp(cum[t + 1] - cum[s_ + 1]) * (gam[s_] + betap[s_ + 1])
                    acc = acc + w * (Cn[b, t, h] @ Bn[b, s_, h].T) @ x[b, s_, h]
                Y[t] = acc + D[h] * x[b, t, h]
            ref[b, :, h] = Y
    assert rel(y, ref) < TOL


def test_per_token_A_decode_continues_the_scan():
    """Decode steps with their own A_t continue the per-token-A scan exactly."""
    d, st = per_token_case(T=20)
    y_full, f_full = run(d, st)
    k = 13
    part = {key: (v[:, :k] if v.ndim >= 3 and key not in ("D",) else v) for key, v in d.items()}
    _, fs = run(part, st)
    ys = []
    for t in range(k, d["x"].shape[1]):
        args = [d[key][:, t] for key in ("x", "B", "C", "dt", "lam", "theta")]
        yt, fs = oracle.step(*args, d["A"][:, t], d["D"], fs)
        ys.append(yt)
    assert rel(np.stack(ys, 1), y_full[:, k:]) < TOL
    assert rel(fs.h, f_full.h) < TOL


# ---------------------------------------------------------------- theta fixed per head
def test_theta_per_head_equals_broadcast_per_token():
    """theta [H, N/2] is the per-token method with theta repeated over tokens:
    same arithmetic, bit for bit (scan and decode step)."""
    s = Shape(2, 23, 2, 5, 8, 2, "f32", 12)
    d = {k: v.double().numpy() for k, v in make_prefill(s, theta_per_head=True).items()}
    assert d["theta"].shape == (2, 4)
    h, bp, xp = (t.double().numpy() for t in make_state(s))
    st = oracle.State(h, bp, xp)
    y1, f1 = run(d, st)
    d2 = dict(d, theta=np.ascontiguousarray(np.broadcast_to(d["theta"][None, None], (2, 23, 2, 4))))
    y2, f2 = run(d2, st)
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(f1.h, f2.h)
    args = [d[k][:, 0] for k in ("x", "B", "C", "dt", "lam")]
    ya, sa = oracle.step(*args, d["theta"], d["A"], d["D"], st)
    yb, sb = oracle.step(*args, d2["theta"][:, 0], d["A"], d["D"], st)
    np.testing.assert_array_equal(ya, yb)
    np.testing.assert_array_equal(sa.h, sb.h)


def test_theta_per_head_free_rotation_closed_form():
    """x = 0, no pending input, theta fixed per head: pair k turns by
    theta_k * sum_t dt_t, so z_t = exp(sum dt (A - i theta_k)) z_0."""
    s = Shape(1, 33, 2, 3, 6, 1, "f32", 13)
    d = {k: v.double().numpy() for k, v in make_prefill(s, theta_per_head=True).items()}
    d["x"][:] = 0.0
    h, bp, xp = (t.double().numpy() for t in make_state(s))
    xp[:] = 0.0
    y, fs = run(d, oracle.State(h, bp, xp))
    cd = np.sum(d["dt"][0], axis=0)                                  # [H]
    z0 = h[0, :, 0::2, :] + 1j * h[0, :, 1::2, :]                   # [H, N/2, P]
    z = np.exp((cd * d["A"])[:, None, None] - 1j * (cd[:, None] * d["theta"])[:, :, None]) * z0
    assert rel(fs.h[0, :, 0::2, :], z.real) < TOL and rel(fs.h[0, :, 1::2, :], z.imag) < TOL


# ---------------------------------------------------------------- BC-norm prologue
def bcn_case(T=21, R=2, seed=14, eps=1e-6):
    from m3_inputs import make_bcnorm
    s = Shape(1, T, 2, 5, 8, R, "f32", seed)
    d = {k: v.double().numpy() for k, v in make_prefill(s).items()}
    bn = {k: (v.double().numpy() if hasattr(v, "double") else v) for k, v in make_bcnorm(s).items()}
    h, bp, xp = (t.double().numpy() for t in make_state(s))
    return d, oracle.BCNorm(bn["wB"], bn["wC"], bn["bB"], bn["bC"], eps), oracle.State(h, bp, xp)


def run_bcn(d, bcn, st=None):
    return oracle.scan(d["x"], d["B"], d["C"], d["dt"], d["lam"], d["theta"], d["A"], d["D"], st, bcnorm=bcn)


def test_bcnorm_row_scale_invariance():
    """The RMS norm divides out any positive scale of a (token, head, rank)
    row: rescaling every row of B and C by its own factor leaves y and the
    state unchanged (eps negligible)."""
    d, bcn, st = bcn_case(eps=1e-300)
    y1, f1 = run_bcn(d, bcn, st)
    rng = np.random.default_rng(3)
    d2 = dict(d)
    d2["B"] = d["B"] * rng.uniform(0.1, 10.0, size=d["B"].shape[:-1] + (1,))
    d2["C"] = d["C"] * rng.uniform(0.1, 10.0, size=d["C"].shape[:-1] + (1,))
    y2, f2 = run_bcn(d2, bcn, st)
    assert rel(y2, y1) < 1e-12 and rel(f2.h, f1.h) < 1e-12 and rel(f2.b_prev, f1.b_prev) < 1e-12


def unit_rms(a):
    return a / np.sqrt(np.mean(a * a, axis=-1, keepdims=True))


def test_bcnorm_identity_on_unit_rms_rows():
    """Rows already at unit RMS, w = 1, no bias: the prologue is the identity."""
    d, bcn, st = bcn_case(eps=1e-300)
    d["B"], d["C"] = unit_rms(d["B"]), unit_rms(d["C"])
    N = d["B"].shape[-1]
    ident = oracle.BCNorm(np.ones(N), np.ones(N), np.zeros_like(bcn.bB), np.zeros_like(bcn.bC), 1e-300)
    y1, f1 = run_bcn(d, ident, st)
    y2, f2 = run(d, st)
    assert rel(y1, y2) < 1e-12 and rel(f1.h, f2.h) < 1e-12


def test_bcnorm_weight_and_bias_placement():
    """Unit-RMS rows: the prologue reduces to B w + b[h, r] (w over the state
    index, b per head and rank), i.e. the plain method on those inputs."""
    d, bcn, st = bcn_case(eps=1e-300)
    d["B"], d["C"] = unit_rms(d["B"]), unit_rms(d["C"])
    y1, f1 = run_bcn(d, bcn, st)
    d2 = dict(d)
    d2["B"] = d["B"] * bcn.wB + bcn.bB[None, None]
    d2["C"] = d["C"] * bcn.wC + bcn.bC[None, None]
    y2, f2 = run(d2, st)
    assert rel(y1, y2) < 1e-12 and rel(f1.h, f2.h) < 1e-12 and rel(f1.b_prev, f2.b_prev) < 1e-12


def test_bcnorm_decode_continues_the_scan():
    d, bcn, st = bcn_case(T=16)
    y_full, f_full = run_bcn(d, bcn, st)
    k = 9
    part = {key: (v[:, :k] if v.ndim >= 3 else v) for key, v in d.items()}
    _, fs = run_bcn(part, bcn, st)
    ys = []
    for t in range(k, 16):
        args = [d[key][:, t] for key in ("x", "B", "C", "dt", "lam", "theta")]
        yt, fs = oracle.step(*args, d["A"], d["D"], fs, bcnorm=bcn)
        ys.append(yt)
    assert rel(np.stack(ys, 1), y_full[:, k:]) < TOL and rel(fs.h, f_full.h) < TOL


def test_bcnorm_eps_inside_the_root_with_both_options():
    """With eps comparable to the rows' mean square, the prologue is
    B / sqrt(mean_n B^2 + eps) * w + b (eps inside the root, as the header
    states), written out here in numpy; checked with per-token A and angle
    rates fixed per head at the same time."""
    from m3_inputs import make_bcnorm
    s = Shape(2, 19, 2, 5, 8, 2, "f32", 15)
    d = {k: v.double().numpy() for k, v in make_prefill(s, a_per_token=True, theta_per_head=True).items()}
    assert d["A"].shape == (2, 19, 2) and d["theta"].shape == (2, 4)
    bn = {k: (v.double().numpy() if hasattr(v, "double") else v) for k, v in make_bcnorm(s).items()}
    eps = 0.3  # the rows' mean square is about 1/N = 0.125
    bcn = oracle.BCNorm(bn["wB"], bn["wC"], bn["bB"], bn["bC"], eps)
    st = oracle.State(*(t.double().numpy() for t in make_state(s)))
    y1, f1 = run_bcn(d, bcn, st)

    def norm(a, w, b):
        return a / np.sqrt(np.mean(a * a, axis=-1, keepdims=True) + eps) * w + b[None, None]

    d2 = dict(d)
    d2["B"], d2["C"] = norm(d["B"], bn["wB"], bn["bB"]), norm(d["C"], bn["wC"], bn["bC"])
    y2, f2 = run(d2, st)
    assert rel(y1, y2) < 1e-12 and rel(f1.h, f2.h) < 1e-12 and rel(f1.b_prev, f2.b_prev) < 1e-12
    # and eps does matter at this size: outside the root it gives another answer
    d3 = dict(d)
    d3["B"] = d["B"] / (np.sqrt(np.mean(d["B"] ** 2, axis=-1, keepdims=True)) + eps) * bn["wB"] + bn["bB"][None, None]
    d3["C"] = d["C"] / (np.sqrt(np.mean(d["C"] ** 2, axis=-1, keepdims=True)) + eps) * bn["wC"] + bn["bC"][None, None]
    y3, _ = run(d3, st)
    assert rel(y3, y1) > 1e-3


# ---------------------------------------------------------------- MIMO projections
def proj_case(T=29, H=2, P=5, N=8, R=3, seed=7):
    from m3_inputs import make_prefill_proj, make_proj
    s = Shape(1, T, H, P, N, R, "f32", seed)
    d = {k: v.double().numpy() for k, v in make_prefill_proj(s).items()}
    w = {k: v.double().numpy() for k, v in make_proj(s).items()}
    return d, oracle.MimoProj(w["wx"], w["wB"], w["wC"], w["wy"])


def run_proj(d, pr, st=None):
    return oracle.scan_proj(d["x"], d["B"], d["C"], d["dt"], d["lam"], d["theta"], d["A"], d["D"], pr, st)


def test_proj_is_a_sum_of_siso_runs():
    """With the projections the rank-R write is still a sum of R outer
    products on one state, so y equals sum_r wy_r * (sum_q SISO runs driven by
    (wB_q b, wx_q x) and read out with wC_r c, plus D wx_r x) -- R^2 rank-1
    runs of the plain scan, combined in numpy."""
    d, pr = proj_case()
    y, _ = run_proj(d, pr)
    x, b, c = d["x"], d["B"], d["C"]
    R = pr.wx.shape[1]
    ref = np.zeros_like(y)
    for r in range(R):
        yr = pr.wx[None, None, :, r] * x * d["D"][None, None, :, None]
        for q in range(R):
            ys, _ = oracle.scan((pr.wx[None, None, :, q] * x)[:, :, :, None],
                                (pr.wB[None, None, :, q] * b)[:, :, :, None],
                                (pr.wC[None, None, :, r] * c)[:, :, :, None],
                                d["dt"], d["lam"], d["theta"], d["A"], np.zeros_like(d["D"]))
            yr = yr + ys[:, :, :, 0]
        ref += pr.wy[None, None, :, r] * yr
    assert rel(y, ref) < TOL


def test_proj_with_unit_weights_is_r_times_siso():
    """wx = wB = wC = 1 and wy = (1, 0, ..., 0): the R identical outer products
    write R copies of the SISO update into the state, so y = R * (SISO scan
    without its D term) + D x."""
    d, pr = proj_case(R=4)
    H, R, P = pr.wx.shape
    N = pr.wB.shape[-1]
    wy = np.zeros((H, R, P))
    wy[:, 0] = 1.0
    unit = oracle.MimoProj(np.ones((H, R, P)), np.ones((H, R, N)), np.ones((H, R, N)), wy)
    y, st = run_proj(d, unit)
    ys, ss = oracle.scan(d["x"][:, :, :, None], d["B"][:, :, :, None], d["C"][:, :, :, None], d["dt"],
                         d["lam"], d["theta"], d["A"], np.zeros_like(d["D"]))
    assert rel(y, R * ys[:, :, :, 0] + d["D"][None, None, :, None] * d["x"]) < TOL
    assert rel(st.h, R * ss.h) < TOL


def test_proj_rank_one_unit_weights_is_siso():
    d, pr = proj_case(R=1)
    H, R, P = pr.wx.shape
    N = pr.wB.shape[-1]
    unit = oracle.MimoProj(np.ones((H, 1, P)), np.ones((H, 1, N)), np.ones((H, 1, N)), np.ones((H, 1, P)))
    y, _ = run_proj(d, unit)
    ys, _ = oracle.scan(d["x"][:, :, :, None], d["B"][:, :, :, None], d["C"][:, :, :, None], d["dt"],
                        d["lam"], d["theta"], d["A"], d["D"])
    np.testing.assert_array_equal(y, ys[:, :, :, 0])


def test_proj_output_is_linear_in_wy_and_state_ignores_it():
    d, pr = proj_case()
    y1, s1 = run_proj(d, pr)
    pr2 = oracle.MimoProj(pr.wx, pr.wB, pr.wC, 2.5 * pr.wy - 0.5)
    y2, s2 = run_proj(d, pr2)
    pr0 = oracle.MimoProj(pr.wx, pr.wB, pr.wC, np.ones_like(pr.wy))
    y0, _ = run_proj(d, pr0)
    assert rel(y2, 2.5 * y1 - 0.5 * y0) < TOL
    np.testing.assert_array_equal(s1.h, s2.h)


def test_proj_prefill_then_decode_equals_full_scan():
    """scan_proj over T1 tokens, then step_proj for the rest, equals one
    scan_proj (the widened pending term crosses the boundary in the state)."""
    d, pr = proj_case(T=21, R=2)
    s = Shape(1, 21, 2, 5, 8, 2, "f32", 7)
    h, bp, xp = (t.double().numpy() for t in make_state(s))
    st0 = oracle.State(h, bp, xp)
    yfull, sfull = run_proj(d, pr, st0)
    T1 = 13
    part = {k: (v[:, :T1] if v.ndim >= 3 else v) for k, v in d.items()}
    y1, st = run_proj(part, pr, st0)
    ys = [y1]
    for t in range(T1, 21):
        yt, st = oracle.step_proj(d["x"][:, t], d["B"][:, t], d["C"][:, t], d["dt"][:, t], d["lam"][:, t],
                                  d["theta"][:, t], d["A"], d["D"], pr, st)
        ys.append(yt[:, None])
    np.testing.assert_allclose(np.concatenate(ys, axis=1), yfull, atol=1e-13, rtol=0)
    np.testing.assert_allclose(st.h, sfull.h, atol=1e-13, rtol=0)
