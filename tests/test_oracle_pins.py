"""Pins for the fp64 oracle: each check ties it to something other than itself.

The pages print no IA output values, so agreement with the authors' own code
is unpinned; every pin here comes from the mathematics of the recurrence the
paper describes (paperlayer.ai summary of 'Interdomain Attention', sec. 3.1-3.2
and sec. D.2; AI-radio page formula extract 'O = Fq U^T Gamma / Fq U^T eta'):
brute force, closed forms, invariants, special cases that reduce to textbook
averages, hand-derived fixtures, finite differences and a tangent/adjoint test.
Each pin is chosen so that a plausible slip in the oracle (dropped conjugate,
wrong decay index, missing b, transposed operand) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(x, r):
    x = np.asarray(x)
    r = np.asarray(r)
    return float(np.max(np.abs(x - r)) / max(np.max(np.abs(r)), 1e-300))


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def small_case(seed=0, B=2, H=2, N=37, d=3, dv=2, M=5):
    q = rnd((B, H, N, d), seed)
    k = rnd((B, H, N, d), seed + 1)
    v = rnd((B, H, N, dv), seed + 2)
    delta = np.exp(np.log(1e-3) + np.random.default_rng(seed + 3).random(H) * (np.log(1e-1) - np.log(1e-3)))
    return q, k, v, delta, M


def feat(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


# ---------------------------------------------------------------- P1 brute force
def test_p1_brute_force_matches_recurrence(oracle_mod):
    q, k, v, delta, M = small_case(N=41, M=6)
    delta = np.array([0.08, 0.3])          # large steps: fast rotation of high modes
    r = oracle_mod.forward(q, k, v, delta, M)
    b = oracle_mod.brute(q, k, v, delta, M)
    assert rel(r["num"], b["num"]) < 1e-12
    assert rel(r["den"], b["den"]) < 1e-12
    assert rel(r["o"], b["o"]) < 1e-10


def _mp_brute(q, k, v, delta, M, A=None):
    """Quadratic form in 40-digit mpmath, one (b,h) slice, zero state.  delta
    is one step for all modes or one per mode; A defaults to S4D-Lin."""
    import mpmath as mp
    mp.mp.dps = 40
    N, d = q.shape
    dv = v.shape[1]

    def xi(x):
        x = mp.mpf(float(x))
        return x + 1 if x > 0 else mp.e ** x

    fq = [[xi(q[t, f]) for f in range(d)] for t in range(N)]
    fk = [[xi(k[t, f]) for f in range(d)] for t in range(N)]
    if A is None:
        A = [mp.mpc(-0.5, mp.pi * m) for m in range(M)]
    else:
        A = [mp.mpc(float(A[2 * m]), float(A[2 * m + 1])) for m in range(M)]
    D = [mp.mpf(float(x)) for x in np.broadcast_to(np.asarray(delta, dtype=float), (M,))]
    lam = [mp.e ** (D[m] * A[m]) for m in range(M)]
    bb = [(lam[m] - 1) / A[m] for m in range(M)]
    out = []
    for t in range(N):
        s = [sum(fq[t][f] * fk[n][f] for f in range(d)) for n in range(t + 1)]
        a = [bb[m] * sum(lam[m] ** (t - n) * s[n] for n in range(t + 1)) for m in range(M)]
        w = [sum((mp.conj(a[m]) * bb[m] * lam[m] ** (t - n)).real for m in range(M)) for n in range(t + 1)]
        den = sum(w)
        out.append([float(sum(w[n] * v[n, j] for n in range(t + 1)) / den) for j in range(dv)])
    return np.array(out)


def test_p1_mpmath_brute_force(oracle_mod):
    q, k, v, delta, M = small_case(B=1, H=1, N=9, d=2, dv=2, M=3)
    delta = np.array([0.37])
    r = oracle_mod.forward(q, k, v, delta, M)
    ref = _mp_brute(q[0, 0], k[0, 0], v[0, 0], delta[0], M)
    assert rel(r["o"][0, 0], ref) < 1e-12


# ---------------------------------------------------------------- P2 eta closed form
def test_p2_eta_closed_form(oracle_mod):
    q, k, v, delta, M = small_case(N=53, M=7)
    r = oracle_mod.forward(q, k, v, delta, M)
    B, H, N, d = q.shape
    _, _, eta = oracle_mod.split_state(r["state"], B, H, M, d, v.shape[-1])
    for h in range(H):
        A = -0.5 + 1j * np.pi * np.arange(M)
        closed = (np.exp(N * delta[h] * A) - 1.0) / A   # b/(1-lambda) = -1/A
        for bi in range(B):
            assert rel(eta[bi, h], closed) < 1e-13


def test_p2_params_zoh(oracle_mod):
    # b = integral_0^Delta exp(A s) ds: check against a midpoint-free Simpson rule
    M, delta = 6, 0.07
    lam, b = oracle_mod.params(M, delta)
    A = -0.5 + 1j * np.pi * np.arange(M)
    s = np.linspace(0.0, delta, 2001)
    w = np.ones_like(s)
    w[1:-1:2] = 4
    w[2:-1:2] = 2
    integral = (np.exp(np.outer(A, s)) * w).sum(axis=1) * (s[1] - s[0]) / 3
    assert rel(b, integral) < 1e-12
    # |lambda| = exp(-Delta/2) for every S4D-Lin mode, arg = pi m Delta
    assert np.allclose(np.abs(lam), math.exp(-0.5 * delta), rtol=0, atol=1e-15)
    assert np.allclose(np.angle(lam), np.angle(np.exp(1j * np.pi * np.arange(M) * delta)), atol=1e-14)


# ---------------------------------------------------------------- P3 first token
def test_p3_first_token_returns_v1(oracle_mod):
    q, k, v, delta, M = small_case(N=5, M=9)
    r = oracle_mod.forward(q, k, v, delta, M)
    assert rel(r["o"][:, :, 0], v[:, :, 0]) < 1e-14
    # den_1 = xi(q1).xi(k1) * sum |b|^2 > 0
    for h in range(q.shape[1]):
        _, b = oracle_mod.params(M, delta[h])
        s = (feat(q[:, h, 0]) * feat(k[:, h, 0])).sum(-1)
        assert rel(r["den"][:, h, 0], s * np.sum(np.abs(b) ** 2)) < 1e-14


# ---------------------------------------------------------------- P4 affine values
def test_p4_constant_and_affine_values(oracle_mod):
    q, k, v, delta, M = small_case(N=30, M=5)
    c = np.full_like(v, 1.7)
    r = oracle_mod.forward(q, k, c, delta, M)
    # den may be small somewhere; compare on num/den consistency instead of o
    assert rel(r["num"], 1.7 * r["den"][..., None] * np.ones_like(c)) < 1e-12
    r0 = oracle_mod.forward(q, k, v, delta, M)
    r1 = oracle_mod.forward(q, k, -2.5 * v + 0.75, delta, M)
    assert rel(r1["num"], -2.5 * r0["num"] + 0.75 * r0["den"][..., None]) < 1e-12
    assert rel(r1["den"], r0["den"]) < 1e-13


# ---------------------------------------------------------------- P5 feature scaling
def test_p5_feature_scaling_leaves_o(oracle_mod):
    q, k, v, delta, M = small_case(N=25, M=4)
    B, H = q.shape[:2]
    lam = np.zeros((H, M), complex)
    b = np.zeros((H, M), complex)
    for h in range(H):
        lam[h], b[h] = oracle_mod.params(M, delta[h])
    fq, fk = feat(q), feat(k)
    r = oracle_mod.forward_features(fq, fk, v, lam, b)
    ref = oracle_mod.forward(q, k, v, delta, M)
    assert rel(r["o"], ref["o"]) < 1e-14
    for alpha in (0.125, 3.0):
        ra = oracle_mod.forward_features(alpha * fq, fk, v, lam, b)
        rb = oracle_mod.forward_features(fq, alpha * fk, v, lam, b)
        assert rel(ra["num"], alpha * r["num"]) < 1e-13
        assert rel(rb["o"], r["o"]) < 1e-12


# ---------------------------------------------------------------- P6 mode additivity
def test_p6_mode_additivity(oracle_mod):
    q, k, v, delta, M = small_case(N=33, M=8)
    B, H = q.shape[:2]
    lam = np.zeros((H, M), complex)
    b = np.zeros((H, M), complex)
    for h in range(H):
        lam[h], b[h] = oracle_mod.params(M, delta[h])
    fq, fk = feat(q), feat(k)
    full = oracle_mod.forward_features(fq, fk, v, lam, b)
    lo = oracle_mod.forward_features(fq, fk, v, lam[:, :3], b[:, :3])
    hi = oracle_mod.forward_features(fq, fk, v, lam[:, 3:], b[:, 3:])
    assert rel(lo["num"] + hi["num"], full["num"]) < 1e-13
    assert rel(lo["den"] + hi["den"], full["den"]) < 1e-13


# ---------------------------------------------------------------- P10 M = 1 -> EMA
def test_p10_single_real_mode_is_normalised_ema(oracle_mod):
    q, k, v, delta, _ = small_case(N=40, M=1)
    r = oracle_mod.forward(q, k, v, delta, 1)
    N = q.shape[2]
    for h in range(q.shape[1]):
        lam = math.exp(-0.5 * delta[h])
        t = np.arange(N)
        W = np.tril(lam ** (t[:, None] - t[None, :]).astype(float))
        W = np.where(t[:, None] >= t[None, :], W, 0.0)
        ema = (W @ v[:, h]) / W.sum(1)[None, :, None]
        assert rel(r["o"][:, h], ema) < 1e-13


# ---------------------------------------------------------------- P11 Delta -> 0
def test_p11_small_step_limit_is_cumulative_mean(oracle_mod):
    q, k, v, _, M = small_case(B=1, H=1, N=24, M=4)
    cm = np.cumsum(v, axis=2) / np.arange(1, v.shape[2] + 1)[None, None, :, None]
    errs = []
    for d in (1e-4, 1e-5, 1e-6):
        r = oracle_mod.forward(q, k, v, np.array([d]), M)
        errs.append(rel(r["o"], cm))
    assert errs[0] / errs[1] > 7 and errs[1] / errs[2] > 7
    assert errs[2] < 1e-4


# ---------------------------------------------------------------- P12/P13 state plumbing
def test_p12_prefill_then_decode_equals_longer_prefill(oracle_mod):
    q, k, v, delta, M = small_case(N=31, M=5)
    n0 = 26
    full = oracle_mod.forward(q, k, v, delta, M)
    part = oracle_mod.forward(q[:, :, :n0], k[:, :, :n0], v[:, :, :n0], delta, M)
    st = part["state"]
    for t in range(n0, q.shape[2]):
        o, num, den, st = oracle_mod.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], delta, M, st)
        assert rel(o, full["o"][:, :, t]) < 1e-12
        assert rel(den, full["den"][:, :, t]) < 1e-12
    assert rel(st, full["state"]) < 1e-12


def test_p13_split_prefill_equals_single_prefill(oracle_mod):
    q, k, v, delta, M = small_case(N=45, M=6)
    n1 = 17
    full = oracle_mod.forward(q, k, v, delta, M)
    a = oracle_mod.forward(q[:, :, :n1], k[:, :, :n1], v[:, :, :n1], delta, M)
    b = oracle_mod.forward(q[:, :, n1:], k[:, :, n1:], v[:, :, n1:], delta, M, state_in=a["state"])
    assert rel(np.concatenate([a["o"], b["o"]], axis=2), full["o"]) < 1e-12
    assert rel(b["state"], full["state"]) < 1e-12


# ---------------------------------------------------------------- golden fixtures
@pytest.mark.parametrize("name", ["m1_real_ema.json", "m1_rotating_mode.json"])
def test_golden_hand_derived(oracle_mod, name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    q = np.array(g["q"])[None, None]
    k = np.array(g["k"])[None, None]
    v = np.array(g["v"])[None, None]
    r = oracle_mod.forward(q, k, v, np.array([g["delta"]]), g["M"], A=np.array(g["A"]))
    assert rel(r["o"][0, 0], np.array(g["o"])) < 1e-14
    if "eta_final" in g:
        _, _, eta = oracle_mod.split_state(r["state"], 1, 1, 1, 1, 1)
        assert abs(eta[0, 0, 0] - complex(*g["eta_final"])) < 1e-14


# ---------------------------------------------------------------- P8 finite differences
def test_p8_finite_differences(oracle_mod):
    B, H, N, d, dv, M = 1, 2, 14, 3, 2, 4
    q, k, v, delta, _ = small_case(seed=11, B=B, H=H, N=N, d=d, dv=dv, M=M)
    delta = np.array([0.09, 0.04])
    dO = rnd((B, H, N, dv), 99)
    g = oracle_mod.backward(q, k, v, delta, dO, M)
    f0 = oracle_mod.forward(q, k, v, delta, M)
    assert rel(g["o"], f0["o"]) < 1e-15

    def loss(q_, k_, v_, d_):
        return float(np.sum(dO * oracle_mod.forward(q_, k_, v_, d_, M)["o"]))

    rng = np.random.default_rng(5)
    for name, arr, grad in (("q", q, g["dq"]), ("k", k, g["dk"]), ("v", v, g["dv"])):
        for _ in range(6):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            h = 1e-6 * max(1.0, abs(arr[idx]))
            xp = arr.copy(); xp[idx] += h
            xm = arr.copy(); xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p, delta) - loss(*args_m, delta)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])
    for hh in range(H):
        h = 1e-7
        dp = delta.copy(); dp[hh] += h
        dm = delta.copy(); dm[hh] -= h
        fd = (loss(q, k, v, dp) - loss(q, k, v, dm)) / (2 * h)
        assert abs(fd - g["dDelta"][hh]) <= 1e-6 * max(1.0, abs(fd)), (hh, fd, g["dDelta"][hh])


# ---------------------------------------------------------------- P9 tangent vs adjoint
def test_p9_tangent_adjoint_dot_product(oracle_mod):
    B, H, N, d, dv, M = 2, 3, 70, 4, 3, 6      # N > 64 crosses a checkpoint block
    q, k, v, delta, _ = small_case(seed=21, B=B, H=H, N=N, d=d, dv=dv, M=M)
    dO = rnd((B, H, N, dv), 7)
    tq, tk, tv = rnd(q.shape, 8), rnd(k.shape, 9), rnd(v.shape, 10)
    td = rnd((H,), 12)
    to = oracle_mod.jvp(q, k, v, delta, tq, tk, tv, td, M)
    g = oracle_mod.backward(q, k, v, delta, dO, M)
    lhs = float(np.sum(dO * to))
    rhs = float(np.sum(g["dq"] * tq) + np.sum(g["dk"] * tk) + np.sum(g["dv"] * tv) + np.sum(g["dDelta"] * td))
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), (lhs, rhs)


def test_backward_batch_sum_of_ddelta(oracle_mod):
    # dDelta sums over the batch: doubling the batch with a copy doubles it
    q, k, v, delta, M = small_case(seed=4, B=1, H=2, N=20, M=3)
    dO = rnd(v.shape, 3)
    g1 = oracle_mod.backward(q, k, v, delta, dO, M)
    cat = lambda x: np.concatenate([x, x], axis=0)
    g2 = oracle_mod.backward(cat(q), cat(k), cat(v), delta, cat(dO), M)
    assert rel(g2["dDelta"], 2 * g1["dDelta"]) < 1e-13


# ---------------------------------------------------------------- trainable A, Delta per (head, mode)
def _modes_case(seed, B=1, H=2, N=14, d=3, dv=2, M=4):
    """Inputs with one Delta per (head, mode) and a general A (decaying modes
    at other frequencies than S4D-Lin)."""
    q, k, v, _, _ = small_case(seed=seed, B=B, H=H, N=N, d=d, dv=dv, M=M)
    rng = np.random.default_rng(seed + 50)
    delta = 0.02 + 0.1 * rng.random((H, M))
    A = np.empty(2 * M)
    A[0::2] = -0.2 - 0.6 * rng.random(M)
    A[1::2] = np.pi * np.arange(M) + 0.7 * rng.random(M)
    return q, k, v, delta, A, M


def test_p1_per_mode_delta_brute_force(oracle_mod):
    q, k, v, delta, A, M = _modes_case(31, B=2, H=2, N=33, M=5)
    r = oracle_mod.forward(q, k, v, delta, M, A=A)
    b = oracle_mod.brute(q, k, v, delta, M, A=A)
    assert rel(r["num"], b["num"]) < 1e-12 and rel(r["den"], b["den"]) < 1e-12
    # one Delta per head is the special case of equal per-mode steps
    dh = np.array([0.05, 0.11])
    r1 = oracle_mod.forward(q, k, v, dh, M, A=A)
    r2 = oracle_mod.forward(q, k, v, np.repeat(dh[:, None], M, axis=1), M, A=A)
    assert rel(r2["o"], r1["o"]) < 1e-15 and rel(r2["state"], r1["state"]) < 1e-15


def test_p1_per_mode_delta_mpmath(oracle_mod):
    q, k, v, delta, A, M = _modes_case(37, B=1, H=1, N=8, d=2, dv=2, M=3)
    r = oracle_mod.forward(q, k, v, delta, M, A=A)
    ref = _mp_brute(q[0, 0], k[0, 0], v[0, 0], delta[0], M, A=A)
    assert rel(r["o"][0, 0], ref) < 1e-12


def test_p8_finite_differences_per_mode_delta_and_A(oracle_mod):
    q, k, v, delta, A, M = _modes_case(41)
    H = delta.shape[0]
    dO = rnd(v.shape, 43)
    g = oracle_mod.backward(q, k, v, delta, dO, M, A=A)
    assert g["dDelta"].shape == delta.shape and g["dA"].shape == (2 * M,)

    def loss(d_, A_):
        return float(np.sum(dO * oracle_mod.forward(q, k, v, d_, M, A=A_)["o"]))

    h = 1e-7
    for hh in range(H):
        for m in range(M):
            dp = delta.copy(); dp[hh, m] += h
            dm = delta.copy(); dm[hh, m] -= h
            fd = (loss(dp, A) - loss(dm, A)) / (2 * h)
            assert abs(fd - g["dDelta"][hh, m]) <= 1e-6 * max(1.0, abs(fd)), (hh, m, fd, g["dDelta"][hh, m])
    for i in range(2 * M):      # d/dRe A_m and d/dIm A_m
        ap = A.copy(); ap[i] += h
        am = A.copy(); am[i] -= h
        fd = (loss(delta, ap) - loss(delta, am)) / (2 * h)
        assert abs(fd - g["dA"][i]) <= 1e-6 * max(1.0, abs(fd)), (i, fd, g["dA"][i])
    # S4D-Lin A as well (the default when A is not given)
    gl = oracle_mod.backward(q, k, v, delta, dO, M)
    A0 = np.empty(2 * M); A0[0::2] = -0.5; A0[1::2] = np.pi * np.arange(M)
    for i in (0, 3):
        ap = A0.copy(); ap[i] += h
        am = A0.copy(); am[i] -= h
        fd = (loss(delta, ap) - loss(delta, am)) / (2 * h)
        assert abs(fd - gl["dA"][i]) <= 1e-6 * max(1.0, abs(fd)), (i, fd, gl["dA"][i])


def test_p9_dot_product_per_mode_delta_and_A(oracle_mod):
    q, k, v, delta, A, M = _modes_case(47, B=2, H=3, N=70, d=4, dv=3, M=6)   # crosses a checkpoint
    dO = rnd(v.shape, 48)
    tq, tk, tv = rnd(q.shape, 49), rnd(k.shape, 50), rnd(v.shape, 51)
    td, tA = rnd(delta.shape, 52), rnd((2 * M,), 53)
    to = oracle_mod.jvp(q, k, v, delta, tq, tk, tv, td, M, A=A, tA=tA)
    g = oracle_mod.backward(q, k, v, delta, dO, M, A=A)
    lhs = float(np.sum(dO * to))
    rhs = float(np.sum(g["dq"] * tq) + np.sum(g["dk"] * tk) + np.sum(g["dv"] * tv)
                + np.sum(g["dDelta"] * td) + np.sum(g["dA"] * tA))
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), (lhs, rhs)
    # per-head Delta: the per-mode gradient summed over modes
    dh = delta[:, 0].copy()
    gh = oracle_mod.backward(q, k, v, dh, dO, M, A=A)
    gm = oracle_mod.backward(q, k, v, np.repeat(dh[:, None], M, axis=1), dO, M, A=A)
    assert rel(gm["dDelta"].sum(axis=1), gh["dDelta"]) < 1e-12 and rel(gm["dA"], gh["dA"]) < 1e-12


# ---------------------------------------------------------------- optional parts of the layer
def test_extended_forward_with_everything_off_is_the_layer(oracle_mod):
    q, k, v, delta, M = small_case(seed=60, N=45, M=6)
    a = oracle_mod.forward(q, k, v, delta, M)
    b = oracle_mod.forward_ex(q, k, v, M, delta=delta)
    assert rel(b["o"], a["o"]) < 1e-15 and rel(b["state"], a["state"]) < 1e-15


def _mp_brute_ex(q, k, v, M, steps, W=None):
    """Quadratic form in 40-digit mpmath for one (b,h) slice with one step per
    token (steps [N]) and an optional readout matrix W [M,M] complex:
        a_t[m]  = sum_{n<=t} b_n[m] exp(A_m sum_{s=n+1..t} Delta_s) s_tn
        a~_t    = W a_t
        w_tn    = Re sum_m conj(a~_t[m]) b_n[m] exp(A_m sum_{s=n+1..t} Delta_s)
        o_t     = sum_n w_tn v_n / sum_n w_tn."""
    import mpmath as mp
    mp.mp.dps = 40
    N, d = q.shape
    dv = v.shape[1]

    def xi(x):
        x = mp.mpf(float(x))
        return x + 1 if x > 0 else mp.e ** x

    fq = [[xi(q[t, f]) for f in range(d)] for t in range(N)]
    fk = [[xi(k[t, f]) for f in range(d)] for t in range(N)]
    A = [mp.mpc(-0.5, mp.pi * m) for m in range(M)]
    D = [mp.mpf(float(x)) for x in steps]
    cum = [mp.mpf(0)]
    for x in D:
        cum.append(cum[-1] + x)        # cum[t+1] = sum_{s<=t} Delta_s
    bn = [[(mp.e ** (D[n] * A[m]) - 1) / A[m] for m in range(M)] for n in range(N)]
    Wm = None if W is None else [[mp.mpc(float(W[i, j].real), float(W[i, j].imag)) for j in range(M)]
                                 for i in range(M)]
    out = []
    for t in range(N):
        s = [sum(fq[t][f] * fk[n][f] for f in range(d)) for n in range(t + 1)]
        dec = [[mp.e ** (A[m] * (cum[t + 1] - cum[n + 1])) for m in range(M)] for n in range(t + 1)]
        a = [sum(bn[n][m] * dec[n][m] * s[n] for n in range(t + 1)) for m in range(M)]
        at = a if Wm is None else [sum(Wm[i][j] * a[j] for j in range(M)) for i in range(M)]
        w = [sum((mp.conj(at[m]) * bn[n][m] * dec[n][m]).real for m in range(M)) for n in range(t + 1)]
        den = sum(w)
        out.append([float(sum(w[n] * v[n, j] for n in range(t + 1)) / den) for j in range(dv)])
    return np.array(out)


def test_selective_steps_mpmath(oracle_mod):
    q, k, v, _, M = small_case(seed=61, B=1, H=1, N=8, d=2, dv=2, M=3)
    steps = 0.01 + 0.3 * np.random.default_rng(62).random((1, 1, 8))
    r = oracle_mod.forward_ex(q, k, v, M, delta_t=steps)
    ref = _mp_brute_ex(q[0, 0], k[0, 0], v[0, 0], M, steps[0, 0])
    assert rel(r["o"][0, 0], ref) < 1e-12


def test_selective_constant_steps_reduce_to_per_head_delta(oracle_mod):
    q, k, v, delta, M = small_case(seed=63, N=40, M=5)
    B, H, N = q.shape[:3]
    steps = np.broadcast_to(delta[None, :, None], (B, H, N)).copy()
    a = oracle_mod.forward(q, k, v, delta, M)
    b = oracle_mod.forward_ex(q, k, v, M, delta_t=steps)
    assert rel(b["o"], a["o"]) < 1e-14 and rel(b["state"], a["state"]) < 1e-13


def test_selective_zero_step_skips_the_token(oracle_mod):
    # A token whose step goes to zero writes nothing (b -> 0) and leaves the
    # memory where it was (lambda -> 1): the other tokens' outputs match the
    # sequence with that token removed.
    q, k, v, _, M = small_case(seed=64, B=1, H=2, N=30, M=4)
    rng = np.random.default_rng(65)
    steps = 0.02 + 0.08 * rng.random((1, 2, 30))
    t0 = 12
    steps_gate = steps.copy()
    steps_gate[:, :, t0] = 1e-13
    r = oracle_mod.forward_ex(q, k, v, M, delta_t=steps_gate)
    drop = lambda x: np.delete(x, t0, axis=2)
    s = oracle_mod.forward_ex(drop(q), drop(k), drop(v), M, delta_t=drop(steps))
    # tokens before t0 are untouched; after t0 the skipped token's write is ~1e-13
    assert rel(np.delete(r["o"], t0, axis=2), s["o"]) < 1e-9


def test_readout_matrix_mpmath_and_identity(oracle_mod):
    q, k, v, _, M = small_case(seed=66, B=1, H=1, N=7, d=2, dv=2, M=3)
    rng = np.random.default_rng(67)
    W = rng.standard_normal((1, M, M)) + 1j * rng.standard_normal((1, M, M))
    delta = np.array([0.2])
    r = oracle_mod.forward_ex(q, k, v, M, delta=delta, W=W)
    ref = _mp_brute_ex(q[0, 0], k[0, 0], v[0, 0], M, np.full(7, 0.2), W=W[0])
    assert rel(r["o"][0, 0], ref) < 1e-11
    # the identity matrix is the plain readout
    q, k, v, delta, M = small_case(seed=68, N=30, M=5)
    eye = np.broadcast_to(np.eye(M, dtype=complex), (2, M, M)).copy()
    a = oracle_mod.forward(q, k, v, delta, M)
    b = oracle_mod.forward_ex(q, k, v, M, delta=delta, W=eye)
    assert rel(b["num"], a["num"]) < 1e-14 and rel(b["den"], a["den"]) < 1e-14


def test_readout_matrix_linear_and_scale_free(oracle_mod):
    q, k, v, delta, M = small_case(seed=69, N=33, M=4)
    rng = np.random.default_rng(70)
    W1 = rng.standard_normal((2, M, M)) + 1j * rng.standard_normal((2, M, M))
    W2 = rng.standard_normal((2, M, M)) + 1j * rng.standard_normal((2, M, M))
    f = lambda W: oracle_mod.forward_ex(q, k, v, M, delta=delta, W=W)
    r1, r2, r12 = f(W1), f(W2), f(W1 + W2)
    assert rel(r12["num"], r1["num"] + r2["num"]) < 1e-12 and rel(r12["den"], r1["den"] + r2["den"]) < 1e-12
    r3 = f(-2.5 * W1)                      # a real scale multiplies num and den alike
    assert rel(r3["num"], -2.5 * r1["num"]) < 1e-13 and rel(r3["o"], r1["o"]) < 1e-12


def test_input_norm_bias_alone_gives_the_bias(oracle_mod):
    # gain 0: the SSM input is the constant bias (beta_k, beta_v), so
    # Gamma_t = eta_t beta_v^T and num_t = den_t beta_v: o_t = beta_v for every t
    q, k, v, delta, M = small_case(seed=71, N=25, M=5)
    H, dx, dv = q.shape[1], q.shape[-1], v.shape[-1]
    bias = np.random.default_rng(72).standard_normal((H, dx + dv))
    r = oracle_mod.forward_ex(q, k, v, M, delta=delta, gain=np.zeros((H, dx + dv)), bias=bias)
    expect = np.broadcast_to(bias[None, :, None, dx:], r["o"].shape)
    assert rel(r["o"], expect) < 1e-12


def test_input_norm_is_scale_free(oracle_mod):
    # without bias, RMSNorm removes any positive per-token scale of the SSM
    # input (features given directly so that both halves scale together);
    # eps is negligible against the inputs' size
    q, k, v, delta, M = small_case(seed=73, N=28, M=4)
    fq, fk = feat(q), feat(k)
    H, dx, dv = q.shape[1], q.shape[-1], v.shape[-1]
    gain = 0.5 + np.random.default_rng(74).random((H, dx + dv))
    c = np.exp(np.random.default_rng(75).standard_normal(q.shape[:3] + (1,)))
    f = lambda kk, vv: oracle_mod.forward_ex(fq, kk, vv, M, delta=delta, gain=gain, eps=1e-30,
                                             map_features=False)["o"]
    assert rel(f(fk * c, v * c), f(fk, v)) < 1e-12
    # and it is not the identity: without the norm the scale matters
    plain = lambda kk, vv: oracle_mod.forward_ex(fq, kk, vv, M, delta=delta, map_features=False)["o"]
    assert rel(plain(fk * c, v * c), plain(fk, v)) > 1e-3


def test_bidirectional_time_reversal_and_first_token(oracle_mod):
    q, k, v, delta, M = small_case(seed=76, N=21, M=4)
    rng = np.random.default_rng(77)
    steps = 0.01 + 0.1 * rng.random(q.shape[:3])
    flip = lambda x: np.flip(x, axis=2).copy()
    o = oracle_mod.forward_bidirectional(q, k, v, M, delta_t=steps)
    o_r = oracle_mod.forward_bidirectional(flip(q), flip(k), flip(v), M, delta_t=flip(steps))
    assert rel(flip(o_r), o) < 1e-14
    # one token: each direction returns v (P3), so the sum is 2 v
    o1 = oracle_mod.forward_bidirectional(q[:, :, :1], k[:, :, :1], v[:, :, :1], M, delta=delta)
    assert rel(o1, 2 * v[:, :, :1]) < 1e-14
