"""Pin P7: the chunked re-association used by the kernels equals the plain
sequential recurrence (paperlayer.ai summary of 'Interdomain Attention',
sec. 3.2 and sec. A.2: chunkwise execution with state passing and a second
pass from corrected initial states).  fp64, CPU only."""
import numpy as np
import pytest

from chunk_algebra import chunk_pass, feat, segmented_pass


def rel(x, r):
    return float(np.max(np.abs(np.asarray(x) - np.asarray(r))) / np.max(np.abs(r)))


def case(seed, N, d=3, dv=2, M=5, delta=0.07):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 1, N, d)); k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, dv))
    return q, k, v, np.array([delta]), M


@pytest.mark.parametrize("C", [1, 2, 3, 16, 64])
@pytest.mark.parametrize("N", [1, 5, 64, 77, 130])
def test_p7_chunked_equals_sequential(oracle_mod, C, N):
    q, k, v, delta, M = case(C * 1000 + N, N)
    ref = oracle_mod.forward(q, k, v, delta, M)
    lam, b = oracle_mod.params(M, delta[0])
    o, num, den, (U, G, e) = chunk_pass(feat(q[0, 0]), feat(k[0, 0]), v[0, 0], lam, b, C)
    assert rel(num, ref["num"][0, 0]) < 1e-11
    assert rel(den, ref["den"][0, 0]) < 1e-11
    Ur, Gr, er = oracle_mod.split_state(ref["state"], 1, 1, M, q.shape[-1], v.shape[-1])
    assert rel(U, Ur[0, 0]) < 1e-11 and rel(G, Gr[0, 0]) < 1e-11 and rel(e, er[0, 0]) < 1e-11


def test_p7_chunked_with_state_in_and_fast_modes(oracle_mod):
    q, k, v, delta, M = case(3, 150, d=4, dv=3, M=64, delta=0.1)
    pre = oracle_mod.forward(q[:, :, :40], k[:, :, :40], v[:, :, :40], delta, M)
    ref = oracle_mod.forward(q[:, :, 40:], k[:, :, 40:], v[:, :, 40:], delta, M, state_in=pre["state"])
    U0, G0, e0 = oracle_mod.split_state(pre["state"], 1, 1, M, 4, 3)
    lam, b = oracle_mod.params(M, delta[0])
    o, num, den, _ = chunk_pass(feat(q[0, 0, 40:]), feat(k[0, 0, 40:]), v[0, 0, 40:], lam, b, 64,
                                S0=(U0[0, 0], G0[0, 0], e0[0, 0]))
    assert rel(num, ref["num"][0, 0]) < 1e-10
    assert rel(den, ref["den"][0, 0]) < 1e-10


@pytest.mark.parametrize("L,N", [(64, 200), (128, 384), (192, 500)])
def test_p7_segmented_two_pass(oracle_mod, L, N):
    q, k, v, delta, M = case(L + N, N, M=8, delta=0.02)
    ref = oracle_mod.forward(q, k, v, delta, M)
    lam, b = oracle_mod.params(M, delta[0])
    o, num, den, (U, G, e) = segmented_pass(feat(q[0, 0]), feat(k[0, 0]), v[0, 0], lam, b, 64, L)
    assert rel(num, ref["num"][0, 0]) < 1e-11
    assert rel(den, ref["den"][0, 0]) < 1e-11
    Ur, Gr, er = oracle_mod.split_state(ref["state"], 1, 1, M, 3, 2)
    assert rel(U, Ur[0, 0]) < 1e-11 and rel(e, er[0, 0]) < 1e-11


@pytest.mark.parametrize("N,C", [(150, 64), (64, 64), (37, 16), (100, 8)])
def test_p7_chunked_reverse_mode_equals_oracle_adjoint(oracle_mod, N, C):
    # the reverse mode of the chunked algorithm (table adjoints for Delta)
    # reproduces the oracle's sequential adjoint
    from chunk_algebra import chunk_backward
    rng = np.random.default_rng(N + C)
    d, dv, M = 5, 3, 7
    q = rng.standard_normal((1, 1, N, d)); k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, dv)); dO = rng.standard_normal((1, 1, N, dv))
    delta = np.array([0.06])
    ref = oracle_mod.backward(q, k, v, delta, dO, M)
    lam, b = oracle_mod.params(M, delta[0])
    A = -0.5 + 1j * np.pi * np.arange(M)
    o, dxq, dxk, dvv, dD = chunk_backward(feat(q[0, 0]), feat(k[0, 0]), v[0, 0], dO[0, 0], lam, b, A, delta[0], C)
    dfeat = lambda x: np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))
    assert rel(o, ref["o"][0, 0]) < 1e-10
    assert rel(dxq * dfeat(q[0, 0]), ref["dq"][0, 0]) < 1e-9
    assert rel(dxk * dfeat(k[0, 0]), ref["dk"][0, 0]) < 1e-9
    assert rel(dvv, ref["dv"][0, 0]) < 1e-9
    assert abs(dD - ref["dDelta"][0]) < 1e-9 * max(1.0, abs(ref["dDelta"][0]))


@pytest.mark.parametrize("N", [1, 64, 77, 200])
def test_p7_chunked_with_readout_matrix(oracle_mod, N):
    # the readout matrix in the chunked form (a = lambda^(i-c) a~, a~~ = W a,
    # X = lambda^(i-c) conj(a~~)) equals the oracle's extended forward with W,
    # also from a prefix's state; with fp16-rounded operands it stays within
    # the bf16 tolerance
    rng = np.random.default_rng(900 + N)
    d, dv, M, P = 4, 3, 6, 30
    q = rng.standard_normal((1, 1, P + N, d)); k = rng.standard_normal((1, 1, P + N, d))
    v = rng.standard_normal((1, 1, P + N, dv))
    delta = np.array([0.05])
    W = (rng.standard_normal((1, M, M)) + 1j * rng.standard_normal((1, M, M))) / np.sqrt(M) + np.eye(M)
    ref = oracle_mod.forward_ex(q, k, v, M, delta=delta, W=W)
    pre = oracle_mod.forward_ex(q[:, :, :P], k[:, :, :P], v[:, :, :P], M, delta=delta, W=W)
    U0, G0, e0 = oracle_mod.split_state(pre["state"], 1, 1, M, d, dv)
    lam, b = oracle_mod.params(M, delta[0])
    sl = slice(P, P + N)
    o, num, den, (U, G, e) = chunk_pass(feat(q[0, 0, sl]), feat(k[0, 0, sl]), v[0, 0, sl], lam, b, 64,
                                        S0=(U0[0, 0], G0[0, 0], e0[0, 0]), W=W[0])
    assert rel(num, ref["num"][0, 0, sl]) < 1e-10
    assert rel(den, ref["den"][0, 0, sl]) < 1e-10
    Ur, Gr, er = oracle_mod.split_state(ref["state"], 1, 1, M, d, dv)
    assert rel(U, Ur[0, 0]) < 1e-10 and rel(G, Gr[0, 0]) < 1e-10 and rel(e, er[0, 0]) < 1e-10
    f16 = lambda x: np.asarray(x, np.float16).astype(np.float64)
    _, num16, den16, _ = chunk_pass(feat(q[0, 0, sl]), feat(k[0, 0, sl]), v[0, 0, sl], lam, b, 64,
                                    S0=(U0[0, 0], G0[0, 0], e0[0, 0]), W=W[0], rnd=f16)
    assert rel(num16, ref["num"][0, 0, sl]) < 1e-2 and rel(den16, ref["den"][0, 0, sl]) < 1e-2


def test_p7_readout_matrix_identity_is_the_plain_chunked_form(oracle_mod):
    # W = I through the a -> a~~ -> X route gives the plain X = s conj(a~)
    rng = np.random.default_rng(7)
    N, d, dv, M = 100, 3, 2, 5
    fq, fk = feat(rng.standard_normal((N, d))), feat(rng.standard_normal((N, d)))
    v = rng.standard_normal((N, dv))
    lam, b = oracle_mod.params(M, 0.08)
    plain = chunk_pass(fq, fk, v, lam, b, 64)
    ident = chunk_pass(fq, fk, v, lam, b, 64, W=np.eye(M, dtype=complex))
    assert rel(ident[1], plain[1]) < 1e-12 and rel(ident[2], plain[2]) < 1e-12


@pytest.mark.parametrize("N", [1, 64, 77, 200])
def test_p7_chunked_with_steps_per_token(oracle_mod, N):
    # selective writing and memory decay in the chunked form: per-chunk
    # tables from the cumulative sum of the steps, the same contractions;
    # equals the oracle's extended forward with delta_t and a general A, from
    # a prefix's state, in fp64; fp16-rounded operands stay within 1e-2 over
    # the bench's step range [5e-3, 1e-1]
    from chunk_algebra import chunk_pass_selective
    rng = np.random.default_rng(1300 + N)
    d, dv, M, P = 4, 3, 6, 30
    q = rng.standard_normal((1, 1, P + N, d)); k = rng.standard_normal((1, 1, P + N, d))
    v = rng.standard_normal((1, 1, P + N, dv))
    dts = np.exp(np.log(5e-3) + rng.random((1, 1, P + N)) * (np.log(1e-1) - np.log(5e-3)))
    Ac = -(0.2 + 0.6 * rng.random(M)) + 1j * (np.pi * np.arange(M) + 0.7 * rng.random(M))
    A = np.empty(2 * M); A[0::2] = Ac.real; A[1::2] = Ac.imag
    ref = oracle_mod.forward_ex(q, k, v, M, A=A, delta_t=dts)
    pre = oracle_mod.forward_ex(q[:, :, :P], k[:, :, :P], v[:, :, :P], M, A=A, delta_t=dts[:, :, :P])
    U0, G0, e0 = oracle_mod.split_state(pre["state"], 1, 1, M, d, dv)
    sl = slice(P, P + N)
    args = (feat(q[0, 0, sl]), feat(k[0, 0, sl]), v[0, 0, sl], dts[0, 0, sl], Ac, 64)
    S0 = (U0[0, 0], G0[0, 0], e0[0, 0])
    o, num, den, (U, G, e) = chunk_pass_selective(*args, S0=S0)
    assert rel(num, ref["num"][0, 0, sl]) < 1e-10
    assert rel(den, ref["den"][0, 0, sl]) < 1e-10
    Ur, Gr, er = oracle_mod.split_state(ref["state"], 1, 1, M, d, dv)
    assert rel(U, Ur[0, 0]) < 1e-10 and rel(G, Gr[0, 0]) < 1e-10 and rel(e, er[0, 0]) < 1e-10
    f16 = lambda x: np.asarray(x, np.float16).astype(np.float64)
    _, num16, den16, _ = chunk_pass_selective(*args, S0=S0, rnd=f16)
    assert rel(num16, ref["num"][0, 0, sl]) < 1e-2 and rel(den16, ref["den"][0, 0, sl]) < 1e-2


def test_p7_steps_per_token_constant_step_is_the_plain_chunked_form(oracle_mod):
    # a constant step reduces the per-chunk tables to the per-head ones
    from chunk_algebra import chunk_pass_selective
    rng = np.random.default_rng(11)
    N, d, dv, M, delta = 150, 3, 2, 5, 0.07
    fq, fk = feat(rng.standard_normal((N, d))), feat(rng.standard_normal((N, d)))
    v = rng.standard_normal((N, dv))
    lam, b = oracle_mod.params(M, delta)
    Ac = -0.5 + 1j * np.pi * np.arange(M)
    plain = chunk_pass(fq, fk, v, lam, b, 64)
    sel = chunk_pass_selective(fq, fk, v, np.full(N, delta), Ac, 64)
    assert rel(sel[1], plain[1]) < 1e-11 and rel(sel[2], plain[2]) < 1e-11
    assert all(rel(x, y) < 1e-11 for x, y in zip(sel[3], plain[3]))
