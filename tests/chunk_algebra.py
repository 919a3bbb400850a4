"""The chunked form of the IA recurrence, in numpy fp64 -- test infrastructure.

The paper runs the S4D recurrence chunkwise (paperlayer.ai summary of
'Interdomain Attention', sec. 3.2 and sec. A.2: parallel work inside chunks of
64 tokens, states passed across chunk boundaries, a second pass recomputing
each chunk from its corrected initial state).  This file writes out the exact
re-association that the tensor-core kernels use, so that the algebra itself is
checked on the CPU against the sequential oracle (pin P7) before any kernel
runs.  It imports nothing from the CUDA path and the CUDA path imports nothing
from here.

Per (b,h), chunk length C, centre c = C // 2, positions i (query) and j (key)
in [0, C), tables per head:
    E'[j,m] = b_m lambda_m^(c-j)          s[i,m] = |lambda_m|^(2(i-c))
The running state is kept scaled, S_hat = lambda^-(C-c-1) S (U, Gamma, eta), so
that the state carried into a chunk and the decayed state it adds to are the
same product R = lambda^C S_hat0 = lambda^(c+1) S0.  For one chunk:
    a~[i]  = sum_{j<=i} S_ij E'[j] + R_U xi(q_i)          (a_i = lambda^(i-c) a~_i)
    X[i]   = s[i] conj(a~[i])                              (= conj(a_i) lambda^(i-c))
    P_ij   = Re sum_m X[i,m] E'[j,m],  masked j <= i
    num_i  = sum_j P_ij v_j + Re sum_m X[i,m] R_Gamma[m]
    den_i  = sum_j P_ij     + Re sum_m X[i,m] R_eta[m]
    S_hat1 = R + sum_j E'[j] x_j^T          (x = xi(k), v, 1)
With a complex readout matrix W (summary sec. A.3: a~~_i = W a_i before the
readout) the readout factor mixes modes, so X is formed from a itself:
    a[i]   = lambda^(i-c) a~[i];  a~~[i] = W a[i];  X[i] = lambda^(i-c) conj(a~~[i])
and P, num, den follow as above (the kernels' extra contraction G_W).
A ragged last chunk is zero-padded; its padded tokens add nothing but still
decay the state, which the end state undoes with lambda^(n_valid - C).
Segments: the local end states of equal segments of L tokens combine as
S_in(s+1) = lambda^L S_in(s) + S_local(s).
"""
import numpy as np


def feat(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def tables(lam, b, C):
    c = C // 2
    j = np.arange(C)
    Ep = b[None, :] * lam[None, :] ** (c - j[:, None])          # [C, M]
    s = np.abs(lam[None, :]) ** (2.0 * (j[:, None] - c))        # [C, M]
    return Ep, s, c


def chunk_pass(fq, fk, v, lam, b, C, S0=None, with_outputs=True, rnd=None, W=None):
    """One (b,h) sequence.  fq, fk [N,d], v [N,dv]; S0 = (U, G, eta) unscaled;
    W [M,M] complex, the readout matrix, or None.

    rnd, if given, is a function applied to every tensor-core operand (to
    emulate fp16/bf16 rounding); accumulations stay fp64 here.
    Returns (o, num, den, (U, G, eta)) with the end state unscaled."""
    N, d = fq.shape
    dv = v.shape[1]
    M = lam.shape[0]
    r = rnd if rnd is not None else (lambda x: x)
    Ep, s, c = tables(lam, b, C)
    sc = lam ** (C - c - 1)        # = lambda^(c-1) when C = 2c
    if S0 is None:
        Uh = np.zeros((M, d), complex); Gh = np.zeros((M, dv), complex); eh = np.zeros(M, complex)
    else:
        Uh, Gh, eh = (S0[0] / sc[:, None], S0[1] / sc[:, None], S0[2] / sc)
    lamC = lam ** C
    o = np.zeros((N, dv)); num = np.zeros((N, dv)); den = np.zeros(N)
    ii = np.arange(C)
    causal = ii[None, :] <= ii[:, None]                      # [i, j]
    Epr = r(Ep.real) + 1j * r(Ep.imag)
    nv = C
    for n0 in range(0, N, C):
        nv = min(C, N - n0)
        Q = np.zeros((C, d)); K = np.zeros((C, d)); V = np.zeros((C, dv)); one = np.zeros(C)
        Q[:nv] = fq[n0:n0 + nv]; K[:nv] = fk[n0:n0 + nv]; V[:nv] = v[n0:n0 + nv]; one[:nv] = 1.0
        Q, K, V = r(Q), r(K), r(V)
        RU, RG, Re_ = lamC[:, None] * Uh, lamC[:, None] * Gh, lamC * eh
        if with_outputs:
            S = Q @ K.T
            Sb = r(np.where(causal & (ii[None, :] < nv), S, 0.0))
            RUr = r(RU.real) + 1j * r(RU.imag)
            at = Sb @ Epr + Q @ RUr.T                            # a~ [C, M]
            if W is None:
                X = s * np.conj(at)
            else:
                lic = lam[None, :] ** (ii[:, None] - c)          # lambda^(i-c) [C, M]
                a = lic * at
                aw = (r(a.real) + 1j * r(a.imag)) @ (r(W.real) + 1j * r(W.imag)).T   # a~~ = W a
                X = lic * np.conj(aw)
            Xr = r(X.real) + 1j * r(X.imag)
            P = np.where(causal, (Xr @ Epr.T).real, 0.0)
            Pr = r(P)
            RGr = r(RG.real) + 1j * r(RG.imag)
            Rer = r(Re_.real) + 1j * r(Re_.imag)
            nm = Pr @ V + (Xr @ RGr).real
            dn = Pr @ one + (Xr @ Rer).real
            o[n0:n0 + nv] = nm[:nv] / dn[:nv, None]
            num[n0:n0 + nv] = nm[:nv]
            den[n0:n0 + nv] = dn[:nv]
        Uh = RU + Epr.T @ K
        Gh = RG + Epr.T @ V
        eh = Re_ + Epr.T @ one
    fix = lam ** (nv - C) if N > 0 else np.ones_like(lam)
    end = (sc[:, None] * fix[:, None] * Uh, sc[:, None] * fix[:, None] * Gh, sc * fix * eh)
    return o, num, den, end


def chunk_pass_selective(fq, fk, v, dts, A, C, S0=None, rnd=None):
    """The chunked form with a step per token (selective writing and memory
    decay, summary sec. 3.3): lambda_t = exp(Delta_t A), b_t = (lambda_t - 1)/A.
    With cs the inclusive cumulative sum of Delta_t inside a chunk, the decay
    from token j to token i is exp(A (cs_i - cs_j)) = exp(A (cs_i - cs_c))
    exp(A (cs_c - cs_j)), so the plain chunk algebra holds with tables per
    chunk instead of per head:
        E'_t[j,m] = b_{j,m} exp(A_m (cs_c - cs_j))
        s_t[i,m]  = |exp(A_m (cs_i - cs_c))|^2
        R         = exp(A cs_c) S0       end: exp(A (cs_last - cs_c)) (R + E'_t^T x)
    Padded tokens take Delta = 0 (lambda = 1, b = 0): they neither write nor
    decay, so a ragged chunk needs no end correction.  The state is kept
    unscaled here.  fq, fk [N,d], v [N,dv], dts [N], A [M] complex."""
    N, d = fq.shape
    dv = v.shape[1]
    M = A.shape[0]
    c = C // 2
    r = rnd if rnd is not None else (lambda x: x)
    if S0 is None:
        U = np.zeros((M, d), complex); G = np.zeros((M, dv), complex); eta = np.zeros(M, complex)
    else:
        U, G, eta = (np.array(x, complex) for x in S0)
    o = np.zeros((N, dv)); num = np.zeros((N, dv)); den = np.zeros(N)
    ii = np.arange(C)
    causal = ii[None, :] <= ii[:, None]
    for n0 in range(0, N, C):
        nv = min(C, N - n0)
        Q = np.zeros((C, d)); K = np.zeros((C, d)); V = np.zeros((C, dv)); one = np.zeros(C); dt = np.zeros(C)
        Q[:nv] = fq[n0:n0 + nv]; K[:nv] = fk[n0:n0 + nv]; V[:nv] = v[n0:n0 + nv]; one[:nv] = 1.0
        dt[:nv] = dts[n0:n0 + nv]
        Q, K, V = r(Q), r(K), r(V)
        cs = np.cumsum(dt)
        lam_t = np.exp(dt[:, None] * A[None, :])
        b_t = (lam_t - 1.0) / A[None, :]
        Ep = b_t * np.exp(A[None, :] * (cs[c] - cs[:, None]))
        Epr = r(Ep.real) + 1j * r(Ep.imag)
        s = np.abs(np.exp(A[None, :] * (cs[:, None] - cs[c]))) ** 2
        rc = np.exp(A * cs[c])
        RU, RG, Re_ = rc[:, None] * U, rc[:, None] * G, rc * eta
        S = Q @ K.T
        Sb = r(np.where(causal & (ii[None, :] < nv), S, 0.0))
        RUr = r(RU.real) + 1j * r(RU.imag)
        at = Sb @ Epr + Q @ RUr.T
        X = s * np.conj(at)
        Xr = r(X.real) + 1j * r(X.imag)
        P = r(np.where(causal, (Xr @ Epr.T).real, 0.0))
        RGr = r(RG.real) + 1j * r(RG.imag)
        Rer = r(Re_.real) + 1j * r(Re_.imag)
        nm = P @ V + (Xr @ RGr).real
        dn = P @ one + (Xr @ Rer).real
        o[n0:n0 + nv] = nm[:nv] / dn[:nv, None]
        num[n0:n0 + nv] = nm[:nv]
        den[n0:n0 + nv] = dn[:nv]
        rend = np.exp(A * (cs[-1] - cs[c]))
        U = rend[:, None] * (RU + Epr.T @ K)
        G = rend[:, None] * (RG + Epr.T @ V)
        eta = rend * (Re_ + Epr.T @ one)
    return o, num, den, (U, G, eta)


def segmented_pass(fq, fk, v, lam, b, C, L):
    """Two-pass form over segments of L tokens (L a multiple of C):
    local end states from zero, an exclusive scan of the carries, then every
    segment recomputed from its carry-in."""
    N = fq.shape[0]
    starts = list(range(0, N, L))
    local = []
    for s0 in starts[:-1]:
        _, _, _, end = chunk_pass(fq[s0:s0 + L], fk[s0:s0 + L], v[s0:s0 + L], lam, b, C,
                                  with_outputs=False)
        local.append(end)
    M, d, dv = lam.shape[0], fq.shape[1], v.shape[1]
    carry = (np.zeros((M, d), complex), np.zeros((M, dv), complex), np.zeros(M, complex))
    lamL = lam ** L
    outs = []
    for si, s0 in enumerate(starts):
        o, num, den, end = chunk_pass(fq[s0:s0 + L], fk[s0:s0 + L], v[s0:s0 + L], lam, b, C, S0=carry)
        outs.append((o, num, den))
        if si < len(local):
            carry = tuple(lamL.reshape((-1,) + (1,) * (x.ndim - 1)) * x + y
                          for x, y in zip(carry, local[si]))
    o = np.concatenate([x[0] for x in outs]); num = np.concatenate([x[1] for x in outs])
    den = np.concatenate([x[2] for x in outs])
    return o, num, den, end


# ----------------------------------------------------------------------------
# Reverse mode of the chunked form, in the real-row representation the
# kernels use: complex rows become k = 2m (re), 2m+1 (im); the per-mode decay
# rotation Rot(z) acts on each (re, im) row pair.  Per chunk, with x = [xi(K) | V]:
#   R = Rot(lambda^C) S_hat0;  a~ = S E'' + xi(Q) R_U^T;  X = s * a~
#   P = mask(X E''^T);  num = P V + X R_G;  den = P 1 + X R_eta;  o = num/den
#   S_hat1 = R + E''^T x
# Backward from dO and the adjoint of S_hat1 (the reverse carry):
#   dnum = dO/den;  dden = -(dO . o)/den;  dP = mask(dnum V^T + dden 1^T)
#   dV = P^T dnum + E'' dS1_G;   dX = dP E'' + dnum R_G^T + dden R_eta^T
#   dR_G = X^T dnum;  dR_eta = X^T dden;  da~ = s * dX;  dS = mask(da~ E''^T)
#   dxiQ = dS xi(K) + da~ R_U;  dxiK = dS^T xi(Q) + E'' dS1_U;  dR_U = da~^T xi(Q)
#   dS_hat0 = Rot(lambda^C)^T (dS1 + [dR_U | dR_G | dR_eta])
# Delta enters only through the per-head tables, so their adjoints are summed
# over every chunk and contracted once with the tables' Delta-derivatives:
#   dE'' += S^T da~ + dP^T X + x dS1^T,  ds += dX * a~,  dlambda^C += sum R conj(S_hat0)
#   d(b lambda^n)/dDelta = (lambda + n A b) lambda^n,  ds/dDelta = 2 Re(A)(i-c) s,
#   d(lambda^C)/dDelta = C A lambda^C.
# ----------------------------------------------------------------------------
def _rows(z):
    """complex [..., M] -> real rows [..., 2M] interleaved (re, im)."""
    out = np.empty(z.shape[:-1] + (2 * z.shape[-1],))
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def _rot(z, Y):
    """Apply the per-mode complex factor z [M] to real rows Y [2M, F]."""
    re, im = Y[0::2], Y[1::2]
    zr, zi = z.real[:, None], z.imag[:, None]
    out = np.empty_like(Y)
    out[0::2] = zr * re - zi * im
    out[1::2] = zi * re + zr * im
    return out


def chunk_backward(fq, fk, v, dO, lam, b, A, delta, C=64):
    """Reverse mode of chunk_pass from a zero state for one (b,h) sequence.

    Returns (o, dxiQ, dxiK, dV, dDelta) -- the feature gradients before the
    xi' factor."""
    N, d = fq.shape
    dv_ = v.shape[1]
    M = lam.shape[0]
    c = C // 2
    j = np.arange(C)
    Ep = b[None, :] * lam[None, :] ** (c - j[:, None])
    E2 = _rows(Ep)                                           # [C, 2M]
    s = np.abs(lam[None, :]) ** (2.0 * (j[:, None] - c))
    s2 = np.repeat(s, 2, axis=1)                             # [C, 2M]
    lamC = lam ** C
    causal = (j[None, :] <= j[:, None]).astype(float)
    nch = (N + C - 1) // C
    # forward, keeping the state at every chunk start
    Sh = np.zeros((2 * M, d + dv_))
    eh = np.zeros(2 * M)
    starts = []
    o = np.zeros((N, dv_))
    for ch in range(nch):
        n0 = ch * C
        nv = min(C, N - n0)
        starts.append((Sh.copy(), eh.copy()))
        Q = np.zeros((C, d)); K = np.zeros((C, d)); V = np.zeros((C, dv_)); one = np.zeros(C)
        Q[:nv] = fq[n0:n0 + nv]; K[:nv] = fk[n0:n0 + nv]; V[:nv] = v[n0:n0 + nv]; one[:nv] = 1
        R = _rot(lamC, Sh)
        Re = _rot(lamC, eh[:, None])[:, 0]
        Mk = causal * (j[None, :] < nv)
        Sb = (Q @ K.T) * Mk
        at = Sb @ E2 + Q @ R[:, :d].T
        X = s2 * at
        P = (X @ E2.T) * causal
        num = P @ V + X @ R[:, d:]
        den = P @ one + X @ Re
        o[n0:n0 + nv] = num[:nv] / den[:nv, None]
        Sh = R + E2.T @ np.concatenate([K, V], axis=1)
        eh = Re + E2.T @ one
    # backward
    dq = np.zeros((N, d)); dk = np.zeros((N, d)); dvv = np.zeros((N, dv_))
    dS1 = np.zeros((2 * M, d + dv_)); de1 = np.zeros(2 * M)
    dE2 = np.zeros_like(E2); ds2 = np.zeros_like(s2); dlamC = np.zeros(M, complex)
    for ch in reversed(range(nch)):
        n0 = ch * C
        nv = min(C, N - n0)
        Sh0, eh0 = starts[ch]
        Q = np.zeros((C, d)); K = np.zeros((C, d)); V = np.zeros((C, dv_)); one = np.zeros(C)
        G = np.zeros((C, dv_)); Oc = np.zeros((C, dv_))
        Q[:nv] = fq[n0:n0 + nv]; K[:nv] = fk[n0:n0 + nv]; V[:nv] = v[n0:n0 + nv]; one[:nv] = 1
        G[:nv] = dO[n0:n0 + nv]; Oc[:nv] = o[n0:n0 + nv]
        R = _rot(lamC, Sh0)
        Re = _rot(lamC, eh0[:, None])[:, 0]
        Mk = causal * (j[None, :] < nv)
        Sb = (Q @ K.T) * Mk
        at = Sb @ E2 + Q @ R[:, :d].T
        X = s2 * at
        P = (X @ E2.T) * causal
        den = P @ one + X @ Re
        den_safe = np.where(np.arange(C) < nv, den, 1.0)
        dnum = G / den_safe[:, None]
        dden = -(G * Oc).sum(1) / den_safe
        dP = (dnum @ V.T + dden[:, None] * one[None, :]) * causal
        dV = P.T @ dnum + E2 @ dS1[:, d:]
        dX = dP @ E2 + dnum @ R[:, d:].T + dden[:, None] * Re[None, :]
        dRG = X.T @ dnum
        dRe = X.T @ dden
        dat = s2 * dX
        dSm = (dat @ E2.T) * Mk
        dRU = dat.T @ Q
        dQ = dSm @ K + dat @ R[:, :d]
        dK = dSm.T @ Q + E2 @ dS1[:, :d]
        x = np.concatenate([K, V], axis=1)
        dE2 += Sb.T @ dat + dP.T @ X + x @ dS1.T + one[:, None] * de1[None, :]
        ds2 += dX * at
        dR = dS1 + np.concatenate([dRU, dRG], axis=1)
        dRe_tot = de1 + dRe
        # adjoint of R = lambda^C S_hat0:  dlambda^C += sum conj(S_hat0) dR  (complex form)
        Sc = Sh0[0::2] + 1j * Sh0[1::2]
        Rc = dR[0::2] + 1j * dR[1::2]
        dlamC += (Rc * np.conj(Sc)).sum(1) + (dRe_tot[0::2] + 1j * dRe_tot[1::2]) * np.conj(eh0[0::2] + 1j * eh0[1::2])
        dS1 = _rot(np.conj(lamC), dR)
        de1 = _rot(np.conj(lamC), dRe_tot[:, None])[:, 0]
        dq[n0:n0 + nv] = dQ[:nv]; dk[n0:n0 + nv] = dK[:nv]; dvv[n0:n0 + nv] = dV[:nv]
    # Delta through the tables
    dEc = dE2[:, 0::2] + 1j * dE2[:, 1::2]
    dEp = lam[None, :] * lam[None, :] ** (c - j[:, None]) + (c - j[:, None]) * A[None, :] * Ep
    ds = ds2[:, 0::2] + ds2[:, 1::2]
    dsd = 2.0 * A.real[None, :] * (j[:, None] - c) * s
    dD = float(np.sum((np.conj(dEc) * dEp).real) + np.sum(ds * dsd)
               + np.sum((np.conj(dlamC) * C * A * lamC).real))
    return o, dq, dk, dvv, dD
