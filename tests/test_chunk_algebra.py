"""The chunkwise-parallel algebra the CUDA kernels implement, restated in fp64
numpy and checked against the token-by-token oracle.

This isolates mistakes in the chunk derivation from mistakes in the kernels.
Derivation ("Gated DeltaNet-2" page, 高效训练 / WY 形式; scalar decay for GDN):
within a chunk with cumulative log-decay G_r and start state S0,

    S_r = Diag(gamma_r) S0 + sum_{j<=r} Diag(gamma_r / gamma_j) k_j u_j^T,

where the pseudo-values u solve (I + L) U~ = Z - E_gamma S0 with
L_rj = sum_i e_r[i] k_j[i] exp(G_r[i] - G_j[i]) for j < r.  With A = (I + L)^-1,
Y = A E_gamma and U = A Z:  U~ = U - Y S0,
O = Q_gamma S0 + tril(A_qk) U~ with A_qk_rj = sum_i q_r[i] k_j[i] exp(G_r[i] - G_j[i]),
S_C = Diag(gamma_C) S0 + K_tail^T U~ with K_tail rows (gamma_C / gamma_j) (.) k_j.
GDN is the case e = beta k, z = beta v, scalar decay.

Only exponents of non-positive numbers are ever formed (exp(G_r - G_j) with
j <= r, exp(G_r), exp(G_C - G_j)), which is what keeps the kernels free of
overflow.  For channel-wise decay the two C x C products are formed per block of
16 rows against a reference point at the block's start (the off-diagonal
blocks) and directly (the diagonal blocks), as the GDN-2 kernel does.
"""
import math

import numpy as np
import pytest

from oracle import oracle as O

rng = np.random.default_rng(7)


def forward_substitution_inverse(L):
    """(I + L)^-1 for strictly lower-triangular L, one row at a time."""
    C = L.shape[0]
    X = np.zeros_like(L)
    for r in range(C):
        X[r] = -L[r] @ X
        X[r, r] = 1.0
    return X


def chunk_gdn(q, k, v, g, beta, S0, C):
    """Scalar-decay chunk form. q,k [T,dk] (already normalised/scaled), v [T,dv],
    g, beta [T]. Returns o [T,dv], S_T."""
    T = q.shape[0]
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(c0 + C, T)
        Kc, Qc, Vc = k[c0:c1], q[c0:c1], v[c0:c1]
        G = np.cumsum(g[c0:c1])
        bc = beta[c0:c1]
        n = c1 - c0
        diff = G[:, None] - G[None, :]
        Gam = np.exp(np.where(np.tril(np.ones((n, n))) > 0, diff, -np.inf))
        L = np.tril(bc[:, None] * (Kc @ Kc.T) * Gam, -1)
        A = forward_substitution_inverse(L)
        W = A @ ((bc * np.exp(G))[:, None] * Kc)
        U = A @ (bc[:, None] * Vc)
        Aqk = np.tril((Qc @ Kc.T) * Gam)
        Unew = U - W @ S
        o[c0:c1] = (np.exp(G)[:, None] * Qc) @ S + Aqk @ Unew
        S = math.exp(G[-1]) * S + (np.exp(G[-1] - G)[:, None] * Kc).T @ Unew
    return o, S


def chunk_gdn2(q, k, v, g, b, w, S0, C, sub=16):
    """Channel-decay chunk form with 16-row sub-blocks. g, b [T,dk]; w [T,dv]."""
    T, dk = q.shape
    S = S0.copy()
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(c0 + C, T)
        n = c1 - c0
        Kc, Qc = k[c0:c1], q[c0:c1]
        G = np.cumsum(g[c0:c1], axis=0)                 # [n, dk]
        E = b[c0:c1] * Kc                                # erase directions
        Z = w[c0:c1] * v[c0:c1]
        Lfull = np.zeros((n, n))
        Aqk = np.zeros((n, n))
        for p0 in range(0, n, sub):
            p1 = min(p0 + sub, n)
            # diagonal block: direct masked contraction, exp(G_r - G_j) <= 1
            for r in range(p0, p1):
                for j in range(p0, r + 1):
                    f = np.exp(G[r] - G[j])
                    if j < r:
                        Lfull[r, j] = np.sum(E[r] * Kc[j] * f)
                    Aqk[r, j] = np.sum(Qc[r] * Kc[j] * f)
            if p0 == 0:
                continue
            # off-diagonal blocks: reference at the last row before the block
            ref = G[p0 - 1]
            left_e = E[p0:p1] * np.exp(G[p0:p1] - ref)   # factors <= 1
            left_q = Qc[p0:p1] * np.exp(G[p0:p1] - ref)
            right = Kc[:p0] * np.exp(ref - G[:p0])        # factors <= 1
            Lfull[p0:p1, :p0] = left_e @ right.T
            Aqk[p0:p1, :p0] = left_q @ right.T
        A = forward_substitution_inverse(Lfull)
        gam = np.exp(G)
        Y = A @ (gam * E)
        U = A @ Z
        Unew = U - Y @ S
        o[c0:c1] = (gam * Qc) @ S + Aqk @ Unew
        S = np.exp(G[-1])[:, None] * S + (np.exp(G[-1] - G) * Kc).T @ Unew
    return o, S


def chunk_gdn_bwd(q, k, v, g, beta, S0, dO, dST, C):
    """Backward of the scalar-decay chunk form above: the derivation a chunkwise
    backward follows.  Chunks are taken from the last, the state gradient carried
    from each chunk to the one before; a chunk's start state comes from the
    forward chunk recurrence.  Per chunk, with K~ = diag(gamma_C / gamma) K,
    U~ = U - W S0, O = diag(gamma) Q S0 + A_qk U~ and S1 = gamma_C S0 + K~^T U~,
    the gradients run back through U = A diag(beta) V, W = A diag(beta gamma) K,
    A = (I + L)^-1 (dL = -A^T dA A^T, kept strictly lower), the Gamma masks and
    G = cumsum(g) (dg = reverse cumulative sum of dG).
    Returns dq, dk, dv, dg, dbeta and the gradient of the initial state."""
    T, dk = q.shape
    starts, S = [], S0.copy()
    for c0 in range(0, T, C):
        starts.append(S.copy())
        _, S = chunk_gdn(q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], g[c0:c0 + C],
                         beta[c0:c0 + C], S, C)
    dq, dk_, dv_ = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, dbeta = np.zeros(T), np.zeros(T)
    dS = dST.copy()
    for ci in reversed(range(len(starts))):
        c0 = ci * C
        c1 = min(c0 + C, T)
        n = c1 - c0
        Kc, Qc, Vc, bc, S = k[c0:c1], q[c0:c1], v[c0:c1], beta[c0:c1], starts[ci]
        G = np.cumsum(g[c0:c1])
        gam = np.exp(G)
        gC = gam[-1]
        low = np.tril(np.ones((n, n)))
        Gam = np.exp(np.where(low > 0, G[:, None] - G[None, :], -np.inf))
        KK, QK = Kc @ Kc.T, Qc @ Kc.T
        M = KK * Gam
        L = np.tril(bc[:, None] * M, -1)
        A = forward_substitution_inverse(L)
        Kb, Vb = (bc * gam)[:, None] * Kc, bc[:, None] * Vc
        W, U = A @ Kb, A @ Vb
        Aqk = np.tril(QK * Gam)
        Ut = U - W @ S
        ratio = gC / gam
        Kt = ratio[:, None] * Kc
        # S1 = gamma_C S0 + K~^T U~
        dS0 = gC * dS
        dgC = float(np.sum(dS * S))
        dKt, dUt = Ut @ dS.T, Kt @ dS
        # O = diag(gamma) Q S0 + A_qk U~
        dOc = dO[c0:c1]
        dgam = np.sum(dOc * (Qc @ S), axis=1)
        dQ = gam[:, None] * (dOc @ S.T)
        dS0 += (gam[:, None] * Qc).T @ dOc
        dAqk = np.tril(dOc @ Ut.T)
        dUt += Aqk.T @ dOc
        # U~ = U - W S0
        dU, dW = dUt, -dUt @ S.T
        dS0 -= W.T @ dUt
        # U = A Vb, W = A Kb
        dA = dU @ Vb.T + dW @ Kb.T
        dVb, dKb = A.T @ dU, A.T @ dW
        dV = bc[:, None] * dVb
        db = np.sum(dVb * Vc, axis=1)
        dK = (bc * gam)[:, None] * dKb
        dbg = np.sum(dKb * Kc, axis=1)
        db += dbg * gam
        dgam += dbg * bc
        # A = (I + L)^-1, L = tril(diag(beta) (K K^T o Gamma), -1)
        dL = np.tril(-A.T @ dA @ A.T, -1)
        db += np.sum(dL * M, axis=1)
        dM = bc[:, None] * dL
        dKK, dGam = dM * Gam, dM * KK
        dK += (dKK + dKK.T) @ Kc
        # A_qk = tril(Q K^T o Gamma)
        dQK = dAqk * Gam
        dGam += dAqk * QK
        dQ += dQK @ Kc
        dK += dQK.T @ Qc
        # K~ = diag(gamma_C / gamma) K
        dK += ratio[:, None] * dKt
        dratio = np.sum(dKt * Kc, axis=1)
        # G: Gamma_rj = exp(G_r - G_j), gamma = exp(G), ratio = exp(G_C - G), gamma_C
        tG = dGam * Gam
        dG = tG.sum(1) - tG.sum(0) + dgam * gam - dratio * ratio
        dG[-1] += float(np.sum(dratio * ratio)) + dgC * gC
        dg[c0:c1] = np.cumsum(dG[::-1])[::-1]
        dq[c0:c1], dk_[c0:c1], dv_[c0:c1], dbeta[c0:c1] = dQ, dK, dV, db
        dS = dS0
    return dq, dk_, dv_, dg, dbeta, dS


def chunk_gdn2_bwd(q, k, v, g, b, w, S0, dO, dST, C):
    """Backward of the channel-decay chunk form, written with the direct masked
    contractions L_rj = sum_c E_rc K_jc Gamma_rjc (j < r) and
    A_qk_rj = sum_c Q_rc K_jc Gamma_rjc (j <= r), Gamma_rjc = exp(G_rc - G_jc) (the
    blocked form of the forward is the same numbers).  Per chunk, with
    E-bar = gamma (.) E, Y = A E-bar, U = A Z, U~ = U - Y S0,
    O = (gamma (.) Q) S0 + A_qk U~ and S1 = diag(gamma_C) S0 + K~^T U~,
    dA = dU Z^T + dY E-bar^T ("Gated DeltaNet-2", Gate-aware 反向传播), then
    dL = -A^T dA A^T (strictly lower), the masked contractions, the Gamma tensor and
    the per-channel reverse cumulative sum for dg."""
    T, dk = q.shape
    starts, S = [], S0.copy()
    for c0 in range(0, T, C):
        starts.append(S.copy())
        _, S = chunk_gdn2(q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], g[c0:c0 + C],
                          b[c0:c0 + C], w[c0:c0 + C], S, C)
    dq, dk_, dv_ = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, db, dw = np.zeros_like(g), np.zeros_like(b), np.zeros_like(w)
    dS = dST.copy()
    for ci in reversed(range(len(starts))):
        c0 = ci * C
        c1 = min(c0 + C, T)
        n = c1 - c0
        Kc, Qc, Vc, S = k[c0:c1], q[c0:c1], v[c0:c1], starts[ci]
        bc, wc = b[c0:c1], w[c0:c1]
        G = np.cumsum(g[c0:c1], axis=0)
        gam = np.exp(G)
        gC = gam[-1]
        low = np.tril(np.ones((n, n)))
        Gam = np.exp(np.where(low[:, :, None] > 0, G[:, None, :] - G[None, :, :], -np.inf))
        E, Z = bc * Kc, wc * Vc
        L = np.tril(np.einsum("rc,jc,rjc->rj", E, Kc, Gam), -1)
        Aqk = np.tril(np.einsum("rc,jc,rjc->rj", Qc, Kc, Gam))
        A = forward_substitution_inverse(L)
        Eb = gam * E
        Y, U = A @ Eb, A @ Z
        Ut = U - Y @ S
        ratio = gC[None, :] / gam
        Kt = ratio * Kc
        # S1 = diag(gamma_C) S0 + K~^T U~
        dS0 = gC[:, None] * dS
        dgC = np.sum(dS * S, axis=1)
        dKt, dUt = Ut @ dS.T, Kt @ dS
        # O = (gamma (.) Q) S0 + A_qk U~
        dOc = dO[c0:c1]
        dQg = dOc @ S.T
        dQ = gam * dQg
        dgam = Qc * dQg
        dS0 += (gam * Qc).T @ dOc
        dAqk = np.tril(dOc @ Ut.T)
        dUt += Aqk.T @ dOc
        # U~ = U - Y S0 ; U = A Z ; Y = A E-bar
        dU, dY = dUt, -dUt @ S.T
        dS0 -= Y.T @ dUt
        dA = dU @ Z.T + dY @ Eb.T
        dZ, dEb = A.T @ dU, A.T @ dY
        dV = wc * dZ
        dwc = Vc * dZ
        dE = gam * dEb
        dgam += E * dEb
        dL = np.tril(-A.T @ dA @ A.T, -1)
        # the masked contractions
        dE += np.einsum("rj,jc,rjc->rc", dL, Kc, Gam)
        dK = np.einsum("rj,rc,rjc->jc", dL, E, Gam) + np.einsum("rj,rc,rjc->jc", dAqk, Qc, Gam)
        dQ += np.einsum("rj,jc,rjc->rc", dAqk, Kc, Gam)
        tG = (np.einsum("rj,rc,jc->rjc", dL, E, Kc) + np.einsum("rj,rc,jc->rjc", dAqk, Qc, Kc)) * Gam
        dG = tG.sum(1) - tG.sum(0)
        # E = b (.) K
        dbc = Kc * dE
        dK += bc * dE
        # K~ = (gamma_C / gamma) (.) K
        dK += ratio * dKt
        dratio = Kc * dKt
        dG -= dratio * ratio
        dG[-1] += np.sum(dratio * ratio, axis=0) + dgC * gC
        dG += dgam * gam
        dg[c0:c1] = np.cumsum(dG[::-1], axis=0)[::-1]
        dq[c0:c1], dk_[c0:c1], dv_[c0:c1], db[c0:c1], dw[c0:c1] = dQ, dK, dV, dbc, dwc
        dS = dS0
    return dq, dk_, dv_, dg, db, dw, dS


def _gates(T, H, A_log, dt_bias, a, b):
    sp = np.log1p(np.exp(a + dt_bias))
    return -np.exp(A_log) * sp, 1 / (1 + np.exp(-b))


@pytest.mark.parametrize("T", [1, 37, 64, 65, 200])
@pytest.mark.parametrize("C", [1, 16, 64])
def test_chunk_gdn_equals_token_oracle(T, C):
    dk, dv = 16, 8
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    q /= np.linalg.norm(q, axis=1, keepdims=True) * 4.0
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    g = -rng.uniform(0.0, 3.0, size=T)
    beta = rng.uniform(0.0, 1.0, size=T)
    S0 = 0.1 * rng.standard_normal((dk, dv))
    o_ref, S_ref = O.gdn_fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                             g[None, :, None], beta[None, :, None], h0=S0[None, None],
                             scale=1.0, l2norm=False, gates_given=True)
    o, S = chunk_gdn(q, k, v, g, beta, S0, C)
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("T", [1, 30, 64, 100])
def test_chunk_gdn2_equals_token_oracle(T):
    dk, dv = 16, 8
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    q /= np.linalg.norm(q, axis=1, keepdims=True) * 4.0
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    # include very fast channels: cumulative decay of several hundred in a chunk
    g = -rng.uniform(0.0, 1.0, size=(T, dk)) * np.linspace(0.1, 40.0, dk)
    b = rng.uniform(0.0, 1.0, size=(T, dk))
    w = rng.uniform(0.0, 1.0, size=(T, dv))
    S0 = 0.1 * rng.standard_normal((dk, dv))
    o_ref, S_ref = O.gdn2_fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                              g[None, :, None], b[None, :, None], w[None, :, None],
                              h0=S0[None, None], scale=1.0, l2norm=False, gates_given=True)
    o, S = chunk_gdn2(q, k, v, g, b, w, S0, 64)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=1e-9, atol=1e-10)


def test_scalar_gates_through_gdn2_chunk_form():
    """The GDN-2 chunk form with b = w = beta 1 and equal channel decay is the
    GDN chunk form."""
    T, dk, dv = 70, 16, 8
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    g = -rng.uniform(0.0, 2.0, size=T)
    beta = rng.uniform(0.0, 1.0, size=T)
    S0 = 0.1 * rng.standard_normal((dk, dv))
    o1, S1 = chunk_gdn(q, k, v, g, beta, S0, 64)
    o2, S2 = chunk_gdn2(q, k, v, np.repeat(g[:, None], dk, 1), np.repeat(beta[:, None], dk, 1),
                        np.repeat(beta[:, None], dv, 1), S0, 64)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S2, S1, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T", [1, 37, 64, 130])
@pytest.mark.parametrize("C", [1, 16, 64])
def test_chunk_gdn_backward_equals_token_backward(T, C):
    """The chunkwise backward against the oracle's token-by-token backward (itself
    pinned by finite differences), same gates and normalised keys."""
    dk, dv = 16, 8
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    q /= np.linalg.norm(q, axis=1, keepdims=True) * 4.0
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    g = -rng.uniform(0.0, 3.0, size=T)
    beta = rng.uniform(0.0, 1.0, size=T)
    S0 = 0.1 * rng.standard_normal((dk, dv))
    dO, dST = rng.standard_normal((T, dv)), rng.standard_normal((dk, dv))
    ref = O.gdn_bwd(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                    beta[None, :, None], None, None, S0[None, None], dO[None, :, None],
                    dST[None, None], scale=1.0, l2norm=False, gates_given=True)
    dq, dk_, dv_, dg, dbeta, dS0 = chunk_gdn_bwd(q, k, v, g, beta, S0, dO, dST, C)
    for got, want in ((dq, ref["dq"][0, :, 0]), (dk_, ref["dk"][0, :, 0]),
                      (dv_, ref["dv"][0, :, 0]), (dg, ref["da"][0, :, 0]),
                      (dbeta, ref["db"][0, :, 0]), (dS0, ref["dh0"][0, 0])):
        np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("T", [1, 30, 64, 100])
@pytest.mark.parametrize("C", [16, 64])
def test_chunk_gdn2_backward_equals_token_backward(T, C):
    """The channel-decay chunkwise backward against the oracle's token-by-token
    Gated DeltaNet-2 backward (pinned by finite differences)."""
    dk, dv = 16, 8
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    q /= np.linalg.norm(q, axis=1, keepdims=True) * 4.0
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    g = -rng.uniform(0.0, 1.0, size=(T, dk))
    b = rng.uniform(0.0, 1.0, size=(T, dk))
    w = rng.uniform(0.0, 1.0, size=(T, dv))
    S0 = 0.1 * rng.standard_normal((dk, dv))
    dO, dST = rng.standard_normal((T, dv)), rng.standard_normal((dk, dv))
    ref = O.gdn2_bwd(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
                     b[None, :, None], w[None, :, None], None, None, S0[None, None],
                     dO[None, :, None], dST[None, None], scale=1.0, l2norm=False,
                     gates_given=True)
    got = chunk_gdn2_bwd(q, k, v, g, b, w, S0, dO, dST, C)
    for x, name in zip(got, ("dq", "dk", "dv", "da", "db", "dw")):
        np.testing.assert_allclose(x, ref[name][0, :, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(got[6], ref["dh0"][0, 0], rtol=1e-9, atol=1e-10)
