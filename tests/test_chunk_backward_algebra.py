"""The chunk form of the backward pass, checked on the CPU against the fp64
oracle's token-by-token derivative.

The chunk algebra (news digest page on Kimi Linear, section "Algorithme
parallele par chunks"), per chunk of C tokens with entering state S:
    G = running sum of log_alpha, Ktil = K e^G, Qtil = Q e^G, Khat = K e^-G,
    Kbar = K e^{G_L - G}, A = strict_tril(diag(beta) Ktil Khat^T),
    T = (I + A)^-1, P = tril(Qtil Khat^T), W = T diag(beta) Ktil,
    U = T diag(beta) V - W S, O = Qtil S + P U,
    S_next = Diag(e^{G_L}) S + Kbar^T U.
Its reverse-mode derivative is written here chunk by chunk, in numpy (this
file's own code; the product has no such path yet).  What it fixes:
  * the reverse state chain is the transpose of the forward transition:
    dS = (Diag(e^{G_L}) + MP^T) dS_next + QP^T dO with MP = -Kbar^T W and
    QP = Qtil - P W, the forward's own chunk operands;
  * the chunk-local gradients (through the triangular inverse, both masks,
    the four gated operands and the running sum) equal the oracle's;
  * the staged form (a forward scan for each chunk's entering state, a
    reverse scan for dL/dS at each chunk's end, then each chunk's own
    token-by-token derivative) reproduces the whole sequence's gradients.
"""
import numpy as np
import pytest


def _case(rng, T, dk, dv):
    q = rng.normal(size=(T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.normal(size=(T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.normal(size=(T, dv))
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(T, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=T)))
    s0 = rng.normal(0.0, 0.5, size=(dk, dv))
    return q, k, v, g, beta, s0


def _chunk(q, k, v, g, beta, S):
    G = np.cumsum(g, axis=0)
    GL = G[-1]
    Kt, Qt, Kh, Kb = k * np.exp(G), q * np.exp(G), k * np.exp(-G), k * np.exp(GL - G)
    n = len(beta)
    A = np.tril(beta[:, None] * (Kt @ Kh.T), -1)
    Tm = np.linalg.inv(np.eye(n) + A)
    P = np.tril(Qt @ Kh.T)
    W = Tm @ (beta[:, None] * Kt)
    U = Tm @ (beta[:, None] * v) - W @ S
    O = Qt @ S + P @ U
    S_next = np.exp(GL)[:, None] * S + Kb.T @ U
    return dict(G=G, GL=GL, Kt=Kt, Qt=Qt, Kh=Kh, Kb=Kb, A=A, Tm=Tm, P=P, W=W, U=U, O=O,
                S_next=S_next)


def _chunk_backward(q, k, v, g, beta, S, c, dO, dS_next):
    """Gradients of one chunk given dL/dO and dL/dS_next; returns
    (dq, dk, dv, dg, dbeta, dS) and the reverse-chain operands."""
    b = beta
    Kt, Qt, Kh, Kb, Tm, P, W, U = (c[x] for x in ("Kt", "Qt", "Kh", "Kb", "Tm", "P", "W", "U"))
    G, GL = c["G"], c["GL"]
    # S_next = Diag(e^GL) S + Kbar^T U
    dS = np.exp(GL)[:, None] * dS_next
    dKb = U @ dS_next.T
    dU = Kb @ dS_next
    dEGL = np.sum(S * dS_next, axis=1)
    # O = Qtil S + P U
    dQt = dO @ S.T
    dS += Qt.T @ dO
    dP = np.tril(dO @ U.T)
    dU += P.T @ dO
    # U = T diag(beta) V - W S
    dW = -dU @ S.T
    dS += -W.T @ dU
    dbV = Tm.T @ dU
    dv = b[:, None] * dbV
    db = np.sum(v * dbV, axis=1)
    dT = dU @ (b[:, None] * v).T
    # W = T diag(beta) Ktil
    dbKt = Tm.T @ dW
    dKt = b[:, None] * dbKt
    db += np.sum(Kt * dbKt, axis=1)
    dT += dW @ (b[:, None] * Kt).T
    # T = (I + A)^-1, A = strict_tril(diag(beta) Ktil Khat^T)
    dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
    db += np.sum(dA * (Kt @ Kh.T), axis=1)
    dKt += (b[:, None] * dA) @ Kh
    dKh = (b[:, None] * dA).T @ Kt
    # P = tril(Qtil Khat^T)
    dQt += dP @ Kh
    dKh += dP.T @ Qt
    # gated operands and the running sum
    dk = dKt * np.exp(G) + dKh * np.exp(-G) + dKb * np.exp(GL - G)
    dq = dQt * np.exp(G)
    dG = dKt * Kt + dQt * Qt - dKh * Kh - dKb * Kb
    dGL = np.sum(dKb * Kb, axis=0) + np.exp(GL) * dEGL
    dg = np.cumsum(dG[::-1], axis=0)[::-1] + dGL[None, :]
    return dq, dk, dv, dg, db, dS


@pytest.mark.parametrize("C", [16, 64])
def test_chunk_backward_matches_oracle(oracle_mod, C):
    rng = np.random.default_rng(21)
    T, dk, dv = 150, 8, 6
    q, k, v, g, beta, s0 = _case(rng, T, dk, dv)
    d_o = rng.normal(size=(T, dv))
    d_sT = rng.normal(size=(dk, dv))
    # forward, keeping each chunk's entering state
    bounds = [(t0, min(t0 + C, T)) for t0 in range(0, T, C)]
    S, states, O = s0.copy(), [], np.zeros((T, dv))
    for t0, t1 in bounds:
        states.append(S.copy())
        c = _chunk(q[t0:t1], k[t0:t1], v[t0:t1], g[t0:t1], beta[t0:t1], S)
        O[t0:t1] = c["O"]
        S = c["S_next"]
    o_ref, s_ref = oracle_mod.kda_recurrence(q[:, None], k[:, None], v[:, None], g[:, None],
                                             beta[:, None], init_state=s0[None, None])
    np.testing.assert_allclose(O, o_ref[:, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(S, s_ref[0, 0], rtol=1e-9, atol=1e-11)
    # backward, chunk by chunk from the end
    grads = [np.zeros_like(x) for x in (q, k, v, g, beta)]
    dS = d_sT.copy()
    for (t0, t1), S_in in zip(reversed(bounds), reversed(states)):
        sl = slice(t0, t1)
        c = _chunk(q[sl], k[sl], v[sl], g[sl], beta[sl], S_in)
        *gc, dS_in = _chunk_backward(q[sl], k[sl], v[sl], g[sl], beta[sl], S_in, c, d_o[sl], dS)
        for acc, x in zip(grads, gc):
            acc[sl] = x
        # the reverse chain is the transpose of the forward transition
        MP = -c["Kb"].T @ c["W"]
        QP = c["Qt"] - c["P"] @ c["W"]
        chain = np.exp(c["GL"])[:, None] * dS + MP.T @ dS + QP.T @ d_o[sl]
        np.testing.assert_allclose(dS_in, chain, rtol=1e-10, atol=1e-12)
        dS = dS_in
    ref = oracle_mod.kda_backward(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                                  d_o[:, None], init_state=s0[None, None],
                                  d_final_state=d_sT[None, None])
    for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta"), grads, ref[:5]):
        np.testing.assert_allclose(x, r[:, 0], rtol=1e-8, atol=1e-10, err_msg=name)
    np.testing.assert_allclose(dS, ref[5][0, 0], rtol=1e-8, atol=1e-10)


def test_staged_backward_reproduces_the_oracle(oracle_mod):
    """The staged form: the forward scan over the chunk operands gives each
    chunk's entering state, the reverse scan dL/dS at each chunk's end; the
    token-by-token derivative of each chunk alone, from those two, then equals
    the whole sequence's (the oracle's backward run per chunk as a sequence of
    its own with init_state = S_in and d_final_state = dS_next)."""
    rng = np.random.default_rng(23)
    T, dk, dv, C = 200, 8, 6, 64
    q, k, v, g, beta, s0 = _case(rng, T, dk, dv)
    d_o = rng.normal(size=(T, dv))
    d_sT = rng.normal(size=(dk, dv))
    bounds = [(t0, min(t0 + C, T)) for t0 in range(0, T, C)]
    ops, S_in = [], []
    S = s0.copy()
    for t0, t1 in bounds:   # forward scan: S <- Diag(e^GL) S + MP S + YT V
        c = _chunk(q[t0:t1], k[t0:t1], v[t0:t1], g[t0:t1], beta[t0:t1], S)
        Tb = c["Tm"] * beta[t0:t1][None, :]
        MP, YT = -c["Kb"].T @ c["W"], c["Kb"].T @ Tb
        QP = c["Qt"] - c["P"] @ c["W"]
        ops.append((np.exp(c["GL"]), MP, YT, QP))
        S_in.append(S.copy())
        S = ops[-1][0][:, None] * S + MP @ S + YT @ v[t0:t1]
    dS_next = [None] * len(bounds)
    dS = d_sT.copy()
    for i in reversed(range(len(bounds))):   # reverse scan
        t0, t1 = bounds[i]
        egl, MP, _, QP = ops[i]
        dS_next[i] = dS.copy()
        dS = egl[:, None] * dS + MP.T @ dS + QP.T @ d_o[t0:t1]
    ref = oracle_mod.kda_backward(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                                  d_o[:, None], init_state=s0[None, None],
                                  d_final_state=d_sT[None, None])
    for i, (t0, t1) in enumerate(bounds):
        sl = slice(t0, t1)
        part = oracle_mod.kda_backward(q[sl, None], k[sl, None], v[sl, None], g[sl, None],
                                       beta[sl, None], d_o[sl, None],
                                       init_state=S_in[i][None, None],
                                       d_final_state=dS_next[i][None, None])
        for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta"), part[:5], ref[:5]):
            np.testing.assert_allclose(x, r[sl], rtol=1e-8, atol=1e-10, err_msg=f"{name} chunk {i}")
        if i == 0:
            np.testing.assert_allclose(part[5], ref[5], rtol=1e-8, atol=1e-10)
    np.testing.assert_allclose(dS, ref[5][0, 0], rtol=1e-8, atol=1e-10)
