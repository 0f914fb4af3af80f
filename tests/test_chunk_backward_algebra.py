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
file's own code, independent of the library's).  What it fixes:
  * the reverse state chain is the transpose of the forward transition:
    dS = (Diag(e^{G_L}) + MP^T) dS_next + QP^T dO with MP = -Kbar^T W and
    QP = Qtil - P W, the forward's own chunk operands;
  * the chunk-local gradients (through the triangular inverse, both masks,
    the four gated operands and the running sum) equal the oracle's;
  * the staged form (a forward scan for each chunk's entering state, a
    reverse scan for dL/dS at each chunk's end, then each chunk's own
    token-by-token derivative) reproduces the whole sequence's gradients;
  * the product form of the chunk gradients (the sequence of matrix products
    the library's tensor-core chunk kernel forms) equals that derivative, and
    with every product operand rounded to bf16 stays within 1e-2 of it.
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


def _chunk_backward_products(q, k, v, g, beta, S, dO, dS_next, rnd):
    """The chunk gradients in the form the tensor-core kernel computes them
    (R = V - Ktil S, U = T_beta R, dU = Kbar dS_next + P^T dO, dR = T_beta^T dU,
    dT_beta = dU R^T, dA = -strict_tril(T^T (dT T^T)), then the stacked
    dQtil / dKtil, dKhat, dKbar), every product operand passed through ``rnd``
    (the identity, or bf16 rounding) and accumulated in fp64; the elementwise
    steps in fp64.  Returns dq, dk, dv, dg, dbeta."""
    G = np.cumsum(g, axis=0)
    GL = G[-1]
    Kt, Qt, Kh, Kb = k * np.exp(G), q * np.exp(G), k * np.exp(-G), k * np.exp(GL - G)
    n = len(beta)
    KK = rnd(Kt) @ rnd(Kh).T
    A = np.tril(beta[:, None] * KK, -1)
    Tm = np.linalg.inv(np.eye(n) + A)
    P = np.tril(rnd(Qt) @ rnd(Kh).T)
    Tb = Tm * beta[None, :]
    R = v - rnd(Kt) @ rnd(S)
    U = rnd(Tb) @ rnd(R)
    dU = rnd(Kb) @ rnd(dS_next) + rnd(P).T @ rnd(dO)
    dR = rnd(Tb).T @ rnd(dU)
    dTb = rnd(dU) @ rnd(R).T
    dbeta = np.sum(dTb * Tm, axis=0)
    dT = dTb * beta[None, :]
    Z = rnd(dT) @ rnd(Tm).T
    dA = np.tril(-(rnd(Tm).T @ rnd(Z)), -1)
    dbeta = dbeta + np.sum(dA * KK, axis=1)
    BdA = beta[:, None] * dA
    dP = np.tril(rnd(dO) @ rnd(U).T)
    dQt = rnd(dO) @ rnd(S).T + rnd(dP) @ rnd(Kh)
    dKt = -(rnd(dR) @ rnd(S).T) + rnd(BdA) @ rnd(Kh)
    dKh = rnd(dP).T @ rnd(Qt) + rnd(BdA).T @ rnd(Kt)
    dKb = rnd(U) @ rnd(dS_next).T
    dq = dQt * np.exp(G)
    dk = dKt * np.exp(G) + dKh * np.exp(-G) + dKb * np.exp(GL - G)
    dG = dKt * Kt + dQt * Qt - dKh * Kh - dKb * Kb
    dGL = np.sum(dKb * Kb, axis=0) + np.exp(GL) * np.sum(S * dS_next, axis=1)
    dg = np.cumsum(dG[::-1], axis=0)[::-1] + dGL[None, :]
    return dq, dk, dR, dg, dbeta


def test_product_form_is_the_chunk_derivative():
    """The product form above equals the chunk derivative written out earlier
    in this file (fp64, no rounding)."""
    rng = np.random.default_rng(29)
    C, dk, dv = 64, 16, 12
    q, k, v, g, beta, s0 = _case(rng, C, dk, dv)
    dO = rng.normal(size=(C, dv))
    dSn = rng.normal(size=(dk, dv))
    c = _chunk(q, k, v, g, beta, s0)
    ref = _chunk_backward(q, k, v, g, beta, s0, c, dO, dSn)
    got = _chunk_backward_products(q, k, v, g, beta, s0, dO, dSn, lambda x: x)
    for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta"), got, ref[:5]):
        np.testing.assert_allclose(x, r, rtol=1e-9, atol=1e-11, err_msg=name)


def test_product_form_in_bf16_operands_stays_within_the_tolerance():
    """The numerics of the tensor-core chunk gradients: every product operand
    rounded to bf16 (fp32 accumulation is closer to fp64 than bf16 rounding is),
    on chunks of the bench's 4096-token workload (q, k unit rows, the gate and
    beta draws of the input recipe, upstream gradients N(0, 1)) with states
    of rms 0.3.  Per gradient, max |x - ref| / max |ref| stays below 1e-2 (it
    measures 2e-3 to 5e-3), under the 2e-2 the chunked backward is tested at."""
    import torch
    from gated_delta_rule_69_b200 import inputs as kin
    w = kin.WORKLOADS["prefill_T4096_H16_d128"]
    inp = kin.generate(w, device="cpu")
    ct = kin.cotangents(w, inp["lengths"], device="cpu")

    def bf16(x):
        return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()

    rng = np.random.default_rng(31)
    h = 3
    for t0 in (0, 640, 2048):
        sl = slice(t0, t0 + 64)
        f = lambda x: x[sl, h].double().numpy()
        args = (f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["log_alpha"]), f(inp["beta"]))
        S = rng.normal(0.0, 0.3, size=(128, 128))
        dSn = rng.normal(0.0, 0.3, size=(128, 128))
        dO = f(ct["d_o"])
        ref = _chunk_backward_products(*args, S, dO, dSn, lambda x: x)
        got = _chunk_backward_products(*args, S, dO, dSn, bf16)
        for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta"), got, ref):
            err = np.max(np.abs(x - r)) / np.max(np.abs(r))
            assert err < 1e-2, (t0, name, err)
