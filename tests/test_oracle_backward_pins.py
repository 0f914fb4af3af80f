"""Pins of the oracle's backward pass (the reverse-mode derivative of the
recurrence) against facts that do not come from its own chain-rule code:
finite differences of the oracle's forward (itself pinned in
test_oracle_pins.py), torch autograd of the recurrence written as plain tensor
ops, and a closed form.  CPU only.

Plausible mistakes and the test that catches each:
  * a dropped term (dk through r, dS through the erase, the decay on dS)
    or a wrong sign                                  -> every-element differences
  * a wrong state used for a step (S_t for S_{t-1}), the block recompute
    off by one at the 64-token boundary               -> varlen directional
                                                        differences, autograd
  * gradients leaking across sequences                -> varlen directional
  * the scalar gate's derivative not summed over channels -> Gated DeltaNet
"""
import numpy as np
import pytest
import torch


def _case(rng, T, H, dk, dv, n):
    q = rng.normal(size=(T, H, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.normal(size=(T, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(T, H, dv))
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(T, H, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    s0 = rng.normal(0.0, 0.5, size=(n, H, dk, dv))
    return dict(q=q, k=k, v=v, g=g, beta=beta, s0=s0)


def _loss(oracle_mod, x, cu, w_o, w_s, gdn=False):
    f = oracle_mod.gdn_recurrence if gdn else oracle_mod.kda_recurrence
    o, fs = f(x["q"], x["k"], x["v"], x["g"], x["beta"], init_state=x["s0"], cu_seqlens=cu)
    return float(np.sum(o * w_o) + np.sum(fs * w_s))


def _grads(oracle_mod, x, cu, w_o, w_s, gdn=False):
    f = oracle_mod.gdn_backward if gdn else oracle_mod.kda_backward
    dq, dk, dv, dg, db, ds0 = f(x["q"], x["k"], x["v"], x["g"], x["beta"], w_o,
                                init_state=x["s0"], d_final_state=w_s, cu_seqlens=cu)
    return dict(q=dq, k=dk, v=dv, g=dg, beta=db, s0=ds0)


def test_backward_every_element_by_central_differences(oracle_mod):
    """Each gradient element against (L(x + e) - L(x - e)) / 2e, two sequences."""
    rng = np.random.default_rng(11)
    T, H, dk, dv = 5, 2, 3, 2
    cu = np.array([0, 2, 5])
    x = _case(rng, T, H, dk, dv, 2)
    w_o = rng.normal(size=(T, H, dv)); w_s = rng.normal(size=(2, H, dk, dv))
    grads = _grads(oracle_mod, x, cu, w_o, w_s)
    eps = 1e-6
    for name, arr in x.items():
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps; lp = _loss(oracle_mod, x, cu, w_o, w_s)
            arr[idx] = old - eps; lm = _loss(oracle_mod, x, cu, w_o, w_s)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grads[name], fd, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("gdn", [False, True])
def test_backward_directional_differences_varlen(oracle_mod, gdn):
    """<grad, D> against the directional difference for a random D per input,
    on two ragged sequences that cross the 64-step recompute boundary (the
    Gated DeltaNet case differentiates the scalar-gate forward, which is its own
    code)."""
    rng = np.random.default_rng(12 + gdn)
    T, H, dk, dv = 203, 2, 8, 5
    cu = np.array([0, 70, 203])
    x = _case(rng, T, H, dk, dv, 2)
    if gdn:
        x["g"] = x["g"][:, :, 0].copy()
    w_o = rng.normal(size=(T, H, dv)); w_s = rng.normal(size=(2, H, dk, dv))
    grads = _grads(oracle_mod, x, cu, w_o, w_s, gdn=gdn)
    eps = 1e-6
    for name in x:
        d = rng.normal(size=x[name].shape)
        base = x[name]
        x[name] = base + eps * d; lp = _loss(oracle_mod, x, cu, w_o, w_s, gdn)
        x[name] = base - eps * d; lm = _loss(oracle_mod, x, cu, w_o, w_s, gdn)
        x[name] = base
        fd = (lp - lm) / (2 * eps)
        an = float(np.sum(grads[name] * d))
        assert abs(an - fd) <= 1e-6 * max(1.0, abs(fd)), (name, an, fd)


def test_backward_matches_autograd(oracle_mod):
    """Against torch autograd (fp64, CPU) of the recurrence written as tensor
    ops: decay, erase with the decayed state, write, read-out."""
    rng = np.random.default_rng(13)
    T, H, dk, dv = 130, 1, 6, 4
    x = _case(rng, T, H, dk, dv, 1)
    w_o = rng.normal(size=(T, H, dv)); w_s = rng.normal(size=(1, H, dk, dv))
    grads = _grads(oracle_mod, x, None, w_o, w_s)
    tx = {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in x.items()}
    S = tx["s0"][0, 0]
    loss = torch.zeros((), dtype=torch.float64)
    for t in range(T):
        S = torch.exp(tx["g"][t, 0])[:, None] * S
        u = tx["beta"][t, 0] * (tx["v"][t, 0] - S.T @ tx["k"][t, 0])
        S = S + torch.outer(tx["k"][t, 0], u)
        loss = loss + (S.T @ tx["q"][t, 0] * torch.tensor(w_o[t, 0])).sum()
    loss = loss + (S * torch.tensor(w_s[0, 0])).sum()
    loss.backward()
    for name, t_ in tx.items():
        np.testing.assert_allclose(grads[name], t_.grad.numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=name)


def test_backward_closed_form_no_write_no_decay(oracle_mod):
    """alpha = 1, beta = 0: o_t = S_0^T q_t, so dq_t = S_0 do_t,
    dS_0 = dS_T + sum_t q_t do_t^T, and k, v get no gradient."""
    rng = np.random.default_rng(14)
    T, H, dk, dv = 70, 2, 5, 3
    x = _case(rng, T, H, dk, dv, 1)
    x["g"][:] = 0.0; x["beta"][:] = 0.0
    w_o = rng.normal(size=(T, H, dv)); w_s = rng.normal(size=(1, H, dk, dv))
    gr = _grads(oracle_mod, x, None, w_o, w_s)
    s0 = x["s0"][0]
    np.testing.assert_allclose(gr["q"], np.einsum("hcj,thj->thc", s0, w_o), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gr["s0"][0], w_s[0] + np.einsum("thc,thj->hcj", x["q"], w_o),
                               rtol=1e-12, atol=1e-12)
    assert np.all(gr["k"] == 0.0) and np.all(gr["v"] == 0.0)
