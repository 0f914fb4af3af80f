"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics,
not by the oracle itself.  CPU only.

Each test names the plausible oracle mistake it catches:
  * decay applied after the erase, or not at all        -> two-channel table,
    beta=0 closed form, gated whole-sequence solve
  * read-out with the pre-update state                  -> exact-write, DeltaNet solve
  * wrong sign of the correction / dropped beta         -> DeltaNet solve, explicit product
  * transposed state (S q instead of S^T q)             -> explicit product (d_k != d_v)
  * state not reset per sequence                        -> varlen split invariant
  * Gated DeltaNet: gate inside the erase, or missing    -> scalar-gate commutation,
    scalar beta=0 closed form, orthonormal overwrite
  * layer prologue / epilogue: a wrong axis, sign or
    constant in the norms, softplus or sigmoid           -> closed forms and invariants
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.linalg import solve_triangular

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _unit_rows(rng, shape):
    x = rng.normal(size=shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_case(rng, T, H, dk, dv, n_seqs=1):
    q = _unit_rows(rng, (T, H, dk))
    k = _unit_rows(rng, (T, H, dk))
    v = rng.normal(size=(T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(T, H, dk))))
    s0 = rng.normal(0.0, 0.5, size=(n_seqs, H, dk, dv))
    return q, k, v, g, beta, s0


# --- the pages' worked examples -------------------------------------------

def test_two_channel_decay_table(oracle_mod):
    """Page table: state (8, 6) -> (4, 3) under alpha=0.5 and (8, 0.6) under
    per-channel alpha=(1.0, 0.1); only Diag(alpha) S applies (beta = 0)."""
    fx = _load("two_channel_decay.json")
    s0 = np.array(fx["state_before"]).reshape(1, 1, 2, 1)
    for case in fx["cases"]:
        g = np.log(np.array(case["alpha"])).reshape(1, 1, 2)
        q = np.zeros((1, 1, 2)); k = np.array([[[0.6, 0.8]]])
        v = np.ones((1, 1, 1)); beta = np.zeros((1, 1))
        _, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
        np.testing.assert_allclose(fs.reshape(2), case["state_after"], rtol=1e-12)


def test_cumulative_decay_magnitude(oracle_mod):
    """Page example: alpha=0.5 over 64 tokens gives gamma ~ 5e-20, 1/gamma ~ 2e19.
    The oracle's state under pure decay is gamma * S0 and stays finite."""
    fx = _load("cumulative_decay.json")
    T = fx["tokens"]
    g = np.full((T, 1, 1), math.log(fx["alpha"]))
    s0 = np.ones((1, 1, 1, 1))
    z = np.zeros((T, 1, 1))
    _, fs = oracle_mod.kda_recurrence(z, z, z, g, np.zeros((T, 1)), init_state=s0)
    gamma = fs.item()
    # the page prints one significant digit
    assert float(f"{gamma:.0e}") == fx["gamma_approx"]
    assert float(f"{1.0 / gamma:.0e}") == fx["inverse_approx"]
    assert gamma == 0.5 ** 64


def test_bounded_gate_arithmetic():
    """Page remark: g >= -5 gives factors >= exp(-5) ~ 6.7e-3 and a 16-token
    tile log-decay in (-80, 0).  Fixes the stress-case bound used by tests."""
    fx = _load("bounded_gate.json")
    assert math.isclose(math.exp(fx["g_min"]), fx["min_factor_approx"], rel_tol=fx["rel_tol"])
    assert fx["g_min"] * fx["tile_tokens"] == fx["tile_logdecay_lower"]


def test_state_size_accounting():
    """Page code block output: 128x128 = 16384 values per head; 20 x 32 heads
    hold 10,485,760 values = 20 MiB in bf16."""
    fx = _load("state_size.json")
    assert fx["d_k"] * fx["d_v"] == fx["values_per_head"]
    total = fx["layers"] * fx["heads"] * fx["values_per_head"]
    assert total == fx["total_values"]
    assert total * 2 / 2 ** 20 == fx["bf16_mib"]


# --- closed forms -----------------------------------------------------------

def test_alpha1_beta0_constant_state(oracle_mod):
    """alpha=1, beta=0: S stays S0, so o_t = S0^T q_t."""
    rng = np.random.default_rng(1)
    T, H, dk, dv = 9, 2, 5, 3
    q, k, v, _, _, s0 = _rand_case(rng, T, H, dk, dv)
    g = np.zeros((T, H, dk)); beta = np.zeros((T, H))
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
    np.testing.assert_allclose(fs, s0, rtol=0, atol=0)
    np.testing.assert_allclose(o, np.einsum("hcj,thc->thj", s0[0], q), rtol=1e-13, atol=1e-14)


def test_beta0_pure_per_channel_decay(oracle_mod):
    """beta=0: S_t = Diag(exp(G_t)) S0 with G_t the running sum of g, so
    o_t = (exp(G_t) * S0)^T q_t."""
    rng = np.random.default_rng(2)
    T, H, dk, dv = 11, 2, 6, 4
    q, k, v, g, _, s0 = _rand_case(rng, T, H, dk, dv)
    beta = np.zeros((T, H))
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
    G = np.cumsum(g, axis=0)
    ref_o = np.einsum("thc,hcj,thc->thj", np.exp(G), s0[0], q)
    np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(fs[0], np.exp(G[-1])[:, :, None] * s0[0], rtol=1e-12)


def test_orthonormal_keys_exact_retrieval(oracle_mod):
    """alpha=1, beta=1, S0=0, orthonormal keys, T <= d_k: after all writes,
    querying with k_j returns v_j exactly (the associative read S^T k)."""
    rng = np.random.default_rng(3)
    dk, dv, T = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.normal(size=(dk, dk)))
    keys = Qm.T[:T]                      # orthonormal rows
    vals = rng.normal(size=(T, dv))
    # T write steps (beta=1), then T read steps (beta=0, q = k_j).
    k = np.concatenate([keys, np.zeros((T, dk))])[:, None, :]
    q = np.concatenate([np.zeros((T, dk)), keys])[:, None, :]
    v = np.concatenate([vals, np.zeros((T, dv))])[:, None, :]
    beta = np.concatenate([np.ones(T), np.zeros(T)])[:, None]
    g = np.zeros((2 * T, 1, dk))
    o, _ = oracle_mod.kda_recurrence(q, k, v, g, beta)
    np.testing.assert_allclose(o[T:, 0], vals, rtol=0, atol=1e-12)


def test_beta1_replaces_completely(oracle_mod):
    """beta_t=1 and |k_t|=1, any alpha and S0: S_t^T k_t = v_t, since
    k^T (I - k k^T) = 0; with q_t = k_t the output is v_t."""
    rng = np.random.default_rng(4)
    T, H, dk, dv = 13, 3, 7, 4
    _, k, v, g, _, s0 = _rand_case(rng, T, H, dk, dv)
    o, _ = oracle_mod.kda_recurrence(k, k, v, g, np.ones((T, H)), init_state=s0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


# --- explicit transition products (tiny inputs) ----------------------------

@pytest.mark.parametrize("seed,T,dk,dv", [(5, 12, 4, 3), (6, 7, 3, 5), (7, 10, 8, 8)])
def test_explicit_transition_product(oracle_mod, seed, T, dk, dv):
    """Dense M_t = (I - beta_t k_t k_t^T) Diag(alpha_t) and the unrolled sum
    S_t = M_t...M_1 S0 + sum_i M_t...M_{i+1} beta_i k_i v_i^T (course page,
    'Verification de comprehension': M_t acts on the incoming state)."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, s0 = _rand_case(rng, T, 1, dk, dv)
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
    M = [(np.eye(dk) - beta[t, 0] * np.outer(k[t, 0], k[t, 0])) @ np.diag(np.exp(g[t, 0]))
         for t in range(T)]
    for t in range(T):
        prod = np.eye(dk)
        for j in range(t, -1, -1):
            prod = prod @ M[j]
        S = prod @ s0[0, 0]
        for i in range(t + 1):
            tail = np.eye(dk)
            for j in range(t, i, -1):
                tail = tail @ M[j]
            S = S + tail @ (beta[i, 0] * np.outer(k[i, 0], v[i, 0]))
        np.testing.assert_allclose(o[t, 0], S.T @ q[t, 0], rtol=1e-11, atol=1e-12)
        if t == T - 1:
            np.testing.assert_allclose(fs[0, 0], S, rtol=1e-11, atol=1e-12)


# --- whole-sequence triangular solves ----------------------------------------

def test_deltanet_alpha1_triangular_solve(oracle_mod):
    """alpha=1 (plain DeltaNet): with u_t = beta_t (v_t - S_{t-1}^T k_t),
    (I + strict_tril(diag(beta) K K^T)) U = diag(beta)(V - K S0);
    S_T = S0 + K^T U and o_t = S0^T q_t + sum_{i<=t} (q_t.k_i) u_i."""
    rng = np.random.default_rng(8)
    T, dk, dv = 24, 6, 5
    q, k, v, _, beta, s0 = _rand_case(rng, T, 1, dk, dv)
    g = np.zeros((T, 1, dk))
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
    K, Q, V, b, S0 = k[:, 0], q[:, 0], v[:, 0], beta[:, 0], s0[0, 0]
    L = np.eye(T) + np.tril(b[:, None] * (K @ K.T), -1)
    U = solve_triangular(L, b[:, None] * (V - K @ S0), lower=True)
    np.testing.assert_allclose(fs[0, 0], S0 + K.T @ U, rtol=1e-11, atol=1e-12)
    ref_o = Q @ S0 + np.tril(Q @ K.T) @ U
    np.testing.assert_allclose(o[:, 0], ref_o, rtol=1e-11, atol=1e-12)


def test_gated_triangular_solve(oracle_mod):
    """General per-channel gate, whole sequence as one block, with G the running
    sum of g: u_t + sum_{i<t} beta_t (k_t e^{G_t-G_i}).k_i u_i
    = beta_t (v_t - S0^T (e^{G_t} k_t)); S_T = e^{G_T} S0 + sum_i e^{G_T-G_i} k_i u_i^T;
    o_t = S0^T (e^{G_t} q_t) + sum_{i<=t} (q_t e^{G_t-G_i}).k_i u_i."""
    rng = np.random.default_rng(9)
    T, dk, dv = 20, 7, 6
    q, k, v, g, beta, s0 = _rand_case(rng, T, 1, dk, dv)
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
    K, Q, V, b, S0 = k[:, 0], q[:, 0], v[:, 0], beta[:, 0], s0[0, 0]
    G = np.cumsum(g[:, 0], axis=0)
    decay = np.exp(G[:, None, :] - G[None, :, :])          # [t, i, c], used for i <= t
    KK = np.einsum("tc,tic,ic->ti", K, decay, K)
    QK = np.einsum("tc,tic,ic->ti", Q, decay, K)
    L = np.eye(T) + np.tril(b[:, None] * KK, -1)
    U = solve_triangular(L, b[:, None] * (V - (K * np.exp(G)) @ S0), lower=True)
    ref_s = np.exp(G[-1])[:, None] * S0 + (K * np.exp(G[-1] - G)).T @ U
    ref_o = (Q * np.exp(G)) @ S0 + np.tril(QK) @ U
    np.testing.assert_allclose(fs[0, 0], ref_s, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o[:, 0], ref_o, rtol=1e-11, atol=1e-12)


# --- invariants -----------------------------------------------------------------

def test_split_and_carry_state(oracle_mod):
    """Running [0, T) equals running [0, m) then [m, T) from the carried state."""
    rng = np.random.default_rng(10)
    T, H, dk, dv, m = 30, 2, 5, 4, 11
    q, k, v, g, beta, s0 = _rand_case(rng, T, H, dk, dv)
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
    o1, s1 = oracle_mod.kda_recurrence(q[:m], k[:m], v[:m], g[:m], beta[:m], init_state=s0)
    o2, s2 = oracle_mod.kda_recurrence(q[m:], k[m:], v[m:], g[m:], beta[m:], init_state=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s2, fs, rtol=1e-13, atol=1e-14)


def test_prefill_equals_repeated_decode(oracle_mod):
    rng = np.random.default_rng(11)
    T, H, dk, dv = 9, 3, 4, 6
    q, k, v, g, beta, s0 = _rand_case(rng, T, H, dk, dv)
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0)
    S = s0
    for t in range(T):
        ot, S = oracle_mod.kda_decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1],
                                           g[t:t + 1], beta[t:t + 1], S)
        np.testing.assert_allclose(ot[0], o[t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S, fs, rtol=1e-13, atol=1e-14)


def test_varlen_resets_state_per_sequence(oracle_mod):
    """Packed sequences with cu_seqlens equal separate runs, each from its own
    initial state."""
    rng = np.random.default_rng(12)
    lens = [5, 1, 8, 3]
    T, H, dk, dv = sum(lens), 2, 4, 3
    q, k, v, g, beta, s0 = _rand_case(rng, T, H, dk, dv, n_seqs=len(lens))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0, cu_seqlens=cu)
    for i in range(len(lens)):
        a, b = cu[i], cu[i + 1]
        oi, si = oracle_mod.kda_recurrence(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b],
                                           init_state=s0[i:i + 1])
        np.testing.assert_allclose(o[a:b], oi, rtol=0, atol=0)
        np.testing.assert_allclose(fs[i:i + 1], si, rtol=0, atol=0)


def test_state_norm_bound(oracle_mod):
    """|k|=1, beta in [0,1], alpha in (0,1]: the transition has spectral norm
    <= 1, so |S_t|_F <= |S_{t-1}|_F + beta_t |v_t| at every step."""
    rng = np.random.default_rng(13)
    T, dk, dv = 40, 6, 5
    q, k, v, g, beta, s0 = _rand_case(rng, T, 1, dk, dv)
    S = s0
    for t in range(T):
        _, S_new = oracle_mod.kda_decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1],
                                              g[t:t + 1], beta[t:t + 1], S)
        assert np.linalg.norm(S_new) <= np.linalg.norm(S) + beta[t, 0] * np.linalg.norm(v[t, 0]) + 1e-12
        S = S_new


def test_empty_sequence_keeps_initial_state(oracle_mod):
    """A zero-length sequence in a packed batch passes its initial state through."""
    rng = np.random.default_rng(14)
    lens = [3, 0, 2]
    T, H, dk, dv = 5, 1, 3, 2
    q, k, v, g, beta, s0 = _rand_case(rng, T, H, dk, dv, n_seqs=3)
    cu = np.concatenate([[0], np.cumsum(lens)])
    _, fs = oracle_mod.kda_recurrence(q, k, v, g, beta, init_state=s0, cu_seqlens=cu)
    np.testing.assert_array_equal(fs[1], s0[1])


# --- Gated DeltaNet (scalar gate) ----------------------------------------------

def test_gdn_equals_kda_with_repeated_gate(oracle_mod):
    """A scalar alpha commutes with (I - beta k k^T): the GDN update taken as
    printed (erase, then decay) equals the KDA update (decay, then erase) with
    the gate repeated over the channels.  The two oracle loops share no step
    order, so a misplaced or missing gate in either shows here."""
    rng = np.random.default_rng(41)
    T, H, dk, dv = 37, 2, 8, 5
    q, k, v, g3, beta, s0 = _rand_case(rng, T, H, dk, dv, n_seqs=2)
    g = g3[..., 0]
    cu = np.array([0, 15, T])
    o1, f1 = oracle_mod.gdn_recurrence(q, k, v, g, beta, s0, cu)
    o2, f2 = oracle_mod.kda_recurrence(q, k, v, np.repeat(g[..., None], dk, axis=-1), beta, s0, cu)
    assert np.abs(o1 - o2).max() < 1e-12 * max(1.0, np.abs(o2).max())
    assert np.abs(f1 - f2).max() < 1e-12 * max(1.0, np.abs(f2).max())


def test_gdn_beta0_scalar_decay(oracle_mod):
    """beta = 0: S_t = (prod_{s<=t} alpha_s) S_0 and o_t = S_t^T q_t."""
    rng = np.random.default_rng(42)
    T, H, dk, dv = 9, 1, 4, 3
    q, k, v, g3, beta, s0 = _rand_case(rng, T, H, dk, dv)
    g = g3[..., 0]
    o, fs = oracle_mod.gdn_recurrence(q, k, v, g, np.zeros_like(beta), s0)
    cum = np.exp(np.cumsum(g[:, 0]))
    for t in range(T):
        expect = cum[t] * (s0[0, 0].T @ q[t, 0])
        assert np.allclose(o[t, 0], expect, rtol=1e-13, atol=1e-13)
    assert np.allclose(fs[0, 0], cum[-1] * s0[0, 0], rtol=1e-13, atol=1e-13)


def test_gdn_orthonormal_overwrite(oracle_mod):
    """alpha = 1, beta = 1 and orthonormal keys: each write replaces the value
    stored under its key, so S_T = (I - sum e_i e_i^T) S_0 + sum e_i v_i^T and
    reading key e_i returns v_i."""
    rng = np.random.default_rng(43)
    dk, dv, m = 6, 4, 4
    basis, _ = np.linalg.qr(rng.normal(size=(dk, dk)))
    keys = basis[:, :m].T                      # m orthonormal rows
    T = m
    k = keys[:, None, :]
    q = keys[:, None, :]
    v = rng.normal(size=(T, 1, dv))
    s0 = rng.normal(size=(1, 1, dk, dv))
    o, fs = oracle_mod.gdn_recurrence(q, k, v, np.zeros((T, 1)), np.ones((T, 1)), s0)
    P = keys.T @ keys
    expect = (np.eye(dk) - P) @ s0[0, 0] + keys.T @ v[:, 0, :]
    assert np.allclose(fs[0, 0], expect, atol=1e-12)
    for t in range(T):
        assert np.allclose(o[t, 0], v[t, 0], atol=1e-12)


# --- the layer prologue and epilogue ---------------------------------------------

def test_l2_normalize_unit_rows(oracle_mod):
    rng = np.random.default_rng(51)
    x = rng.normal(size=(7, 3, 16)) * 5.0
    y = oracle_mod.l2_normalize(x, 0.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-14)
    # direction kept: y is x scaled by a positive number per row
    ratio = y / x
    assert np.allclose(ratio, ratio[..., :1], rtol=1e-12)
    assert np.all(ratio > 0)
    # a [3, 4] row has norm 5
    assert np.allclose(oracle_mod.l2_normalize(np.array([3.0, 4.0]), 0.0), [0.6, 0.8])


def test_kimi_gate_closed_forms(oracle_mod):
    """log alpha = -e^A softplus(z): z = 0, A = 0 gives -ln 2; A = ln 3 triples
    it; z -> +inf gives -e^A z; z -> -inf gives -e^A e^z."""
    z = np.array([0.0, 0.0, 40.0, -40.0]).reshape(4, 1, 1)
    A0 = np.zeros(1)
    g = oracle_mod.kimi_log_alpha(z, A0)[:, 0, 0]
    assert abs(g[0] + math.log(2.0)) < 1e-15
    assert abs(g[2] + 40.0) < 1e-12
    assert abs(g[3] + math.exp(-40.0)) < 1e-28
    g3 = oracle_mod.kimi_log_alpha(z, np.array([math.log(3.0)]))[:, 0, 0]
    assert abs(g3[0] + 3.0 * math.log(2.0)) < 1e-14
    assert np.all(oracle_mod.kimi_log_alpha(np.linspace(-5, 5, 11).reshape(11, 1, 1), A0) < 0)


def test_sigmoid_values(oracle_mod):
    assert oracle_mod.sigmoid(0.0) == 0.5
    assert abs(oracle_mod.sigmoid(math.log(3.0)) - 0.75) < 1e-15
    assert abs(oracle_mod.sigmoid(-40.0) - math.exp(-40.0)) < 1e-30


def test_rms_norm_gate(oracle_mod):
    rng = np.random.default_rng(52)
    o = rng.normal(size=(5, 2, 8)) * 3.0
    y = oracle_mod.rms_norm_gate(o, None, None, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-14)   # unit RMS per row
    w = rng.normal(size=8)
    yw = oracle_mod.rms_norm_gate(o, np.zeros((5, 2, 8)), w, 0.0)
    assert np.allclose(yw, 0.5 * y * w, atol=1e-14)                        # sigmoid(0) = 1/2
    # RMS of (1, 1, 1, 1) * 2 is 2: the row becomes (1, 1, 1, 1)
    assert np.allclose(oracle_mod.rms_norm_gate(np.full((1, 1, 4), 2.0), None, None, 0.0), 1.0)
