"""KDA oracle, Python side: builds and calls the fp64 C recurrence in
``kda_oracle.c``.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path and never imports the product package.

The recurrence (page "Kimi Linear" on docsaid.org, section "KDA : une
decroissance propre a chaque canal"; course page "Attention lineaire et
recurrence", section "Kimi Delta Attention = les trois remedes combines"):

    S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t

``gdn_recurrence`` is the Gated DeltaNet special case (one scalar gate per
token and head), written from its own update equation.  ``kda_backward`` and
``gdn_backward`` are the recurrence's reverse-mode derivative.

Inputs are float64 numpy arrays holding exactly the values the GPU sees (bf16
inputs are widened exactly).  Pins of this oracle (closed forms, exact
retrieval, explicit transition products, invariants) are in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE semantics: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-std=c11", _SRC, "-o", tmp, "-lm"],
            check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            lib.kda_oracle_recurrence.argtypes = [
                dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                dp, dp, ctypes.c_int]
            lib.kda_oracle_recurrence.restype = ctypes.c_int
            lib.gdn_oracle_recurrence.argtypes = lib.kda_oracle_recurrence.argtypes
            lib.gdn_oracle_recurrence.restype = ctypes.c_int
            lib.kda_oracle_max_threads.restype = ctypes.c_int
            lib.kda_oracle_backward.argtypes = [
                dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
            lib.kda_oracle_backward.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the oracle's OpenMP region uses by default."""
    return int(_load().kda_oracle_max_threads())


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def kda_recurrence(q, k, v, g, beta, init_state=None, cu_seqlens=None,
                   nthreads: int = 0):
    """Run the recurrence over packed sequences.

    q, k, g: [T, H, d_k]; v: [T, H, d_v]; beta: [T, H];
    init_state: [N, H, d_k, d_v] or None (zeros);
    cu_seqlens: [N+1] int offsets or None (one sequence of length T).
    Returns (o [T, H, d_v], final_state [N, H, d_k, d_v]) as float64.
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    if k.shape != (T, H, dk) or g.shape != (T, H, dk):
        raise ValueError("q, k, g must share shape [T, H, d_k]")
    if v.shape[:2] != (T, H) or beta.shape != (T, H):
        raise ValueError("v must be [T, H, d_v] and beta [T, H]")
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != T:
        raise ValueError("cu_seqlens must start at 0 and end at T")
    s0 = None if init_state is None else _f64(init_state)
    if s0 is not None and s0.shape != (n, H, dk, dv):
        raise ValueError("init_state must be [N, H, d_k, d_v]")
    o = np.zeros((T, H, dv), dtype=np.float64)
    fs = np.zeros((n, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        n, H, dk, dv, _ptr(o), _ptr(fs), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_recurrence failed with code {rc}")
    return o, fs


def gdn_recurrence(q, k, v, g, beta, init_state=None, cu_seqlens=None,
                   nthreads: int = 0):
    """Gated DeltaNet over packed sequences: as kda_recurrence with one gate
    value per (token, head), g [T, H] (the scalar-gate update, taken as
    printed: erase, then decay, then write)."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    if k.shape != (T, H, dk) or g.shape != (T, H):
        raise ValueError("q, k must share shape [T, H, d_k] and g be [T, H]")
    if v.shape[:2] != (T, H) or beta.shape != (T, H):
        raise ValueError("v must be [T, H, d_v] and beta [T, H]")
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != T:
        raise ValueError("cu_seqlens must start at 0 and end at T")
    s0 = None if init_state is None else _f64(init_state)
    if s0 is not None and s0.shape != (n, H, dk, dv):
        raise ValueError("init_state must be [N, H, d_k, d_v]")
    o = np.zeros((T, H, dv), dtype=np.float64)
    fs = np.zeros((n, H, dk, dv), dtype=np.float64)
    rc = _load().gdn_oracle_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        n, H, dk, dv, _ptr(o), _ptr(fs), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_recurrence failed with code {rc}")
    return o, fs


def gdn_decode_step(q, k, v, g, beta, state, nthreads: int = 0):
    """One Gated DeltaNet step for each of B sequences (g [B, H])."""
    B = np.asarray(q).shape[0]
    cu = np.arange(B + 1, dtype=np.int64)
    return gdn_recurrence(q, k, v, g, beta, init_state=state, cu_seqlens=cu,
                          nthreads=nthreads)


def kda_decode_step(q, k, v, g, beta, state, nthreads: int = 0):
    """One recurrence step for each of B independent sequences.

    q, k, g: [B, H, d_k]; v: [B, H, d_v]; beta: [B, H]; state [B, H, d_k, d_v].
    Returns (o [B, H, d_v], new_state).  A decode step is the recurrence on B
    sequences of length one each.
    """
    B = np.asarray(q).shape[0]
    cu = np.arange(B + 1, dtype=np.int64)
    return kda_recurrence(q, k, v, g, beta, init_state=state, cu_seqlens=cu,
                          nthreads=nthreads)


# ---- backward pass ------------------------------------------------------------
# The reverse-mode derivative of the recurrence, step by step (the chain rule
# written out in kda_oracle.c, kda_oracle_backward).

def kda_backward(q, k, v, g, beta, d_o, init_state=None, d_final_state=None,
                 cu_seqlens=None, nthreads: int = 0):
    """Gradients of a loss L through kda_recurrence.

    d_o = dL/do [T, H, d_v]; d_final_state = dL/dS_T [N, H, d_k, d_v] or None
    (zero).  Returns (dq, dk, dv, dg, dbeta, d_init_state) as float64 arrays in
    the inputs' shapes (d_init_state = dL/dS_0, [N, H, d_k, d_v]).
    """
    q, k, v, g, beta, d_o = (_f64(x) for x in (q, k, v, g, beta, d_o))
    T, H, dk = q.shape
    dv = v.shape[2]
    if k.shape != (T, H, dk) or g.shape != (T, H, dk):
        raise ValueError("q, k, g must share shape [T, H, d_k]")
    if v.shape[:2] != (T, H) or beta.shape != (T, H) or d_o.shape != v.shape:
        raise ValueError("v and d_o must be [T, H, d_v] and beta [T, H]")
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != T:
        raise ValueError("cu_seqlens must start at 0 and end at T")
    s0 = None if init_state is None else _f64(init_state)
    dsT = None if d_final_state is None else _f64(d_final_state)
    for x in (s0, dsT):
        if x is not None and x.shape != (n, H, dk, dv):
            raise ValueError("states must be [N, H, d_k, d_v]")
    dq = np.zeros((T, H, dk)); dkk = np.zeros((T, H, dk)); dg = np.zeros((T, H, dk))
    dvv = np.zeros((T, H, dv)); db = np.zeros((T, H)); ds0 = np.zeros((n, H, dk, dv))
    rc = _load().kda_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n, H, dk, dv,
        _ptr(d_o), _ptr(dsT), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(db),
        _ptr(ds0), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_backward failed with code {rc}")
    return dq, dkk, dvv, dg, db, ds0


def gdn_backward(q, k, v, g, beta, d_o, init_state=None, d_final_state=None,
                 cu_seqlens=None, nthreads: int = 0):
    """Gradients through gdn_recurrence (g [T, H]).  A scalar gate is the
    per-channel gate with every channel equal, so its derivative is the sum of
    the per-channel derivatives over the key channels (the chain rule for a
    broadcast); the rest is kda_backward."""
    g = _f64(g)
    dk_ = np.asarray(q).shape[2]
    dq, dkk, dvv, dg, db, ds0 = kda_backward(
        q, k, v, np.repeat(g[:, :, None], dk_, axis=2), beta, d_o, init_state=init_state,
        d_final_state=d_final_state, cu_seqlens=cu_seqlens, nthreads=nthreads)
    return dq, dkk, dvv, dg.sum(axis=2), db, ds0


# ---- the layer's prologue and epilogue around the recurrence ----------------
# (page "Kimi Linear" on docsaid.org, section "Les autres pieces": q and k
# L2-normalised, beta a sigmoid, the output RMS-normalised per head then gated
# by a sigmoid; course page "Attention lineaire et recurrence": Kimi Linear's
# decay -e^A Softplus(z).)  Elementwise, in fp64.

def l2_normalize(x, eps):
    """x / sqrt(sum over the last axis of x^2 + eps)."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def softplus(z):
    """log(1 + e^z), overflow-free: max(z, 0) + log1p(e^{-|z|})."""
    z = _f64(z)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def sigmoid(x):
    """1 / (1 + e^{-x}), as e^x / (1 + e^x) for x < 0 (no cancellation)."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def kimi_log_alpha(gate_z, A_log):
    """log alpha = -exp(A_log[h]) softplus(z); gate_z [T, H, d_k], A_log [H]."""
    return -np.exp(_f64(A_log))[None, :, None] * softplus(gate_z)


def rms_norm_gate(o, out_gate, norm_weight, eps):
    """o / sqrt(mean over d_v of o^2 + eps) * w * sigmoid(out_gate) per (token, head)."""
    o = _f64(o)
    y = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    if norm_weight is not None:
        y = y * _f64(norm_weight)
    if out_gate is not None:
        y = y * sigmoid(out_gate)
    return y


def kda_layer(q, k, v, gate_z, A_log, beta_logit, out_gate=None, norm_weight=None,
              qk_eps=1e-6, norm_eps=1e-6, init_state=None, cu_seqlens=None, nthreads: int = 0):
    """Prologue, the KDA recurrence, epilogue.  Returns (o, final_state)."""
    o, fs = kda_recurrence(l2_normalize(q, qk_eps), l2_normalize(k, qk_eps), v,
                           kimi_log_alpha(gate_z, A_log), sigmoid(beta_logit),
                           init_state=init_state, cu_seqlens=cu_seqlens, nthreads=nthreads)
    return rms_norm_gate(o, out_gate, norm_weight, norm_eps), fs
