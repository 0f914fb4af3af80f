"""Shared helpers for the GPU-vs-oracle parity tests.

Error measure (elementwise relative error is ill-posed near zero): for each
(sequence, head) slice, err = max|x - ref| / max|ref|, and the test takes the
worst slice.  Tolerances: 2e-2 for bf16 I/O, 1e-4 for the fp32 test mode.
"""
import numpy as np
import torch

import oracle
from gated_delta_rule_69_b200.inputs import as_float64

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def slice_rel_err(x, ref, axis_slices):
    """Worst per-slice max-abs error over max-abs reference.  ``axis_slices``
    is a list of index tuples selecting the slices."""
    worst = 0.0
    for sl in axis_slices:
        r = ref[sl]
        scale = np.max(np.abs(r))
        d = np.max(np.abs(x[sl] - r)) if r.size else 0.0
        if scale == 0.0:
            e = d
        else:
            e = d / scale
        if not np.isfinite(e) or not np.all(np.isfinite(x[sl])):
            return float("inf")
        worst = max(worst, float(e))
    return worst


def o_err(o_gpu, o_ref, cu, H):
    """Worst (sequence, head) error of the outputs [T, H, d_v]."""
    sl = [(slice(int(cu[i]), int(cu[i + 1])), h) for i in range(len(cu) - 1)
          for h in range(H) if cu[i + 1] > cu[i]]
    return slice_rel_err(o_gpu, o_ref, sl)


def state_err(s_gpu, s_ref):
    n, H = s_ref.shape[:2]
    return slice_rel_err(s_gpu, s_ref, [(i, h) for i in range(n) for h in range(H)])


def run_oracle(inp, heads=None, seqs=None):
    """Oracle on the given inputs dict (see gated_delta_rule_69_b200.inputs),
    restricted to some heads and sequences.  Returns (o, final_state, cu)
    for the restricted problem: o [T_sel, H_sel, d_v], state [N_sel, H_sel, ...]."""
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    n = len(cu) - 1
    seqs = list(range(n)) if seqs is None else list(seqs)
    H = inp["q"].shape[1]
    heads = list(range(H)) if heads is None else list(heads)
    rows = np.concatenate([np.arange(cu[i], cu[i + 1]) for i in seqs]) if seqs else np.zeros(0, np.int64)
    lens = [int(cu[i + 1] - cu[i]) for i in seqs]
    sub_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    rows_t = torch.as_tensor(rows, device=inp["q"].device)
    hh = torch.as_tensor(heads, device=inp["q"].device)

    def pick(t):
        return as_float64(t.index_select(0, rows_t).index_select(1, hh))

    s0 = inp["init_state"]
    s0 = None if s0 is None else as_float64(
        s0.index_select(0, torch.as_tensor(seqs, device=s0.device)).index_select(1, hh))
    o, fs = oracle.kda_recurrence(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]),
                                  pick(inp["log_alpha"]), pick(inp["beta"]),
                                  init_state=s0, cu_seqlens=sub_cu)
    return o, fs, sub_cu, rows, heads


def to_device(inp, device="cuda"):
    out = {}
    for key, val in inp.items():
        out[key] = val.to(device) if isinstance(val, torch.Tensor) else val
    return out
