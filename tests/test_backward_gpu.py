"""Backward pass through the C ABI (kda_backward / gdn_backward) against the
fp64 oracle's reverse-mode derivative, element by element.

The kernel computes in fp32 on exactly the values the oracle is given (bf16
inputs widen exactly), and writes fp32 gradients, so the bound is set by fp32
rounding, not by bf16 outputs: per (sequence, head) slice,
max|x - ref| / max|ref| <= 1e-3 for every gradient.  The recurrence is
contractive (|alpha| <= 1, ||I - beta k k^T|| <= 1 for unit k), so the rounding
of each step is not amplified along the sequence; a step sums 128-256 terms of
size O(1) (relative error ~ 1e-6 each), and the sequences here run to 4096
steps: 1e-3 leaves two orders of magnitude, and a wrong term moves the error
to O(1).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin
from parity_util import slice_rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_69_b200 import build
    build.build()
    import oracle
    oracle.build()


def kda():
    from gated_delta_rule_69_b200 import kda as k
    return k


def f64(t):
    return None if t is None else t.detach().cpu().double().numpy()


def case(T, H, dk, dv, dtype="bf16", seed=0, lengths=None, init_std=0.02, scalar_gate=False,
         dfs_scale=1.0):
    w = kin.Workload("bwd", "prefill", H=H, d_k=dk, d_v=dv, dtype=dtype, seed=seed, T=T,
                     init_std=init_std)
    inp = kin.generate(w, device=DEV, lengths=lengths)
    if scalar_gate:
        inp["log_alpha"] = inp["log_alpha"][..., 0].contiguous()
    ct = kin.cotangents(w, inp["lengths"], device=DEV)
    inp["d_o"] = ct["d_o"]
    inp["d_final_state"] = None if dfs_scale == 0 else ct["d_final_state"] * dfs_scale
    return inp


def run_gpu(inp, scalar_gate=False, workspace=None):
    fn = kda().gdn_backward if scalar_gate else kda().kda_backward
    out = fn(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["d_o"],
             init_state=inp["init_state"], d_final_state=inp["d_final_state"],
             cu_seqlens=inp["cu_seqlens"], workspace=workspace)
    torch.cuda.synchronize()
    return [f64(x) for x in out]


def run_oracle(inp, scalar_gate=False, heads=None):
    import oracle
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    H = inp["q"].shape[1]
    hs = list(range(H)) if heads is None else list(heads)
    sel = lambda t: None if t is None else f64(t)[:, hs] if t.dim() >= 2 else f64(t)
    st = lambda t: None if t is None else f64(t)[:, hs]
    fn = oracle.gdn_backward if scalar_gate else oracle.kda_backward
    ref = fn(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["log_alpha"]),
             sel(inp["beta"]), sel(inp["d_o"]), init_state=st(inp["init_state"]),
             d_final_state=st(inp["d_final_state"]), cu_seqlens=cu)
    return ref, cu, hs


NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_init_state")


def check(gpu, ref, cu, hs):
    """Worst per-(sequence, head) error of each gradient; gpu outputs are
    restricted to the heads ``hs`` the oracle ran."""
    errs = {}
    n = len(cu) - 1
    for name, x, r in zip(NAMES, gpu, ref):
        x = x[:, hs]
        if name == "d_init_state":
            sl = [(i, j) for i in range(n) for j in range(len(hs))]
        else:
            sl = [(slice(int(cu[i]), int(cu[i + 1])), j) for i in range(n)
                  for j in range(len(hs)) if cu[i + 1] > cu[i]]
        errs[name] = slice_rel_err(x, r, sl)
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, f"gradient errors above {TOL}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (64, 96), (32, 128)])
def test_backward_fp32_shapes(dk, dv):
    """fp32 inputs, two ragged sequences crossing the 64-step blocks."""
    inp = case(0, 2, dk, dv, dtype="fp32", seed=3, lengths=[70, 131])
    ref, cu, hs = run_oracle(inp)
    check(run_gpu(inp), ref, cu, hs)


@pytest.mark.parametrize("lengths", [[300], [1, 64, 65, 0, 190, 128]])
def test_backward_bf16_varlen(lengths):
    """bf16 inputs, d = 128; single tokens, exact blocks, an empty sequence."""
    inp = case(0, 3, 128, 128, seed=4, lengths=lengths, dfs_scale=50.0)
    ref, cu, hs = run_oracle(inp)
    check(run_gpu(inp), ref, cu, hs)


def test_backward_no_initial_state_no_final_gradient():
    inp = case(0, 2, 128, 128, seed=5, lengths=[100, 29], init_std=0.0, dfs_scale=0.0)
    assert inp["init_state"] is None and inp["d_final_state"] is None
    ref, cu, hs = run_oracle(inp)
    check(run_gpu(inp), ref, cu, hs)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_gdn_backward(dtype):
    inp = case(0, 2, 128, 128, dtype=dtype, seed=6, lengths=[77, 140], scalar_gate=True,
               dfs_scale=50.0)
    ref, cu, hs = run_oracle(inp, scalar_gate=True)
    check(run_gpu(inp, scalar_gate=True), ref, cu, hs)


def test_backward_full_size_sampled_heads():
    """The bench workload (T = 4096, H = 16, d = 128, bf16) in the launch the
    bench times; the oracle runs two of the heads."""
    w = kin.WORKLOADS["prefill_T4096_H16_d128"]
    inp = kin.generate(w, device=DEV)
    ct = kin.cotangents(w, inp["lengths"], device=DEV)
    inp.update(d_o=ct["d_o"], d_final_state=ct["d_final_state"])
    gpu = run_gpu(inp)
    ref, cu, hs = run_oracle(inp, heads=[0, 11])
    check(gpu, ref, cu, hs)


def test_backward_repeatable_within_tolerance_and_workspace_reuse():
    """Two calls on one workspace agree (fp32 atomics may reorder the last bits)."""
    inp = case(0, 2, 128, 128, seed=7, lengths=[200, 60])
    n = inp["cu_seqlens"].numel() - 1
    ws = torch.empty(kda().kda_backward_workspace_size(n, 260, 2, 128, 128), dtype=torch.uint8,
                     device=DEV)
    a = run_gpu(inp, workspace=ws)
    b = run_gpu(inp, workspace=ws)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-5, atol=1e-6)


def test_backward_bad_cu_seqlens_sets_error_word():
    """A decreasing cu_seqlens entry: the affected sequence is skipped (every
    access stays inside [0, T)) and the workspace error word is set."""
    inp = case(0, 1, 32, 32, dtype="fp32", seed=8, lengths=[100, 28])
    inp["cu_seqlens"] = torch.tensor([0, 100, 50, 128], dtype=torch.int32, device=DEV)
    inp["init_state"] = None
    inp["d_final_state"] = None
    ws = torch.empty(kda().kda_backward_workspace_size(3, 128, 1, 32, 32), dtype=torch.uint8,
                     device=DEV)
    kda().kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["d_o"],
                       cu_seqlens=inp["cu_seqlens"], workspace=ws)
    assert kda().kda_check_workspace_error(ws) == kda().KDA_ERR_INVALID_ARG
