"""kda_backward_chunked (bf16, d = 128, chunk boundary states from the chunk
records) against the fp64 oracle's derivative, at the bf16 tolerance: the
boundary states carry the records' bf16 rounding, as the prefill's own states
do (per (sequence, head) slice, max|x - ref| / max|ref| <= 2e-2).  The
chunk-local gradients run on the tensor cores except for chunks that decay
past e^-80 on some channel, which the token-by-token kernel takes; one case
mixes both within a sequence and a head."""
import numpy as np
import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin
from test_backward_gpu import NAMES, f64, run_oracle
from parity_util import slice_rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 2e-2


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


def case(lengths, H, seed, init_std=0.02, dfs_scale=50.0):
    w = kin.Workload("bwdc", "prefill", H=H, d_k=128, d_v=128, dtype="bf16", seed=seed, T=0,
                     init_std=init_std)
    inp = kin.generate(w, device=DEV, lengths=lengths)
    ct = kin.cotangents(w, inp["lengths"], device=DEV)
    inp["d_o"] = ct["d_o"]
    inp["d_final_state"] = None if dfs_scale == 0 else ct["d_final_state"] * dfs_scale
    return inp


def run(inp):
    out = kda().kda_backward_chunked(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                     inp["d_o"], init_state=inp["init_state"],
                                     d_final_state=inp["d_final_state"],
                                     cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    return [f64(x) for x in out]


def errors(gpu, ref, cu, hs):
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
    return errs


@pytest.mark.parametrize("lengths", [[300], [1, 64, 65, 0, 190, 128]])
def test_backward_chunked_varlen(lengths):
    inp = case(lengths, 3, seed=4)
    ref, cu, hs = run_oracle(inp)
    errs = errors(run(inp), ref, cu, hs)
    assert all(e <= TOL for e in errs.values()), errs


def test_backward_chunked_no_state():
    inp = case([100, 29], 2, seed=5, init_std=0.0, dfs_scale=0.0)
    ref, cu, hs = run_oracle(inp)
    errs = errors(run(inp), ref, cu, hs)
    assert all(e <= TOL for e in errs.values()), errs


def test_backward_chunked_full_size_sampled_heads():
    w = kin.WORKLOADS["prefill_T4096_H16_d128"]
    inp = kin.generate(w, device=DEV)
    ct = kin.cotangents(w, inp["lengths"], device=DEV)
    inp.update(d_o=ct["d_o"], d_final_state=ct["d_final_state"])
    gpu = run(inp)
    ref, cu, hs = run_oracle(inp, heads=[0, 11])
    errs = errors(gpu, ref, cu, hs)
    assert all(e <= TOL for e in errs.values()), errs


def test_backward_chunked_slow_chunks_take_the_step_kernel():
    """Chunks whose decay passes e^-80 on one channel (over the chunk: the
    prefill's secondary form; within a 16-token block: the pairwise form) sit
    between ordinary chunks of the same sequence and head; their gradients
    come from the token-by-token kernel, the others' from the tensor cores."""
    inp = case([300, 140], 2, seed=6)
    g = inp["log_alpha"].float()
    g[64:128, 0, 5] = -2.0     # -128 over the chunk, -32 per 16-token block
    g[128:192, 1, 9] = -6.0    # -96 within a 16-token block
    g[300 + 64:300 + 128, 0, 17] = -1.5
    inp["log_alpha"] = g.to(inp["log_alpha"].dtype)
    ref, cu, hs = run_oracle(inp)
    errs = errors(run(inp), ref, cu, hs)
    assert all(e <= TOL for e in errs.values()), errs


@pytest.mark.parametrize("lengths", [[300], [1, 64, 65, 0, 190, 128]])
def test_gdn_backward_chunked(lengths):
    """The Gated DeltaNet gate (one log_alpha per token and head) through the
    same chunked path, against the oracle's gdn derivative; dlog_alpha is the
    channel sum of the per-channel one."""
    inp = case(lengths, 3, seed=8)
    inp["log_alpha"] = inp["log_alpha"][..., 0].contiguous()
    ref, cu, hs = run_oracle(inp, scalar_gate=True)
    out = kda().gdn_backward_chunked(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                     inp["d_o"], init_state=inp["init_state"],
                                     d_final_state=inp["d_final_state"], cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    errs = errors([f64(x) for x in out], ref, cu, hs)
    assert all(e <= TOL for e in errs.values()), errs


def test_gdn_backward_chunked_slow_chunks():
    """A scalar gate of -2 per token over one chunk of one head (-128 over the
    chunk) and of -6 within a 16-token block of another: those chunks take the
    step kernel, the rest the tensor cores."""
    inp = case([300, 140], 2, seed=9)
    g = inp["log_alpha"][..., 0].float().contiguous()
    g[64:128, 0] = -2.0
    g[128:192, 1] = -6.0
    inp["log_alpha"] = g.to(inp["q"].dtype)
    ref, cu, hs = run_oracle(inp, scalar_gate=True)
    out = kda().gdn_backward_chunked(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                     inp["d_o"], init_state=inp["init_state"],
                                     d_final_state=inp["d_final_state"], cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    errs = errors([f64(x) for x in out], ref, cu, hs)
    assert all(e <= TOL for e in errs.values()), errs
