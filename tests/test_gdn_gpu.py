"""Gated DeltaNet (one scalar gate per token and head) through the C ABI:
gdn_prefill / gdn_decode_step against the fp64 oracle's own scalar-gate
recurrence, and bit for bit against kda_prefill / kda_decode_step fed the
same gate repeated over the key channels (the kernels spread the scalar gate
over the channels in shared memory, so both must round identically)."""
import numpy as np
import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin
from parity_util import TOL, o_err, state_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


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
    return t.detach().cpu().double().numpy()


def gdn_case(T, H, dk, dv, dtype="bf16", seed=0, lengths=None, init_std=0.02, gate=None):
    """The prefill input recipe, with the scalar gate taken from channel 0 of
    the per-channel draw (-softplus(N(-2, 1))) or set to a constant."""
    w = kin.Workload("gdn", "prefill", H=H, d_k=dk, d_v=dv, dtype=dtype, seed=seed, T=T,
                     init_std=init_std)
    inp = kin.generate(w, device=DEV, lengths=lengths)
    g = inp["log_alpha"][..., 0].contiguous()
    if gate is not None:
        g = torch.full_like(g, gate)
    inp["log_alpha"] = g
    return inp


def run_gdn(inp, workspace=None):
    q = inp["q"]
    T, H, _ = q.shape
    dv = inp["v"].shape[-1]
    o = torch.full((T, H, dv), float("nan"), dtype=q.dtype, device=DEV)
    n = inp["cu_seqlens"].numel() - 1
    o, fs = kda().gdn_prefill(q, inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"],
                              num_seqs=n, o=o, workspace=workspace)
    torch.cuda.synchronize()
    return o, fs


def oracle_gdn(inp):
    import oracle
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    s0 = None if inp["init_state"] is None else f64(inp["init_state"])
    o, fs = oracle.gdn_recurrence(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                  f64(inp["log_alpha"]), f64(inp["beta"]), s0, cu)
    return o, fs, cu


@pytest.mark.parametrize("lengths", [None, [1, 64, 130, 200, 63]])
def test_gdn_prefill_tensor_core(lengths):
    T = 300 if lengths is None else sum(lengths)
    inp = gdn_case(T, 3, 128, 128, seed=5, lengths=lengths)
    o, fs = run_gdn(inp)
    ref_o, ref_s, cu = oracle_gdn(inp)
    assert o_err(f64(o), ref_o, cu, 3) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]


@pytest.mark.parametrize("gate", [0.0, -1.5, -6.0, float("-inf")])
def test_gdn_prefill_gate_extremes(gate):
    """alpha = 1; a chunk decay of e^-96 (one reference per 16-token block);
    e^-96 within a block (pairwise path); alpha = 0."""
    inp = gdn_case(256, 2, 128, 128, seed=6, gate=gate)
    o, fs = run_gdn(inp)
    ref_o, ref_s, cu = oracle_gdn(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]


def test_gdn_prefill_single_kernel_path():
    inp = gdn_case(200, 2, 128, 128, seed=7, lengths=[77, 123])
    ws = torch.empty(kda().kda_prefill_workspace_size(2, 1, 1, 16, 16), dtype=torch.uint8, device=DEV)
    o, fs = run_gdn(inp, workspace=ws)
    ref_o, ref_s, cu = oracle_gdn(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (128, 128)])
def test_gdn_prefill_fp32(dk, dv):
    inp = gdn_case(100, 2, dk, dv, dtype="fp32", seed=dk + dv, lengths=[37, 63])
    o, fs = run_gdn(inp)
    ref_o, ref_s, cu = oracle_gdn(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["fp32"]
    assert state_err(f64(fs), ref_s) <= TOL["fp32"]


@pytest.mark.parametrize("small_ws", [False, True])
@pytest.mark.parametrize("gate", [None, -3.0])
def test_gdn_bitwise_equals_kda_with_repeated_gate(small_ws, gate):
    inp = gdn_case(190, 2, 128, 128, seed=8, lengths=[90, 100], gate=gate)
    ws = None
    if small_ws:
        ws = torch.empty(kda().kda_prefill_workspace_size(2, 1, 1, 16, 16), dtype=torch.uint8,
                         device=DEV)
    o1, f1 = run_gdn(inp, workspace=ws)
    g3 = inp["log_alpha"][..., None].expand(-1, -1, 128).contiguous()
    o2, f2 = kda().kda_prefill(inp["q"], inp["k"], inp["v"], g3, inp["beta"],
                               init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"],
                               num_seqs=2, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.equal(f1, f2)


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, "bf16"), (16, 32, "fp32")])
def test_gdn_decode_step(dk, dv, dtype):
    import oracle
    w = kin.Workload("dec", "decode", H=3, d_k=dk, d_v=dv, dtype=dtype, seed=9, batch=5,
                     init_std=0.02)
    inp = kin.generate(w, device=DEV)
    g = inp["log_alpha"][..., 0].contiguous()
    s0 = inp["init_state"].clone()
    o = torch.full((5, 3, dv), float("nan"), dtype=inp["q"].dtype, device=DEV)
    kda().gdn_decode_step(inp["q"], inp["k"], inp["v"], g, inp["beta"], inp["init_state"], o=o)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.gdn_decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(g),
                                          f64(inp["beta"]), f64(s0))
    assert o_err(f64(o), ref_o, np.arange(6), 3) <= TOL[dtype]
    assert state_err(f64(inp["init_state"]), ref_s) <= TOL[dtype]


def test_gdn_prefill_then_decode():
    """The state a GDN prefill hands over continues under gdn_decode_step as
    under the oracle's longer prefill."""
    import oracle
    T1, T2, H = 130, 4, 2
    inp = gdn_case(T1 + T2, H, 128, 128, seed=10)
    ref_o, ref_s, cu = oracle_gdn(inp)
    k = kda()
    o1, st = k.gdn_prefill(inp["q"][:T1], inp["k"][:T1], inp["v"][:T1], inp["log_alpha"][:T1],
                           inp["beta"][:T1], init_state=inp["init_state"])
    outs = [o1]
    for t in range(T1, T1 + T2):
        sl = slice(t, t + 1)
        outs.append(k.gdn_decode_step(inp["q"][sl], inp["k"][sl], inp["v"][sl],
                                      inp["log_alpha"][sl], inp["beta"][sl], st))
    torch.cuda.synchronize()
    o = torch.cat(outs)
    assert o_err(f64(o), ref_o, cu, H) <= TOL["bf16"]
    assert state_err(f64(st), ref_s) <= TOL["bf16"]
