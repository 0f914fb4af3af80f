"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Outputs are pre-filled with NaN so that any element a kernel fails to write
shows up as an infinite error."""
import numpy as np
import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin
from parity_util import TOL, o_err, run_oracle, state_err

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


def make(T, H, dk, dv, dtype="bf16", seed=0, lengths=None, init_std=0.0, device=DEV):
    w = kin.Workload("case", "prefill", H=H, d_k=dk, d_v=dv, dtype=dtype, seed=seed,
                     T=T, init_std=init_std)
    return kin.generate(w, device=device, lengths=lengths)


def gpu_prefill(inp, use_cu=True):
    q = inp["q"]
    T, H, _ = q.shape
    dv = inp["v"].shape[-1]
    o = torch.full((T, H, dv), float("nan"), dtype=q.dtype, device=q.device)
    cu = inp["cu_seqlens"] if use_cu else None
    n = inp["cu_seqlens"].numel() - 1
    o, fs = kda().kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              init_state=inp["init_state"], cu_seqlens=cu, num_seqs=n, o=o)
    torch.cuda.synchronize()
    return o, fs


def f64(t):
    return t.detach().cpu().double().numpy()


# --- decode ----------------------------------------------------------------------

def decode_inputs(B, H, dk, dv, dtype, seed):
    w = kin.Workload("dec", "decode", H=H, d_k=dk, d_v=dv, dtype=dtype, seed=seed,
                     batch=B, init_std=0.02)
    return kin.generate(w, device=DEV)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 16), (16, 128), (128, 128)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_decode_step_shapes(dk, dv, dtype):
    import oracle
    inp = decode_inputs(5, 3, dk, dv, dtype, seed=dk * 1000 + dv)
    s0 = inp["init_state"].clone()
    o = torch.full((5, 3, dv), float("nan"), dtype=inp["q"].dtype, device=DEV)
    kda().kda_decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          inp["init_state"], o=o)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.kda_decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                          f64(inp["log_alpha"]), f64(inp["beta"]), f64(s0))
    # a decode batch is B sequences of one token each
    cu = np.arange(6)
    assert o_err(f64(o), ref_o, cu, 3) <= TOL[dtype]
    assert state_err(f64(inp["init_state"]), ref_s) <= TOL[dtype]


def test_decode_full_size_chained():
    """Batch 256 x 32 heads x 128 x 128 (the decode workload), three chained
    steps, every output and state element against the oracle."""
    import oracle
    w = kin.WORKLOADS["decode_B256_H32_d128"]
    state = kin.generate(w, device=DEV)["init_state"]
    ref_s = f64(state)
    for step in range(3):
        inp = kin.generate(kin.Workload("dec", "decode", H=32, d_k=128, d_v=128, dtype="bf16",
                                        seed=w.seed + 10 + step, batch=256), device=DEV)
        o = torch.full((256, 32, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
        kda().kda_decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              state, o=o)
        torch.cuda.synchronize()
        ref_o, ref_s = oracle.kda_decode_step(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                                              f64(inp["log_alpha"]), f64(inp["beta"]), ref_s)
        assert o_err(f64(o), ref_o, np.arange(257), 32) <= TOL["bf16"]
        assert state_err(f64(state), ref_s) <= 1e-5   # fp32 state, fp32 arithmetic


def test_decode_empty_batch_is_noop():
    z = torch.zeros(0, 2, 16, device=DEV)
    o = kda().kda_decode_step(z, z, z, z, torch.zeros(0, 2, device=DEV),
                              torch.zeros(0, 2, 16, 16, device=DEV))
    assert o.shape == (0, 2, 16)


# --- prefill: fp32 test mode and ragged shapes -------------------------------------

def test_prefill_tiny_fp32_workload():
    """The tiny workload (T=64, H=1, d=16, fp32, zero state) at 1e-4."""
    inp = kin.generate(kin.WORKLOADS["tiny_T64_H1_d16_fp32"], device=DEV)
    o, fs = gpu_prefill(inp)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 1) <= TOL["fp32"]
    assert state_err(f64(fs), ref_s) <= TOL["fp32"]


@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 200])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (128, 128)])
def test_prefill_fp32_ragged(T, dk, dv):
    inp = make(T, 2, dk, dv, dtype="fp32", seed=T * 7 + dk, init_std=0.02)
    o, fs = gpu_prefill(inp)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["fp32"]
    assert state_err(f64(fs), ref_s) <= TOL["fp32"]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_prefill_varlen_with_empty_sequences(dtype):
    lens = [0, 1, 64, 65, 130, 0, 7, 200]
    inp = make(0, 3, 128, 128, dtype=dtype, seed=77, lengths=lens, init_std=0.02)
    o, fs = gpu_prefill(inp)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 3) <= TOL[dtype]
    assert state_err(f64(fs), ref_s) <= TOL[dtype]
    # zero-length sequences pass their initial state through unchanged
    assert torch.equal(fs[0], inp["init_state"][0]) and torch.equal(fs[5], inp["init_state"][5])


def test_prefill_equal_lengths_without_cu_seqlens():
    inp = make(0, 2, 64, 64, dtype="bf16", seed=5, lengths=[96, 96, 96], init_std=0.02)
    o, fs = gpu_prefill(inp, use_cu=False)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]


def test_prefill_state_aliasing_in_place():
    inp = make(300, 2, 128, 128, dtype="bf16", seed=9, init_std=0.02)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    st = inp["init_state"]
    o, fs = kda().kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                              init_state=st, cu_seqlens=inp["cu_seqlens"], final_state=st)
    torch.cuda.synchronize()
    assert fs.data_ptr() == st.data_ptr()
    assert state_err(f64(st), ref_s) <= TOL["bf16"]


def test_prefill_bad_cu_seqlens_reports_device_error():
    """A non-monotone cu_seqlens is caught by the kernel's own check: the call
    writes the error word and processes nothing for the bad sequences."""
    inp = make(0, 1, 16, 16, dtype="fp32", seed=3, lengths=[10, 10])
    bad = torch.tensor([0, 15, 10, 20], dtype=torch.int32, device=DEV)
    k = kda()
    ws = torch.empty(k.kda_prefill_workspace_size(3, 20, 1, 16, 16), dtype=torch.uint8, device=DEV)
    k.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                  cu_seqlens=bad, workspace=ws)
    assert k.kda_check_workspace_error(ws) == k.KDA_ERR_INVALID_ARG
    k.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                  cu_seqlens=inp["cu_seqlens"], workspace=ws)
    assert k.kda_check_workspace_error(ws) == k.KDA_OK


# --- prefill: numeric stress cases ---------------------------------------------------

def _stress(kind, T=256, H=2):
    inp = make(T, H, 128, 128, dtype="bf16", seed=11, init_std=0.02)
    g = inp["log_alpha"]
    if kind == "alpha_half":          # the page's example: gamma = 0.5^64 per chunk
        inp["log_alpha"] = torch.full_like(g, float(np.log(0.5)))
    elif kind == "gate_floor":        # bounded-gate floor g = -5 on every channel
        inp["log_alpha"] = torch.full_like(g, -5.0)
    elif kind == "alpha_one":
        inp["log_alpha"] = torch.zeros_like(g)
    elif kind == "alpha_zero":        # alpha = 0: the state is wiped every token
        inp["log_alpha"] = torch.full_like(g, float("-inf"))
    elif kind == "beta_zero":
        inp["beta"] = torch.zeros_like(inp["beta"])
    elif kind == "beta_one_qk":       # replace completely, read back with q = k
        inp["beta"] = torch.ones_like(inp["beta"])
        inp["q"] = inp["k"].clone()
    elif kind == "decay_near_limit":  # a chunk decays by e^-76.8: still the product form
        inp["log_alpha"] = torch.full_like(g, -1.2)
    elif kind == "decay_past_limit":  # e^-83.2 per chunk: one reference per 16-token block
        inp["log_alpha"] = torch.full_like(g, -1.3)
    elif kind == "decay_blocks":      # e^-48 per 16-token block, e^-192 per chunk
        inp["log_alpha"] = torch.full_like(g, -3.0)
    elif kind == "decay_past_block":  # e^-96 within a 16-token block: the pairwise path
        inp["log_alpha"] = torch.full_like(g, -6.0)
    elif kind == "decay_spikes":      # a -60 spike every 16 tokens on half the channels
        g2 = g.clone()
        g2[::16, :, 1::2] = -60.0
        inp["log_alpha"] = g2
    elif kind == "spikes_in_block":   # two -50 spikes in one block on a few channels
        g2 = g.clone()
        g2[3::64, :, :8] = -50.0
        g2[9::64, :, :8] = -50.0
        inp["log_alpha"] = g2
    elif kind == "mixed_extremes":    # half the channels keep, half forget fast
        g2 = g.clone()
        g2[..., ::2] = 0.0
        g2[..., 1::2] = -20.0
        inp["log_alpha"] = g2
    return inp


@pytest.mark.parametrize("kind", ["alpha_half", "gate_floor", "alpha_one", "alpha_zero",
                                  "beta_zero", "beta_one_qk", "mixed_extremes",
                                  "decay_near_limit", "decay_past_limit", "decay_blocks",
                                  "decay_past_block", "decay_spikes", "spikes_in_block"])
def test_prefill_stress(kind):
    inp = _stress(kind)
    o, fs = gpu_prefill(inp)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]
    if kind == "beta_one_qk":
        # o_t = v_t up to bf16 rounding of the inputs and output
        assert torch.allclose(o.float(), inp["v"].float(), atol=3e-2, rtol=2e-2)


# --- prefill then decode: the state hand-off -------------------------------------------

def test_prefill_then_decode_equals_longer_prefill():
    T1, T2, H = 130, 5, 2
    inp = make(T1 + T2, H, 128, 128, dtype="bf16", seed=21, init_std=0.02)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    k = kda()
    o1, st = k.kda_prefill(inp["q"][:T1], inp["k"][:T1], inp["v"][:T1],
                           inp["log_alpha"][:T1], inp["beta"][:T1], init_state=inp["init_state"])
    outs = [o1]
    for t in range(T1, T1 + T2):
        sl = slice(t, t + 1)
        outs.append(k.kda_decode_step(inp["q"][sl], inp["k"][sl], inp["v"][sl],
                                      inp["log_alpha"][sl], inp["beta"][sl], st))
    torch.cuda.synchronize()
    o = torch.cat(outs)
    assert o_err(f64(o), ref_o, cu, H) <= TOL["bf16"]
    assert state_err(f64(st), ref_s) <= TOL["bf16"]


def test_prefill_single_kernel_path_with_small_workspace():
    """With only the minimum workspace the bf16 d=128 case takes the
    single-kernel tensor-core path; it must match the oracle as well."""
    lens = [130, 0, 64, 257, 1]
    inp = make(0, 2, 128, 128, dtype="bf16", seed=31, lengths=lens, init_std=0.02)
    k = kda()
    small = (256 + ((len(lens) * 4 + 255) // 256) * 256)
    assert small < k.kda_prefill_workspace_size(len(lens), sum(lens), 2, 128, 128)
    ws = torch.empty(small, dtype=torch.uint8, device=DEV)
    o = torch.full((sum(lens), 2, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    o, fs = k.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"], o=o,
                          workspace=ws)
    torch.cuda.synchronize()
    assert k.kda_check_workspace_error(ws) == k.KDA_OK
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]


def test_prefill_many_short_sequences():
    """180 (sequence, head) units of ragged lengths, empty ones included: more
    units than SMs, so the chain runs one CTA per (sequence, head) over the
    whole d_v, after the preparation."""
    rng = np.random.default_rng(123)
    lens = [int(x) for x in rng.integers(0, 200, size=60)]
    lens[3] = 0
    lens[17] = 64
    inp = make(0, 3, 128, 128, dtype="bf16", seed=123, lengths=lens, init_std=0.02)
    o, fs = gpu_prefill(inp)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 3) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]
    assert torch.equal(fs[3], inp["init_state"][3])


def test_prefill_whole_dv_chain_overlapped():
    """40 units of 500-1500 tokens: the chain runs one CTA per (sequence,
    head) over the whole d_v, overlapped with the preparation (records
    consumed as their ready flags appear)."""
    rng = np.random.default_rng(321)
    lens = [int(x) for x in rng.integers(500, 1500, size=10)]
    inp = make(0, 4, 128, 128, dtype="bf16", seed=321, lengths=lens, init_std=0.02)
    o, fs = gpu_prefill(inp)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 4) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]


def test_prefill_single_kernel_path_fast_decay():
    """The single-kernel path on gates of -2 per token (a chunk decays by
    e^-128): every chunk takes the pairwise path."""
    lens = [130, 0, 64, 257, 1]
    inp = make(0, 2, 128, 128, dtype="bf16", seed=37, lengths=lens, init_std=0.02)
    inp["log_alpha"] = torch.full_like(inp["log_alpha"], -2.0)
    k = kda()
    small = (256 + ((len(lens) * 4 + 255) // 256) * 256)
    ws = torch.empty(small, dtype=torch.uint8, device=DEV)
    o = torch.full((sum(lens), 2, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    o, fs = k.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"], o=o,
                          workspace=ws)
    torch.cuda.synchronize()
    assert k.kda_check_workspace_error(ws) == k.KDA_OK
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, 2) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]
