"""Full-size prefill workloads through the same C-ABI call bench.py times,
checked against the fp64 oracle on every output and state element of the
sampled (sequence, head) units."""
import numpy as np
import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin
from parity_util import TOL, o_err, run_oracle, state_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_69_b200 import build
    build.build()
    import oracle
    oracle.build()


def _run(inp):
    from gated_delta_rule_69_b200 import kda
    T, H, _ = inp["q"].shape
    o = torch.full((T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    o, fs = kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"], o=o)
    torch.cuda.synchronize()
    return o, fs


def _check(inp, o, fs, heads, seqs):
    ref_o, ref_s, sub_cu, rows, hs = run_oracle(inp, heads=heads, seqs=seqs)
    rows_t = torch.as_tensor(rows, device="cuda")
    hh = torch.as_tensor(hs, device="cuda")
    got_o = o.index_select(0, rows_t).index_select(1, hh).double().cpu().numpy()
    got_s = fs.index_select(0, torch.as_tensor(seqs, device="cuda")).index_select(1, hh)
    e_o = o_err(got_o, ref_o, sub_cu, len(hs))
    e_s = state_err(got_s.double().cpu().numpy(), ref_s)
    assert bool(torch.isfinite(o).all()), "unwritten or non-finite outputs"
    assert e_o <= TOL["bf16"], e_o
    assert e_s <= TOL["bf16"], e_s
    return e_o, e_s


def test_prefill_T4096_H16_all_heads():
    w = kin.WORKLOADS["prefill_T4096_H16_d128"]
    inp = kin.generate(w, device="cuda")
    o, fs = _run(inp)
    _check(inp, o, fs, heads=list(range(16)), seqs=[0])


def test_prefill_T131072_H32_sampled_heads():
    """Long prefill: 4 heads drawn from a seeded generator, all 131072 tokens."""
    w = kin.WORKLOADS["prefill_T131072_H32_d128"]
    inp = kin.generate(w, device="cuda")
    o, fs = _run(inp)
    heads = sorted(np.random.default_rng(w.seed).choice(32, 4, replace=False).tolist())
    _check(inp, o, fs, heads=heads, seqs=[0])


def test_varlen_16seq_all_units():
    """Packed varlen batch: every one of the 16 sequences and all 32 heads
    (512 units, about 4.3 M (token, head) pairs), each checked on every
    output and final-state element, so that every sequence's state reset and
    ragged last chunk is compared.  The oracle runs on 4 heads at a time to
    bound host memory (its fp64 copies of 4 heads are ~3 GB)."""
    w = kin.WORKLOADS["varlen_16seq_256to16384_H32_d128"]
    inp = kin.generate(w, device="cuda")
    o, fs = _run(inp)
    seqs = list(range(len(inp["lengths"])))
    worst_o = worst_s = 0.0
    for h0 in range(0, 32, 4):
        e_o, e_s = _check(inp, o, fs, heads=list(range(h0, h0 + 4)), seqs=seqs)
        worst_o, worst_s = max(worst_o, e_o), max(worst_s, e_s)
    print(f"varlen all units: worst o error {worst_o:.3e}, worst state error {worst_s:.3e}")
