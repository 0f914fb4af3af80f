"""Context parallelism on one GPU: the ranks run one after another (their
kernels never wait on each other), the exchange replaced by stacking the
pairs; the concatenated outputs and the last segment's end state against the
oracle and against one kda_prefill call over the whole sequence."""
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


def f64(t):
    return t.detach().cpu().double().numpy()


@pytest.mark.parametrize("cuts", [[300, 200, 500], [640, 360], [64, 1, 200, 135]])
def test_cp_prefill_emulated_ranks(cuts):
    from gated_delta_rule_69_b200 import context_parallel as cp
    from gated_delta_rule_69_b200 import kda
    T, H = sum(cuts), 4
    w = kin.Workload("cp", "prefill", H=H, d_k=128, d_v=128, dtype="bf16", seed=71, T=T,
                     init_std=0.02)
    inp = kin.generate(w, device=DEV)
    edges = np.concatenate([[0], np.cumsum(cuts)])
    segs = [tuple(inp[x][a:e].contiguous() for x in ("q", "k", "v", "log_alpha", "beta"))
            for a, e in zip(edges[:-1], edges[1:])]
    pairs = [cp.local_pair(*s) for s in segs]
    ms = torch.cat([p[0] for p in pairs])
    ss = torch.cat([p[1] for p in pairs])
    outs, s_last = [], None
    for r, s in enumerate(segs):
        o_r, s_r = cp.cp_prefill(*s, init_state=inp["init_state"], rank=r,
                                 exchange_fn=lambda m, st: (ms, ss))
        outs.append(o_r)
        s_last = s_r
    torch.cuda.synchronize()
    o = torch.cat(outs)
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    assert o_err(f64(o), ref_o, cu, H) <= TOL["bf16"]
    assert state_err(f64(s_last), ref_s) <= TOL["bf16"]
    # and close to the single call over the whole sequence
    o1, s1 = kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                             init_state=inp["init_state"])
    torch.cuda.synchronize()
    assert o_err(f64(o), f64(o1), cu, H) <= TOL["bf16"]


def test_cp_combine_matches_host_products():
    """kda_cp_combine against the same products in fp64 on the host."""
    from gated_delta_rule_69_b200 import kda
    g = torch.Generator(device="cpu").manual_seed(72)
    n, H, dk, dv = 3, 2, 128, 64
    M = (torch.randn(n, H, dk, dk, generator=g) * 0.05).to(DEV)
    St = torch.randn(n, H, dk, dv, generator=g).to(DEV)
    S0 = torch.randn(H, dk, dv, generator=g).to(DEV)
    for r in range(n + 1):
        out = kda.kda_cp_combine(M[:r].contiguous(), St[:r].contiguous(), S0)
        ref = f64(S0)
        for i in range(r):
            ref = np.einsum("hij,hjk->hik", f64(M[i]), ref) + f64(St[i])
        torch.cuda.synchronize()
        assert np.abs(f64(out) - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())
    zero = kda.kda_cp_combine(M[:0].contiguous(), St[:0].contiguous(), None)
    assert float(zero.abs().max()) == 0.0


def test_cp_local_and_finish_match_plain_prefills():
    """kda_cp_local's pair equals the two plain prefills it stands for (v = 0
    from the identity, and from zero), and kda_cp_finish over the kept
    records equals a plain prefill from the same entering state."""
    from gated_delta_rule_69_b200 import context_parallel as cp
    from gated_delta_rule_69_b200 import kda
    T, H = 333, 3
    w = kin.Workload("cpl", "prefill", H=H, d_k=128, d_v=128, dtype="bf16", seed=73, T=T,
                     init_std=0.02)
    inp = kin.generate(w, device=DEV)
    args = tuple(inp[x] for x in ("q", "k", "v", "log_alpha", "beta"))
    ws = cp.workspace_for(inp["q"])
    m, st = kda.kda_cp_local(*args, ws)
    eye = torch.eye(128, device=DEV).expand(1, H, 128, 128).contiguous()
    _, m_ref = kda.kda_prefill(args[0], args[1], torch.zeros_like(args[2]), args[3], args[4],
                               init_state=eye)
    _, st_ref = kda.kda_prefill(*args)
    torch.cuda.synchronize()
    assert torch.equal(m, m_ref)
    assert torch.equal(st, st_ref)
    o, fs = kda.kda_cp_finish(args[2], inp["init_state"], ws)
    o_ref, fs_ref = kda.kda_prefill(*args, init_state=inp["init_state"])
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    assert torch.equal(fs, fs_ref)
