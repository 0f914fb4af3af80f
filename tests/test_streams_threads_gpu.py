"""Calls from several host threads and on side streams.

* Two host threads make the library's first calls in a fresh process at the
  same time, each on its own stream: the per-device launch settings are set
  up under a lock, and both results equal a later serial call bit for bit
  (the prefill is deterministic: each record's arithmetic does not depend on
  which SM computes it).
* A call on a side stream with no workspace given: the binding allocates the
  workspace for that stream, so memory the caller allocates and overwrites on
  the default stream right after the call cannot be the workspace the call's
  kernels are still reading.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin
from parity_util import TOL, o_err, run_oracle, state_err

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_69_b200 import build
    build.build()
    import oracle
    oracle.build()


_THREADS_SCRIPT = textwrap.dedent("""
    import sys, threading
    sys.path.insert(0, {root!r})
    import torch
    from gated_delta_rule_69_b200 import inputs as kin
    from gated_delta_rule_69_b200 import kda
    torch.cuda.init()
    cases = []
    for i, (T, H, lens) in enumerate([(700, 3, None), (0, 4, [300, 0, 129, 64])]):
        w = kin.Workload("thr", "prefill", H=H, d_k=128, d_v=128, dtype="bf16",
                         seed=70 + i, T=T, init_std=0.02)
        cases.append(kin.generate(w, device="cuda", lengths=lens))
    torch.cuda.synchronize()
    gate = threading.Barrier(2)
    outs = [None, None]
    errs = []

    def work(i):
        try:
            s = torch.cuda.Stream()
            inp = cases[i]
            gate.wait()
            with torch.cuda.stream(s):
                o, fs = kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                        inp["beta"], init_state=inp["init_state"],
                                        cu_seqlens=inp["cu_seqlens"], stream=s)
            s.synchronize()
            outs[i] = (o, fs)
        except Exception as e:  # reported by the main thread
            errs.append(repr(e))

    ts = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errs, errs
    for i, inp in enumerate(cases):
        o, fs = kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"])
        torch.cuda.synchronize()
        assert torch.equal(o, outs[i][0]), i
        assert torch.equal(fs, outs[i][1]), i
    torch.save([(outs[i][0].cpu(), outs[i][1].cpu()) for i in range(2)], sys.argv[1])
    print("threads ok")
""")


def test_first_calls_from_two_threads(tmp_path):
    script = tmp_path / "threads.py"
    script.write_text(_THREADS_SCRIPT.format(root=ROOT))
    out = tmp_path / "outs.pt"
    r = subprocess.run([sys.executable, str(script), str(out)], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "threads ok" in r.stdout
    # and the threaded results against the oracle
    got = torch.load(out)
    for i, (T, H, lens) in enumerate([(700, 3, None), (0, 4, [300, 0, 129, 64])]):
        w = kin.Workload("thr", "prefill", H=H, d_k=128, d_v=128, dtype="bf16",
                         seed=70 + i, T=T, init_std=0.02)
        inp = kin.generate(w, device="cuda", lengths=lens)
        ref_o, ref_s, cu, _, _ = run_oracle(inp)
        o, fs = got[i]
        assert o_err(o.double().numpy(), ref_o, cu, H) <= TOL["bf16"]
        assert state_err(fs.double().numpy(), ref_s) <= TOL["bf16"]


def test_side_stream_call_keeps_its_workspace():
    from gated_delta_rule_69_b200 import kda
    w = kin.Workload("side", "prefill", H=8, d_k=128, d_v=128, dtype="bf16", seed=81,
                     T=2048, init_std=0.02)
    inp = kin.generate(w, device="cuda")
    need = kda.kda_prefill_workspace_size(1, 2048, 8, 128, 128)
    side = torch.cuda.Stream()
    results = []
    for _ in range(3):
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            torch.cuda._sleep(50_000_000)   # the side stream's work starts well after the code below
        o, fs = kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                init_state=inp["init_state"], stream=side)
        # on the default stream: buffers of the workspace's size, overwritten at once
        junk = [torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda") for _ in range(2)]
        del junk
        torch.cuda.current_stream().wait_stream(side)
        results.append((o.clone(), fs.clone()))
    torch.cuda.synchronize()
    ref_o, ref_s, cu, _, _ = run_oracle(inp)
    for o, fs in results:
        assert o_err(o.double().cpu().numpy(), ref_o, cu, 8) <= TOL["bf16"]
        assert state_err(fs.double().cpu().numpy(), ref_s) <= TOL["bf16"]
    assert all(torch.equal(results[0][0], r[0]) for r in results[1:])
