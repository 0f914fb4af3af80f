"""Context parallelism end to end under a process group: cp_prefill on two and
three ranks (spawned processes, a gloo group whose exchange travels through
host copies), every rank's outputs and the last rank's end state checked
against the fp64 oracle over the whole sequence.

All ranks share the one GPU of this test: their kernels never wait on each
other (the only exchange is the host-side all-gather), so they may run in any
order.  A multi-GPU run takes the same path with NCCL."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_delta_rule_69_b200 import inputs as kin
from parity_util import TOL, o_err, state_err

pytestmark = pytest.mark.gpu

CASES = {2: ([700, 333], 3), 3: ([64, 129, 300], 2)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_delta_rule_69_b200 import build
    build.build()
    import oracle
    oracle.build()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(world):
    cuts, H = CASES[world]
    w = kin.Workload("cpr", "prefill", H=H, d_k=128, d_v=128, dtype="bf16", seed=90 + world,
                     T=sum(cuts), init_std=0.02)
    return kin.generate(w, device="cpu"), cuts


def _worker(rank, world, port, tmpdir):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        from gated_delta_rule_69_b200 import context_parallel as cp
        inp, cuts = _inputs(world)
        a = sum(cuts[:rank])
        sl = slice(a, a + cuts[rank])
        seg = [inp[x][sl].cuda() for x in ("q", "k", "v", "log_alpha", "beta")]
        o, s_end = cp.cp_prefill(*seg, init_state=inp["init_state"].cuda())
        torch.cuda.synchronize()
        torch.save((o.cpu(), s_end.cpu()), os.path.join(tmpdir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_cp_prefill_ranks_match_the_oracle(world, tmp_path):
    import oracle
    from gated_delta_rule_69_b200.inputs import as_float64
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    inp, cuts = _inputs(world)
    T = sum(cuts)
    H = inp["q"].shape[1]
    ref_o, ref_s = oracle.kda_recurrence(*(as_float64(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta")),
                                         init_state=as_float64(inp["init_state"]),
                                         cu_seqlens=np.array([0, T]))
    outs = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    o = torch.cat([x[0] for x in outs]).double().numpy()
    assert o_err(o, ref_o, np.array([0, T]), H) <= TOL["bf16"]
    # each rank's own segment, measured on its own scale too
    edges = np.concatenate([[0], np.cumsum(cuts)])
    for r in range(world):
        assert o_err(o[edges[r]:edges[r + 1]], ref_o[edges[r]:edges[r + 1]],
                     np.array([0, cuts[r]]), H) <= TOL["bf16"], r
    assert state_err(outs[-1][1].double().numpy(), ref_s) <= TOL["bf16"]
