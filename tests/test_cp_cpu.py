"""Context parallelism, on the CPU: the segment decomposition checked with the
fp64 oracle, and the exchange step with two gloo ranks.

Decomposition (course page "Attention lineaire et recurrence", section
"Verification de comprehension"): a segment's pair is (M, S~), M the final
state of the recurrence over the segment with v = 0 from the identity, S~ the
final state from zero; the state entering segment r is M_{r-1} S_in(r-1) +
S~_{r-1}; running every segment from its entering state reproduces the whole
sequence.  This fixes the reading the GPU module follows (it calls the same
steps through the library)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _rand(rng, T, H, dk, dv):
    q = rng.normal(size=(T, H, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.normal(size=(T, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(T, H, dv))
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    s0 = rng.normal(0.0, 0.5, size=(1, H, dk, dv))
    return q, k, v, g, b, s0


@pytest.mark.parametrize("cuts", [[50, 60, 40], [1, 99], [64, 64, 64, 8]])
def test_segment_decomposition_reproduces_the_sequence(oracle_mod, cuts):
    rng = np.random.default_rng(61)
    T, H, dk = sum(cuts), 2, 16
    q, k, v, g, b, s0 = _rand(rng, T, H, dk, dk)
    o_full, s_full = oracle_mod.kda_recurrence(q, k, v, g, b, s0)
    edges = np.concatenate([[0], np.cumsum(cuts)])
    eye = np.broadcast_to(np.eye(dk), (1, H, dk, dk)).copy()
    pairs = []
    for a, e in zip(edges[:-1], edges[1:]):
        sl = slice(a, e)
        _, st = oracle_mod.kda_recurrence(q[sl], k[sl], v[sl], g[sl], b[sl], None)
        _, m = oracle_mod.kda_recurrence(q[sl], k[sl], np.zeros_like(v[sl]), g[sl], b[sl], eye)
        pairs.append((m[0], st[0]))
    s_in = s0[0]
    outs = []
    for r, (a, e) in enumerate(zip(edges[:-1], edges[1:])):
        sl = slice(a, e)
        o_r, s_r = oracle_mod.kda_recurrence(q[sl], k[sl], v[sl], g[sl], b[sl], s_in[None])
        outs.append(o_r)
        m, st = pairs[r]
        s_next = np.einsum("hij,hjk->hik", m, s_in) + st
        assert np.allclose(s_next, s_r[0], atol=1e-11)   # M S_in + S~ = the segment's own end state
        s_in = s_next
    assert np.allclose(np.concatenate(outs), o_full, atol=1e-11)
    assert np.allclose(s_in, s_full[0], atol=1e-11)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gated_delta_rule_69_b200 import context_parallel as cp
        H, dk, dv = 2, 4, 8
        m = torch.full((1, H, dk, dk), float(rank + 1))
        st = torch.full((1, H, dk, dv), 10.0 * (rank + 1))
        ms, ss = cp.exchange(m, st)
        ok = (ms.shape == (world, H, dk, dk) and ss.shape == (world, H, dk, dv) and
              all(torch.all(ms[r] == r + 1) and torch.all(ss[r] == 10.0 * (r + 1)) for r in range(world)))
        out[rank] = 1 if ok else 0
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_gathers_pairs_in_rank_order(world):
    ctx = mp.get_context("spawn")
    out = ctx.Array("i", [0] * world)
    mp.start_processes(_exchange_worker, args=(world, _free_port(), out), nprocs=world,
                       join=True, start_method="spawn")
    assert list(out) == [1] * world
