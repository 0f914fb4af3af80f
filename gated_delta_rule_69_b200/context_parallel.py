"""KDA context parallelism: one sequence cut into consecutive segments, one per
rank (course page "Attention lineaire et recurrence", section "Verification de
comprehension": a segment carries its cumulative transition M and the state it
generates locally, S~; the state entering segment r is S_in(r) = M_{r-1}
S_in(r-1) + S~_{r-1}).

Per rank, all on the GPU in the library's kernels, with one chunk
preparation:
  1. kda_cp_local: the segment's chunk records, then over them the state
     chain from zero (S~) and from the identity with v counting as zero (M);
  2. exchange: all-gather of (M, S~) over the group (NCCL over NVLink);
  3. kda_cp_combine forms S_in(rank) from the pairs of lower ranks;
  4. kda_cp_finish: the chain once more over the same records from S_in(rank):
     the outputs, and on the last rank the sequence's final state.
The pages give the decomposition, not a schedule: this one runs the chain
three times per rank (two before the exchange), the preparation once.
"""
from __future__ import annotations

import contextlib

import torch

from . import kda


def workspace_for(q):
    T, H, dk = q.shape
    n = kda.kda_prefill_workspace_size(1, T, H, dk, dk)
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def local_pair(q, k, v, log_alpha, beta, workspace=None, stream=None):
    """(M, S~) of one segment, each [1, H, d_k, d_*]; the segment's chunk
    records stay in ``workspace`` (allocated if None) for the final pass."""
    if v.shape[-1] != q.shape[-1]:
        raise ValueError("context parallelism needs d_v = d_k (M is d_k x d_k)")
    if workspace is None:
        ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
        with ctx:   # the workspace belongs to the stream its kernels run on
            workspace = workspace_for(q)
    return kda.kda_cp_local(q, k, v, log_alpha, beta, workspace, stream=stream)


def exchange(m, s_tilde, group=None):
    """All-gather of every rank's (M, S~): returns [world, H, d_k, d_*] each, in
    rank order, on the device of ``m``.  Over NCCL the device tensors travel
    directly (NVLink); a gloo group exchanges host copies."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    host = dist.get_backend(group) != "nccl"
    dev = m.device
    m_x = m.contiguous().cpu() if host else m.contiguous()
    s_x = s_tilde.contiguous().cpu() if host else s_tilde.contiguous()
    ms = [torch.empty_like(m_x) for _ in range(world)]
    ss = [torch.empty_like(s_x) for _ in range(world)]
    dist.all_gather(ms, m_x, group=group)
    dist.all_gather(ss, s_x, group=group)
    return torch.cat(ms).to(dev), torch.cat(ss).to(dev)


def cp_prefill(q, k, v, log_alpha, beta, init_state=None, group=None, workspace=None,
               stream=None, exchange_fn=None, rank=None):
    """Context-parallel KDA prefill of one sequence.  This rank holds the
    segment q, k, v, log_alpha, beta ([T_r, H, ...]) at position `rank` (its
    rank in `group`); init_state [1, H, d_k, d_v] is the sequence's initial
    state, the same on every rank (or None).  Returns (o for the segment, the
    state after it); the last rank's is the sequence's final state.
    ``exchange_fn(m, s_tilde)`` replaces the collective (returns the stacked
    pairs of all ranks), e.g. to run the ranks one after another on one GPU.
    With ``stream``, every step, the collective included, is ordered on it
    (it becomes torch's current stream for the call)."""
    if rank is None:
        import torch.distributed as dist
        rank = dist.get_rank(group)
    # every allocation below, the workspace included, belongs to the stream
    # the work runs on, so torch's allocator reuses its memory only after
    # that work in the stream's order
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        if workspace is None:
            workspace = workspace_for(q)
        m, s_tilde = local_pair(q, k, v, log_alpha, beta, workspace=workspace, stream=stream)
        if exchange_fn is not None:
            ms, ss = exchange_fn(m, s_tilde)
        else:
            ms, ss = exchange(m, s_tilde, group)
        s0 = None if init_state is None else init_state.reshape(init_state.shape[-3:]).contiguous()
        s_in = kda.kda_cp_combine(ms[:rank].contiguous(), ss[:rank].contiguous(), s0,
                                  stream=stream)
        return kda.kda_cp_finish(v, s_in.unsqueeze(0), workspace, stream=stream)
