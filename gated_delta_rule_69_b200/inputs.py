"""Seeded synthetic inputs for the KDA operator.

This module holds no arithmetic of the recurrence itself: only the input
distributions the Kimi Linear pages describe for the operator's inputs, drawn
from a seeded torch generator.  Both the CUDA path's tests and the oracle's
tests take their inputs from here.

Distributions (page "Kimi Linear" on docsaid.org, section "Les autres pieces";
news digest page, section "Configuration du modele Kimi Linear"):
  * q, k ~ N(0, 1) then L2-normalised over d_k per (token, head)
    (the pages L2-normalise q and k to keep eigenvalues stable);
  * v ~ N(0, 1);
  * beta = sigmoid(N(0, 1)) per (token, head) (a linear map then a sigmoid);
  * log_alpha = -softplus(N(-2, 1)) per (token, head, key channel), i.e. the
    Kimi Linear decay g = -exp(A) softplus(z) with A = 0;
  * initial state ~ N(0, 0.02^2) in fp32 where a workload has one
    (0.02 is the standard deviation).
Values are drawn in fp32 and rounded once to the I/O dtype (bf16 or fp32).
Draw order: sequence lengths (varlen only), q, k, v, beta logits, gate logits,
initial state.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    """One synthetic operator workload."""
    name: str
    kind: str                      # "prefill" or "decode"
    H: int
    d_k: int
    d_v: int
    dtype: str                     # "bf16" or "fp32" (I/O dtype; state is fp32)
    seed: int
    T: int = 0                     # prefill: tokens per sequence (fixed lengths)
    num_seqs: int = 1
    varlen: tuple = ()             # (lo, hi) inclusive length range for varlen
    batch: int = 0                 # decode: independent sequences
    init_std: float = 0.0          # 0 -> zero initial state
    note: str = field(default="", compare=False)


WORKLOADS = {
    "tiny_T64_H1_d16_fp32": Workload(
        "tiny_T64_H1_d16_fp32", "prefill", H=1, d_k=16, d_v=16, dtype="fp32",
        seed=1000, T=64),
    "prefill_T4096_H16_d128": Workload(
        "prefill_T4096_H16_d128", "prefill", H=16, d_k=128, d_v=128,
        dtype="bf16", seed=1001, T=4096),
    "prefill_T131072_H32_d128": Workload(
        "prefill_T131072_H32_d128", "prefill", H=32, d_k=128, d_v=128,
        dtype="bf16", seed=1002, T=131072, init_std=0.02),
    "varlen_16seq_256to16384_H32_d128": Workload(
        "varlen_16seq_256to16384_H32_d128", "prefill", H=32, d_k=128, d_v=128,
        dtype="bf16", seed=1003, num_seqs=16, varlen=(256, 16384),
        init_std=0.02),
    # a smaller case of the 131072-token workload's kernels (same heads and
    # chain plan), small enough for a full profiler capture
    "prefill_T16384_H32_d128": Workload(
        "prefill_T16384_H32_d128", "prefill", H=32, d_k=128, d_v=128,
        dtype="bf16", seed=1005, T=16384, init_std=0.02),
    "decode_B256_H32_d128": Workload(
        "decode_B256_H32_d128", "decode", H=32, d_k=128, d_v=128,
        dtype="bf16", seed=1004, batch=256, init_std=0.02),
}

_TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32}


def seq_lengths(w: Workload) -> list:
    """Per-sequence lengths, drawn first from the workload's generator."""
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    return _lengths(w, gen)


def _lengths(w: Workload, gen: torch.Generator) -> list:
    if w.kind == "decode":
        return [1] * w.batch
    if w.varlen:
        lo, hi = w.varlen
        return [int(x) for x in torch.randint(lo, hi + 1, (w.num_seqs,), generator=gen)]
    return [w.T] * w.num_seqs


def _normal(shape, gen, mean=0.0, std=1.0, device="cpu"):
    x = torch.empty(shape, dtype=torch.float32, device=device)
    x.normal_(mean, std, generator=gen)
    return x


def generate(w: Workload, device: str = "cpu", lengths=None) -> dict:
    """Draw one workload's inputs.

    Returns a dict of tensors on ``device``:
      q, k, log_alpha [T_tot, H, d_k]; v [T_tot, H, d_v]; beta [T_tot, H]
      (decode: T_tot = batch), all in the I/O dtype;
      init_state [N, H, d_k, d_v] fp32 or None;
      cu_seqlens int32 [N+1] (on ``device``), lengths (python list).
    ``lengths`` overrides the drawn sequence lengths (for smaller test cases).
    Large workloads are much faster to draw with device="cuda"; the values
    then differ from a CPU draw with the same seed.
    """
    gen = torch.Generator(device=device).manual_seed(w.seed)
    cpu_gen = torch.Generator(device="cpu").manual_seed(w.seed)
    drawn = _lengths(w, cpu_gen)
    if lengths is None:
        lengths = drawn
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    H, dk, dv = w.H, w.d_k, w.d_v
    io = _TORCH_DTYPE[w.dtype]

    q = F.normalize(_normal((T, H, dk), gen, device=device), dim=-1)
    k = F.normalize(_normal((T, H, dk), gen, device=device), dim=-1)
    v = _normal((T, H, dv), gen, device=device)
    beta = torch.sigmoid(_normal((T, H), gen, device=device))
    log_alpha = -F.softplus(_normal((T, H, dk), gen, mean=-2.0, device=device))
    n = len(lengths)
    init = None
    if w.init_std > 0:
        init = _normal((n, H, dk, dv), gen, std=w.init_std, device=device)
    cu = torch.zeros(n + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    return dict(q=q.to(io), k=k.to(io), v=v.to(io), beta=beta.to(io),
                log_alpha=log_alpha.to(io), init_state=init,
                cu_seqlens=cu.to(device), lengths=lengths)


def cotangents(w: Workload, lengths, device: str = "cpu", seed_offset: int = 500) -> dict:
    """Seeded upstream gradients for the backward pass (the pages train the
    layer but give no gradient statistics; a loss's gradients are taken as
    N(0, 1) per output element and N(0, 0.02^2) per final-state element):
    d_o [T_tot, H, d_v] in the I/O dtype, d_final_state [N, H, d_k, d_v] fp32.
    Drawn from their own generator (seed + seed_offset)."""
    gen = torch.Generator(device=device).manual_seed(w.seed + seed_offset)
    T, n = int(sum(lengths)), len(lengths)
    d_o = _normal((T, w.H, w.d_v), gen, device=device).to(_TORCH_DTYPE[w.dtype])
    d_fs = _normal((n, w.H, w.d_k, w.d_v), gen, std=0.02, device=device)
    return dict(d_o=d_o, d_final_state=d_fs)


def as_float64(t):
    """Exact widening of a tensor's values to a float64 numpy array (for the
    oracle)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()
