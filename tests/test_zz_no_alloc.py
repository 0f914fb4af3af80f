"""kda_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory (for instance an engine whose device memory all
belongs to its own pool, or a plugin host that only passes a stream and
tensors).  Its scratch is a fixed array inside libkda.so, so these tests
check that it gives the same results as kda_prefill with a caller-provided
workspace, call after call, and that it refuses problems larger than that
array.

This file is named to be collected last, so that a run stopping at the first
failure has run every other test before it."""
import ctypes

import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin


def _kda():
    from gated_delta_rule_69_b200 import build, kda
    build.build()
    return kda


def test_noalloc_rejects_too_many_sequences_on_host():
    """More sequences than the built-in array can order: a clear error, and
    no CUDA call is made (the pointers below are never dereferenced)."""
    kda = _kda()
    L = kda.lib()
    fake = ctypes.c_void_p(1 << 20)
    st = L.kda_prefill_noalloc(fake, fake, fake, fake, fake, None, fake, 4097, 4097 * 64, 1,
                               128, 128, kda.KDA_BF16, ctypes.c_void_p(1 << 24), None, None)
    assert st == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,dk,dv,tol", [("bf16", 128, 128, 2e-2), ("fp32", 64, 32, 1e-4)])
def test_noalloc_matches_prefill_two_calls(dtype, dk, dv, tol):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda = _kda()
    w = kin.Workload("noalloc", "prefill", H=3, d_k=dk, d_v=dv, dtype=dtype, seed=4242, T=0,
                     init_std=0.02)
    # two different problems, so the second call cannot pass on the first
    # call's leftovers in the shared scratch array
    for lengths in ([70, 0, 129, 64], [200, 1]):
        inp = kin.generate(w, device="cuda", lengths=lengths)
        args = (inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"])
        ref_o, ref_s = kda.kda_prefill(*args, init_state=inp["init_state"],
                                       cu_seqlens=inp["cu_seqlens"])
        o = torch.full_like(ref_o, float("nan"))
        o, s = kda.kda_prefill_noalloc(*args, init_state=inp["init_state"],
                                       cu_seqlens=inp["cu_seqlens"], o=o)
        torch.cuda.synchronize()
        scale_o = ref_o.float().abs().max().clamp_min(1e-30)
        scale_s = ref_s.abs().max().clamp_min(1e-30)
        assert torch.isfinite(o.float()).all()
        assert ((o.float() - ref_o.float()).abs().max() / scale_o).item() <= tol
        assert ((s - ref_s).abs().max() / scale_s).item() <= tol


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 16)])
def test_noalloc_reports_device_errors(dtype, d):
    """The device-side check of cu_seqlens (a non-monotone one here) leaves
    its error word in the built-in array, where kda_check_workspace_error with
    no workspace reads it; the next good call clears it."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kda = _kda()
    w = kin.Workload("noalloc_err", "prefill", H=1, d_k=d, d_v=d, dtype=dtype, seed=4343, T=0)
    inp = kin.generate(w, device="cuda", lengths=[10, 10])
    args = (inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"])
    bad = torch.tensor([0, 15, 10, 20], dtype=torch.int32, device="cuda")
    kda.kda_prefill_noalloc(*args, cu_seqlens=bad)
    assert kda.kda_check_workspace_error() == kda.KDA_ERR_INVALID_ARG
    kda.kda_prefill_noalloc(*args, cu_seqlens=inp["cu_seqlens"])
    assert kda.kda_check_workspace_error() == kda.KDA_OK
