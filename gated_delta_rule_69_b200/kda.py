"""Thin Python binding of libkda.so (the C ABI declared in include/kda.h).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  Functions carry the C names and take torch CUDA tensors (or
None for the optional ones); outputs are allocated here when not supplied.
There is no CPU path: without the built library, or without a CUDA device,
every call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")
_lib = None

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_ERR_CUDA = range(5)
KDA_BF16, KDA_FP32 = 0, 1
EXPORTED = ("kda_status_string", "kda_version", "kda_prefill_workspace_size",
            "kda_prefill", "kda_decode_step", "kda_check_workspace_error",
            "kda_prefill_noalloc", "gdn_prefill", "gdn_decode_step", "kda_layer_prefill",
            "kda_layer_decode_step", "kda_cp_combine", "kda_cp_local", "kda_cp_finish",
            "kda_backward_workspace_size", "kda_backward", "gdn_backward",
            "kda_backward_chunked_workspace_size", "kda_backward_chunked", "gdn_backward_chunked",
            "kda_layer_prefill_workspace_size")


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def lib():
    """Load libkda.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with "
                "`python -m gated_delta_rule_69_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.kda_status_string.argtypes = [ctypes.c_int]
        L.kda_status_string.restype = ctypes.c_char_p
        L.kda_version.restype = ctypes.c_int
        L.kda_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32]
        L.kda_prefill_workspace_size.restype = sz
        L.kda_layer_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32]
        L.kda_layer_prefill_workspace_size.restype = sz
        L.kda_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                  ctypes.c_int, vp, vp, vp, sz, vp]
        L.kda_prefill.restype = ctypes.c_int
        L.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                      ctypes.c_int, vp, vp]
        L.kda_decode_step.restype = ctypes.c_int
        L.gdn_prefill.argtypes = L.kda_prefill.argtypes
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_decode_step.argtypes = L.kda_decode_step.argtypes
        L.gdn_decode_step.restype = ctypes.c_int
        f32 = ctypes.c_float
        L.kda_layer_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, f32, f32, vp, vp, i32, i64,
                                        i32, i32, i32, ctypes.c_int, vp, vp, vp, sz, vp]
        L.kda_layer_prefill.restype = ctypes.c_int
        L.kda_layer_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, f32, f32, vp, i32, i32,
                                            i32, i32, ctypes.c_int, vp, vp]
        L.kda_layer_decode_step.restype = ctypes.c_int
        L.kda_cp_combine.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp]
        L.kda_cp_combine.restype = ctypes.c_int
        L.kda_cp_local.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, ctypes.c_int, vp, vp, vp,
                                   vp, sz, vp]
        L.kda_cp_local.restype = ctypes.c_int
        L.kda_cp_finish.argtypes = [vp, vp, i64, i32, i32, i32, ctypes.c_int, vp, vp, vp, sz, vp]
        L.kda_cp_finish.restype = ctypes.c_int
        L.kda_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                          ctypes.c_int, vp, vp, vp]
        L.kda_prefill_noalloc.restype = ctypes.c_int
        L.kda_backward_workspace_size.argtypes = [i32, i64, i32, i32, i32]
        L.kda_backward_workspace_size.restype = sz
        L.kda_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                   ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.kda_backward.restype = ctypes.c_int
        L.gdn_backward.argtypes = L.kda_backward.argtypes
        L.gdn_backward.restype = ctypes.c_int
        L.kda_backward_chunked_workspace_size.argtypes = [i32, i64, i32]
        L.kda_backward_chunked_workspace_size.restype = sz
        L.kda_backward_chunked.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, vp, vp,
                                           vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.kda_backward_chunked.restype = ctypes.c_int
        L.gdn_backward_chunked.argtypes = L.kda_backward_chunked.argtypes
        L.gdn_backward_chunked.restype = ctypes.c_int
        L.kda_check_workspace_error.argtypes = [vp, vp]
        L.kda_check_workspace_error.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _on(stream):
    """Allocations made for a call that runs on ``stream`` belong to that
    stream: torch's caching allocator then hands their memory to later work
    only in that stream's order, so a buffer the call frees on return cannot
    be reused while the call's kernels still read it."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _check_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def kda_layer_prefill_workspace_size(num_seqs: int, total_tokens: int, H: int, d_k: int, d_v: int) -> int:
    """Workspace for kda_layer_prefill with its prologue as a pass of its own
    (0 for shapes the layer path does not take)."""
    return int(lib().kda_layer_prefill_workspace_size(num_seqs, total_tokens, H, d_k, d_v))


def kda_prefill_workspace_size(num_seqs: int, total_tokens: int, H: int, d_k: int, d_v: int) -> int:
    return int(lib().kda_prefill_workspace_size(num_seqs, total_tokens, H, d_k, d_v))


def kda_prefill(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None,
                num_seqs=None, o=None, final_state=None, workspace=None,
                output_final_state=True, stream=None):
    """Chunkwise KDA prefill.  Shapes: q, k, log_alpha [T, H, d_k]; v [T, H, d_v];
    beta [T, H]; init_state [N, H, d_k, d_v] fp32 or None; cu_seqlens int32
    [N+1] on the device or None (num_seqs equal sequences, default 1).
    Returns (o, final_state); final_state is None if output_final_state is False.
    """
    if log_alpha.shape != q.shape:
        raise ValueError("log_alpha must have q's shape [T, H, d_k]")
    return _prefill("kda_prefill", q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs,
                    o, final_state, workspace, output_final_state, stream)


def gdn_prefill(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None,
                num_seqs=None, o=None, final_state=None, workspace=None,
                output_final_state=True, stream=None):
    """Chunkwise Gated DeltaNet prefill: as kda_prefill with one gate value per
    (token, head), log_alpha [T, H]."""
    if log_alpha.shape != q.shape[:2]:
        raise ValueError("log_alpha must be [T, H]")
    return _prefill("gdn_prefill", q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs,
                    o, final_state, workspace, output_final_state, stream)


def _prefill(fn, q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, o, final_state,
             workspace, output_final_state, stream):
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        n = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
    else:
        n = 1 if num_seqs is None else int(num_seqs)
    need = kda_prefill_workspace_size(n, T, H, dk, dv)
    with _on(stream):
        if o is None:
            o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
        if final_state is None and output_final_state:
            final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check_cuda(q, k, v, log_alpha, beta, init_state, cu_seqlens, o, final_state, workspace)
    st = getattr(lib(), fn)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
        _ptr(cu_seqlens), n, T, H, dk, dv, _dtype_code(q), _ptr(o), _ptr(final_state),
        _ptr(workspace), workspace.numel(), _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, fn)
    return o, final_state


def kda_decode_step(q, k, v, log_alpha, beta, state, o=None, stream=None):
    """One KDA step per sequence; ``state`` [B, H, d_k, d_v] fp32 is updated in
    place.  Returns o [B, H, d_v]."""
    if log_alpha.shape != q.shape:
        raise ValueError("log_alpha must have q's shape [B, H, d_k]")
    return _decode("kda_decode_step", q, k, v, log_alpha, beta, state, o, stream)


def gdn_decode_step(q, k, v, log_alpha, beta, state, o=None, stream=None):
    """One Gated DeltaNet step per sequence (log_alpha [B, H]); ``state`` is
    updated in place.  Returns o [B, H, d_v]."""
    if log_alpha.shape != q.shape[:2]:
        raise ValueError("log_alpha must be [B, H]")
    return _decode("gdn_decode_step", q, k, v, log_alpha, beta, state, o, stream)


def _decode(fn, q, k, v, log_alpha, beta, state, o, stream):
    B, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        with _on(stream):
            o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check_cuda(q, k, v, log_alpha, beta, state, o)
    st = getattr(lib(), fn)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state),
        B, H, dk, dv, _dtype_code(q), _ptr(o), _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, fn)
    return o


def kda_check_workspace_error(workspace=None, stream=None) -> int:
    """Synchronise and return the status of the device-side checks; with
    workspace None, those of kda_prefill_noalloc on the current device."""
    device = workspace.device if workspace is not None else torch.device("cuda", torch.cuda.current_device())
    return int(lib().kda_check_workspace_error(_ptr(workspace), _stream(stream, device)))


def kda_prefill_noalloc(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None,
                        num_seqs=None, o=None, final_state=None, output_final_state=True,
                        stream=None):
    """kda_prefill without a workspace: the library's own fixed device array
    serves as scratch (see include/kda.h).  Same shapes and results as
    kda_prefill; calls that overlap on the GPU must be serialised."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        n = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
    else:
        n = 1 if num_seqs is None else int(num_seqs)
    with _on(stream):
        if o is None:
            o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
        if final_state is None and output_final_state:
            final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
    _check_cuda(q, k, v, log_alpha, beta, init_state, cu_seqlens, o, final_state)
    st = lib().kda_prefill_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
        _ptr(cu_seqlens), n, T, H, dk, dv, _dtype_code(q), _ptr(o), _ptr(final_state),
        _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, "kda_prefill_noalloc")
    return o, final_state


def kda_layer_prefill(q, k, v, gate_z, A_log, beta_logit, out_gate=None, norm_weight=None,
                      qk_eps=1e-6, norm_eps=1e-6, init_state=None, cu_seqlens=None,
                      num_seqs=None, o=None, final_state=None, workspace=None,
                      output_final_state=True, stream=None):
    """KDA prefill with the layer prologue and epilogue (see include/kda.h):
    raw q, k, gate pre-activation gate_z [T, H, d_k], A_log [H] fp32,
    beta_logit [T, H]; optional out_gate [T, H, d_v] and norm_weight [d_v]
    fp32.  bf16, d = 128.  The default workspace takes the path with the
    prologue as a pass of its own; one of kda_prefill_workspace_size bytes
    runs it inside the chunk preparation."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    if gate_z.shape != q.shape or beta_logit.shape != q.shape[:2] or A_log.shape != (H,):
        raise ValueError("gate_z [T, H, d_k], beta_logit [T, H], A_log [H] expected")
    if A_log.dtype != torch.float32 or (norm_weight is not None and norm_weight.dtype != torch.float32):
        raise TypeError("A_log and norm_weight must be float32")
    if cu_seqlens is not None:
        n = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
    else:
        n = 1 if num_seqs is None else int(num_seqs)
    need = kda_layer_prefill_workspace_size(n, T, H, dk, dv) or kda_prefill_workspace_size(n, T, H, dk, dv)
    with _on(stream):
        if o is None:
            o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
        if final_state is None and output_final_state:
            final_state = torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check_cuda(q, k, v, gate_z, A_log, beta_logit, out_gate, norm_weight, init_state,
                cu_seqlens, o, final_state, workspace)
    st = lib().kda_layer_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate_z), _ptr(A_log), _ptr(beta_logit), _ptr(out_gate),
        _ptr(norm_weight), float(qk_eps), float(norm_eps), _ptr(init_state), _ptr(cu_seqlens),
        n, T, H, dk, dv, _dtype_code(q), _ptr(o), _ptr(final_state), _ptr(workspace),
        workspace.numel(), _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, "kda_layer_prefill")
    return o, final_state


def kda_layer_decode_step(q, k, v, gate_z, A_log, beta_logit, state, out_gate=None,
                          norm_weight=None, qk_eps=1e-6, norm_eps=1e-6, o=None, stream=None):
    """One KDA step per sequence with the layer prologue / epilogue fused in;
    ``state`` [B, H, d_k, d_v] fp32 is updated in place.  Returns o [B, H, d_v]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if gate_z.shape != q.shape or beta_logit.shape != q.shape[:2] or A_log.shape != (H,):
        raise ValueError("gate_z [B, H, d_k], beta_logit [B, H], A_log [H] expected")
    if A_log.dtype != torch.float32 or (norm_weight is not None and norm_weight.dtype != torch.float32):
        raise TypeError("A_log and norm_weight must be float32")
    if o is None:
        with _on(stream):
            o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check_cuda(q, k, v, gate_z, A_log, beta_logit, out_gate, norm_weight, state, o)
    st = lib().kda_layer_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate_z), _ptr(A_log), _ptr(beta_logit), _ptr(out_gate),
        _ptr(norm_weight), float(qk_eps), float(norm_eps), _ptr(state), B, H, dk, dv,
        _dtype_code(q), _ptr(o), _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, "kda_layer_decode_step")
    return o


def kda_cp_combine(M, S_tilde, S0=None, S_in=None, stream=None):
    """The state a segment starts from, given the stacked (M, S~) of the
    segments before it: M [n, H, d_k, d_k], S_tilde [n, H, d_k, d_v] fp32, S0
    [H, d_k, d_v] or None.  Returns S_in [H, d_k, d_v]."""
    n, H, dk, _ = M.shape
    dv = S_tilde.shape[-1]
    if S_in is None:
        with _on(stream):
            S_in = torch.empty((H, dk, dv), dtype=torch.float32, device=M.device)
    _check_cuda(M, S_tilde, S0, S_in)
    st = lib().kda_cp_combine(_ptr(M), _ptr(S_tilde), _ptr(S0), _ptr(S_in), n, H, dk, dv,
                              _stream(stream, M.device))
    if st != KDA_OK:
        raise KdaError(st, "kda_cp_combine")
    return S_in


def kda_cp_local(q, k, v, log_alpha, beta, workspace, o_scratch=None, stream=None):
    """One segment's (M [1, H, d_k, d_k], S~ [1, H, d_k, d_v]); the chunk records
    stay in ``workspace`` for kda_cp_finish.  bf16, d = 128, one sequence.
    ``o_scratch`` is accepted for the interface and not written."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    with _on(stream):
        M = torch.empty((1, H, dk, dk), dtype=torch.float32, device=q.device)
        S = torch.empty((1, H, dk, dv), dtype=torch.float32, device=q.device)
    _check_cuda(q, k, v, log_alpha, beta, workspace, o_scratch)
    st = lib().kda_cp_local(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), T, H, dk, dv,
                            _dtype_code(q), _ptr(M), _ptr(S), _ptr(o_scratch), _ptr(workspace),
                            workspace.numel(), _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, "kda_cp_local")
    return M, S


def kda_cp_finish(v, S_in, workspace, o=None, final_state=None, output_final_state=True,
                  stream=None):
    """The segment's outputs and end state from S_in, over the records a
    kda_cp_local call left in ``workspace``."""
    T, H, dv = v.shape
    dk = S_in.shape[-2] if S_in is not None else dv
    with _on(stream):
        if o is None:
            o = torch.empty((T, H, dv), dtype=v.dtype, device=v.device)
        if final_state is None and output_final_state:
            final_state = torch.empty((1, H, dk, dv), dtype=torch.float32, device=v.device)
    _check_cuda(v, S_in, workspace, o, final_state)
    st = lib().kda_cp_finish(_ptr(v), _ptr(S_in), T, H, dk, dv, _dtype_code(v), _ptr(o),
                             _ptr(final_state), _ptr(workspace), workspace.numel(),
                             _stream(stream, v.device))
    if st != KDA_OK:
        raise KdaError(st, "kda_cp_finish")
    return o, final_state


def kda_backward_workspace_size(num_seqs: int, total_tokens: int, H: int, d_k: int, d_v: int) -> int:
    return int(lib().kda_backward_workspace_size(num_seqs, total_tokens, H, d_k, d_v))


def kda_backward(q, k, v, log_alpha, beta, d_o, init_state=None, d_final_state=None,
                 cu_seqlens=None, num_seqs=None, workspace=None, want_d_init_state=True,
                 stream=None):
    """Gradients through kda_prefill given d_o = dL/do [T, H, d_v] and
    d_final_state = dL/dS_T (or None).  Returns fp32 (dq, dk, dv, dlog_alpha,
    dbeta, d_init_state); d_init_state is None unless wanted."""
    if log_alpha.shape != q.shape:
        raise ValueError("log_alpha must have q's shape [T, H, d_k]")
    return _backward("kda_backward", q, k, v, log_alpha, beta, d_o, init_state, d_final_state,
                     cu_seqlens, num_seqs, workspace, want_d_init_state, stream)


def gdn_backward(q, k, v, log_alpha, beta, d_o, init_state=None, d_final_state=None,
                 cu_seqlens=None, num_seqs=None, workspace=None, want_d_init_state=True,
                 stream=None):
    """kda_backward for the Gated DeltaNet gate (log_alpha and dlog_alpha [T, H])."""
    if log_alpha.shape != q.shape[:2]:
        raise ValueError("log_alpha must be [T, H]")
    return _backward("gdn_backward", q, k, v, log_alpha, beta, d_o, init_state, d_final_state,
                     cu_seqlens, num_seqs, workspace, want_d_init_state, stream)


def _backward(fn, q, k, v, log_alpha, beta, d_o, init_state, d_final_state, cu_seqlens,
              num_seqs, workspace, want_d_init_state, stream):
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        n = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
    else:
        n = 1 if num_seqs is None else int(num_seqs)
    f32 = dict(dtype=torch.float32, device=q.device)
    with _on(stream):
        dq = torch.empty((T, H, dk), **f32)
        dkk = torch.empty((T, H, dk), **f32)
        dvv = torch.empty((T, H, dv), **f32)
        dg = torch.empty(tuple(log_alpha.shape), **f32)
        db = torch.empty((T, H), **f32)
        ds0 = torch.empty((n, H, dk, dv), **f32) if want_d_init_state else None
        if workspace is None:
            need = kda_backward_workspace_size(n, T, H, dk, dv)
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check_cuda(q, k, v, log_alpha, beta, d_o, init_state, d_final_state, cu_seqlens, workspace)
    st = getattr(lib(), fn)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
        _ptr(cu_seqlens), n, T, H, dk, dv, _dtype_code(q), _ptr(d_o), _ptr(d_final_state),
        _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(db), _ptr(ds0), _ptr(workspace),
        workspace.numel(), _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, fn)
    return dq, dkk, dvv, dg, db, ds0


def kda_backward_chunked_workspace_size(num_seqs: int, total_tokens: int, H: int) -> int:
    return int(lib().kda_backward_chunked_workspace_size(num_seqs, total_tokens, H))


def kda_backward_chunked(q, k, v, log_alpha, beta, d_o, init_state=None, d_final_state=None,
                         cu_seqlens=None, num_seqs=None, workspace=None, want_d_init_state=True,
                         stream=None):
    """kda_backward by chunks (bf16, d = 128): same arguments and outputs."""
    if log_alpha.shape != q.shape:
        raise ValueError("log_alpha must have q's shape [T, H, d_k]")
    return _backward_chunked("kda_backward_chunked", q, k, v, log_alpha, beta, d_o, init_state,
                             d_final_state, cu_seqlens, num_seqs, workspace, want_d_init_state, stream)


def gdn_backward_chunked(q, k, v, log_alpha, beta, d_o, init_state=None, d_final_state=None,
                         cu_seqlens=None, num_seqs=None, workspace=None, want_d_init_state=True,
                         stream=None):
    """kda_backward_chunked for the Gated DeltaNet gate (log_alpha and
    dlog_alpha [T, H])."""
    if log_alpha.shape != q.shape[:2]:
        raise ValueError("log_alpha must be [T, H]")
    return _backward_chunked("gdn_backward_chunked", q, k, v, log_alpha, beta, d_o, init_state,
                             d_final_state, cu_seqlens, num_seqs, workspace, want_d_init_state, stream)


def _backward_chunked(fn, q, k, v, log_alpha, beta, d_o, init_state, d_final_state, cu_seqlens,
                      num_seqs, workspace, want_d_init_state, stream):
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        n = cu_seqlens.numel() - 1
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
    else:
        n = 1 if num_seqs is None else int(num_seqs)
    f32 = dict(dtype=torch.float32, device=q.device)
    with _on(stream):
        dq = torch.empty((T, H, dk), **f32)
        dkk = torch.empty((T, H, dk), **f32)
        dvv = torch.empty((T, H, dv), **f32)
        dg = torch.empty(tuple(log_alpha.shape), **f32)
        db = torch.empty((T, H), **f32)
        ds0 = torch.empty((n, H, dk, dv), **f32) if want_d_init_state else None
        if workspace is None:
            need = kda_backward_chunked_workspace_size(n, T, H)
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check_cuda(q, k, v, log_alpha, beta, d_o, init_state, d_final_state, cu_seqlens, workspace)
    st = getattr(lib(), fn)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(init_state),
        _ptr(cu_seqlens), n, T, H, _ptr(d_o), _ptr(d_final_state), _ptr(dq), _ptr(dkk),
        _ptr(dvv), _ptr(dg), _ptr(db), _ptr(ds0), _ptr(workspace), workspace.numel(),
        _stream(stream, q.device))
    if st != KDA_OK:
        raise KdaError(st, fn)
    return dq, dkk, dvv, dg, db, ds0
