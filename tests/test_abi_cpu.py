"""libkda.so loads on a host without a GPU, exports every function that
include/kda.h declares, and rejects bad arguments on the host before any CUDA
call.  CPU only: the pointers passed here are never dereferenced."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_69_b200 import build, kda
    build.build()
    return kda.lib()


def _declared_functions():
    names = []
    for path in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if path.endswith(".h"):
            text = open(os.path.join(ROOT, "include", path)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b((?:kda|gdn)_\w+)\s*\(", text)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert "kda_prefill" in names and "kda_decode_step" in names
    assert "gdn_prefill" in names and "gdn_decode_step" in names
    for n in names:
        assert hasattr(L, n), f"libkda.so does not export {n}"


def test_binding_names_match_header():
    from gated_delta_rule_69_b200 import kda
    for n in _declared_functions():
        if n in ("kda_status_string", "kda_version"):
            continue
        assert hasattr(kda, n), f"binding lacks {n}"


def test_status_strings(L):
    for s in range(5):
        assert L.kda_status_string(s).startswith(b"KDA_")
    assert L.kda_status_string(99) == b"KDA_ERR_UNKNOWN"


def test_workspace_size(L):
    ws = L.kda_prefill_workspace_size
    assert ws(1, 4096, 16, 128, 128) >= 256
    assert ws(1, 4096, 16, 128, 128) % 256 == 0
    assert ws(0, 10, 1, 16, 16) == 0
    assert ws(1, 10, 1, 48, 16) == 0
    assert ws(1, -1, 1, 16, 16) == 0


def test_layer_workspace_size(L):
    """The layer's workspace is the prefill's plus what its prologue pass
    leaves for the operator: the inverse norms of the k and q rows (fp32 pairs),
    log_alpha per (token, head, channel) and beta per (token, head) in bf16,
    each 256-byte aligned; the normalised q and k are never written."""
    up = lambda x: (x + 255) // 256 * 256
    for n, T, H in ((1, 4096, 16), (1, 131072, 32), (16, 133_000, 32), (3, 1, 1)):
        base = L.kda_prefill_workspace_size(n, T, H, 128, 128)
        lay = L.kda_layer_prefill_workspace_size(n, T, H, 128, 128)
        assert lay == up(base) + up(T * H * 8) + up(T * H * 128 * 2) + up(T * H * 2), (n, T, H)
    assert L.kda_layer_prefill_workspace_size(1, 4096, 16, 64, 128) == 0
    assert L.kda_layer_prefill_workspace_size(0, 4096, 16, 128, 128) == 0


FAKE = 1 << 20  # 16-byte aligned, never dereferenced on the host


def _prefill(L, fn="kda_prefill", **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, g=FAKE * 4, b=FAKE * 5, s0=None, cu=None,
             n=1, T=64, H=1, dk=16, dv=16, dt=1, o=FAKE * 64, fs=None, ws=FAKE * 128,
             wsb=4096)
    a.update(kw)
    return getattr(L, fn)(a["q"], a["k"], a["v"], a["g"], a["b"], a["s0"], a["cu"],
                          a["n"], a["T"], a["H"], a["dk"], a["dv"], a["dt"], a["o"],
                          a["fs"], a["ws"], a["wsb"], None)


def test_prefill_rejects_on_host(L):
    assert _prefill(L, n=0) == 1
    assert _prefill(L, H=0) == 1
    assert _prefill(L, T=-1) == 1
    assert _prefill(L, dt=7) == 1
    assert _prefill(L, dk=48) == 2
    assert _prefill(L, dv=256) == 2
    assert _prefill(L, q=None) == 1
    assert _prefill(L, q=FAKE + 4) == 1            # misaligned
    assert _prefill(L, n=3, T=64) == 1             # T % N != 0 without cu_seqlens
    assert _prefill(L, ws=None) == 3
    assert _prefill(L, wsb=16) == 3
    assert _prefill(L, ws=FAKE * 128 + 16) == 1    # workspace not 256-aligned
    assert _prefill(L, o=FAKE + 64) == 1           # o overlaps q


def _decode(L, fn="kda_decode_step", **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, g=FAKE * 4, b=FAKE * 5, s=FAKE * 16,
             B=4, H=2, dk=16, dv=16, dt=1, o=FAKE * 64)
    a.update(kw)
    return getattr(L, fn)(a["q"], a["k"], a["v"], a["g"], a["b"], a["s"], a["B"],
                             a["H"], a["dk"], a["dv"], a["dt"], a["o"], None)


def test_decode_rejects_on_host(L):
    assert _decode(L, B=0) == 0                    # empty batch: no-op
    assert _decode(L, B=-1) == 1
    assert _decode(L, H=0) == 1
    assert _decode(L, dk=8) == 2
    assert _decode(L, s=None) == 1
    assert _decode(L, o=FAKE * 16 + 32) == 1       # o overlaps the state
    assert _decode(L, v=FAKE * 3 + 2) == 1         # not element-aligned (fp32)
    assert _decode(L, s=FAKE * 16 + 8) == 1        # state not 16-byte aligned


def test_gdn_rejects_on_host(L):
    # the scalar gate needs only element alignment; everything else as for KDA
    assert _prefill(L, "gdn_prefill", g=FAKE * 4 + 4, ws=None) == 3   # alignment passed, no workspace
    assert _prefill(L, "gdn_prefill", g=FAKE * 4 + 2) == 1            # fp32 gate not 4-byte aligned
    assert _prefill(L, "gdn_prefill", n=0) == 1
    assert _prefill(L, "gdn_prefill", dk=48) == 2
    assert _prefill(L, "gdn_prefill", q=FAKE + 4) == 1
    # o [64, 1, 16] fp32 at FAKE * 64 (4 KB) overlaps a gate placed right below its end
    assert _prefill(L, "gdn_prefill", g=FAKE * 64 + 4096 - 128) == 1
    assert _decode(L, "gdn_decode_step", B=0) == 0
    assert _decode(L, "gdn_decode_step", g=FAKE * 4 + 2) == 1
    assert _decode(L, "gdn_decode_step", s=None) == 1


def test_binding_checks_gate_shape():
    import torch
    from gated_delta_rule_69_b200 import kda
    x = torch.zeros(4, 2, 16)
    with pytest.raises(ValueError):
        kda.gdn_decode_step(x, x, x, x, torch.zeros(4, 2), torch.zeros(4, 2, 16, 16))
    with pytest.raises(ValueError):
        kda.kda_decode_step(x, x, x, torch.zeros(4, 2), torch.zeros(4, 2), torch.zeros(4, 2, 16, 16))


def test_binding_refuses_cpu_tensors():
    import torch
    from gated_delta_rule_69_b200 import kda
    x = torch.zeros(4, 1, 16)
    with pytest.raises((ValueError, RuntimeError, AssertionError)):
        kda.kda_decode_step(x, x, x, x, torch.zeros(4, 1), torch.zeros(4, 1, 16, 16))


def _backward(L, fn="kda_backward", **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, g=FAKE * 4, b=FAKE * 5, s0=None, cu=None,
             n=1, T=64, H=1, dk=32, dv=32, dt=1, do=FAKE * 6, dfs=None, dq=FAKE * 64,
             dkk=FAKE * 65, dvv=FAKE * 66, dg=FAKE * 67, db=FAKE * 68, ds0=None,
             ws=FAKE * 128, wsb=1 << 30)
    a.update(kw)
    return getattr(L, fn)(a["q"], a["k"], a["v"], a["g"], a["b"], a["s0"], a["cu"], a["n"],
                          a["T"], a["H"], a["dk"], a["dv"], a["dt"], a["do"], a["dfs"],
                          a["dq"], a["dkk"], a["dvv"], a["dg"], a["db"], a["ds0"], a["ws"],
                          a["wsb"], None)


def test_backward_workspace_size(L):
    ws = L.kda_backward_workspace_size
    # kept states: one 128 x 128 fp32 state per 64 tokens per head, plus slack per sequence
    assert ws(1, 4096, 16, 128, 128) >= 4096 // 64 * 16 * 128 * 128 * 4
    assert ws(0, 64, 1, 32, 32) == 0
    assert ws(1, 64, 1, 16, 32) == 0
    assert ws(1, 64, 1, 32, 48) == 0


def test_backward_rejects_on_host(L):
    for fn in ("kda_backward", "gdn_backward"):
        assert _backward(L, fn, n=0) == 1
        assert _backward(L, fn, dt=5) == 1
        assert _backward(L, fn, dk=16) == 2
        assert _backward(L, fn, dv=48) == 2
        assert _backward(L, fn, do=None) == 1
        assert _backward(L, fn, dq=None) == 1
        assert _backward(L, fn, n=3) == 1                   # T % N != 0 without cu_seqlens
        assert _backward(L, fn, v=FAKE * 3 + 4) == 1        # v not 16-byte aligned
        assert _backward(L, fn, dvv=FAKE * 66 + 8) == 1     # dv not 16-byte aligned
        assert _backward(L, fn, wsb=1024) == 3
        assert _backward(L, fn, ws=FAKE * 128 + 16) == 1    # workspace not 256-aligned
        assert _backward(L, fn, dq=FAKE + 64) == 1          # dq overlaps q
        assert _backward(L, fn, dkk=FAKE * 64 + 64) == 1    # dk overlaps dq
        assert _backward(L, fn, ds0=FAKE * 128 + 4096) == 1  # d_init_state inside the workspace


def test_binding_checks_backward_gate_shape():
    import torch
    from gated_delta_rule_69_b200 import kda
    x = torch.zeros(4, 2, 32)
    b = torch.zeros(4, 2)
    with pytest.raises(ValueError):   # per-head gate given to the per-channel entry
        kda.kda_backward(x, x, x, b, b, x)
    with pytest.raises(ValueError):   # per-channel gate given to the per-head entry
        kda.gdn_backward(x, x, x, x, b, x)


def _backward_chunked(L, fn="kda_backward_chunked", **kw):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, g=FAKE * 4, b=FAKE * 5, s0=None, cu=None,
             n=1, T=64, H=1, do=FAKE * 6, dfs=None, dq=FAKE * 64, dkk=FAKE * 65,
             dvv=FAKE * 66, dg=FAKE * 67, db=FAKE * 68, ds0=None, ws=FAKE * 128, wsb=1 << 40)
    a.update(kw)
    return getattr(L, fn)(a["q"], a["k"], a["v"], a["g"], a["b"], a["s0"], a["cu"], a["n"],
                          a["T"], a["H"], a["do"], a["dfs"], a["dq"], a["dkk"], a["dvv"],
                          a["dg"], a["db"], a["ds0"], a["ws"], a["wsb"], None)


def test_backward_chunked_workspace_size(L):
    ws = L.kda_backward_chunked_workspace_size
    # at least the prefill's split workspace and two bf16 state tiles (32 KB each) per record
    for n, T, H in ((1, 4096, 16), (3, 1000, 2)):
        chunks = T // 64 + n
        assert ws(n, T, H) >= L.kda_prefill_workspace_size(n, T, H, 128, 128) + 2 * chunks * H * 32768
    assert ws(0, 64, 1) == 0


def test_backward_chunked_rejects_on_host(L):
    """Every refusal is decided on the host, before any CUDA call."""
    for fn in ("kda_backward_chunked", "gdn_backward_chunked"):
        assert _backward_chunked(L, fn, n=0) == 1
        assert _backward_chunked(L, fn, T=0) == 1
        assert _backward_chunked(L, fn, n=3) == 1                # T % N != 0 without cu_seqlens
        assert _backward_chunked(L, fn, do=None) == 1
        assert _backward_chunked(L, fn, dq=None) == 1
        assert _backward_chunked(L, fn, q=FAKE + 4) == 1         # q not 16-byte aligned
        assert _backward_chunked(L, fn, dvv=FAKE * 66 + 8) == 1  # dv not 16-byte aligned
        assert _backward_chunked(L, fn, dq=FAKE * 64 + 2) == 1   # dq not 4-byte aligned
        assert _backward_chunked(L, fn, b=FAKE * 5 + 1) == 1     # beta not 2-byte aligned
        assert _backward_chunked(L, fn, wsb=1024) == 3           # workspace too small
        assert _backward_chunked(L, fn, ws=None) == 3
        assert _backward_chunked(L, fn, ws=FAKE * 128 + 16) == 1  # workspace not 256-aligned
    # the per-channel gate is a 16-byte aligned tile; the scalar gate needs 2 bytes only
    assert _backward_chunked(L, "kda_backward_chunked", g=FAKE * 4 + 2) == 1
    assert _backward_chunked(L, "gdn_backward_chunked", g=FAKE * 4 + 1) == 1


BF16, FP32 = 0, 1   # kda_dtype


def test_cp_entries_reject_on_host(L):
    """kda_cp_combine / kda_cp_local / kda_cp_finish decide every refusal on the
    host: shapes without a kernel, null or misaligned pointers, too small or
    misaligned workspaces, outputs over inputs."""
    big = 1 << 40
    ws = FAKE * 1024
    # combine: S_in [H, d_k, d_v] from n_prev (M, S~) pairs
    cmb = lambda **kw: L.kda_cp_combine(kw.get("M", FAKE), kw.get("St", FAKE * 2), kw.get("S0", None),
                                        kw.get("Sin", FAKE * 8), kw.get("n", 1), kw.get("H", 1),
                                        kw.get("dk", 32), kw.get("dv", 32), None)
    assert cmb(n=-1) == 1
    assert cmb(H=0) == 1
    assert cmb(dv=16) == 2                       # d_v below 32
    assert cmb(dk=48) == 2
    assert cmb(Sin=None) == 1
    assert cmb(M=None) == 1                      # n_prev > 0 needs M and S~
    assert cmb(Sin=FAKE * 8 + 2) == 1            # not 4-byte aligned
    assert cmb(Sin=FAKE + 64) == 1               # S_in inside M
    # local: bf16, d = 128 only
    loc = lambda **kw: L.kda_cp_local(kw.get("q", FAKE), kw.get("k", FAKE * 2), kw.get("v", FAKE * 3),
                                      kw.get("g", FAKE * 4), kw.get("b", FAKE * 5), kw.get("T", 64),
                                      kw.get("H", 1), kw.get("dk", 128), kw.get("dv", 128),
                                      kw.get("dt", BF16), kw.get("M", FAKE * 8), kw.get("St", FAKE * 9),
                                      kw.get("os", None), kw.get("ws", ws), kw.get("wsb", big), None)
    assert loc(T=0) == 1
    assert loc(dt=FP32) == 2
    assert loc(dk=64) == 2
    assert loc(M=None) == 1
    assert loc(q=FAKE + 8) == 1                  # not 16-byte aligned
    assert loc(b=FAKE * 5 + 1) == 1
    assert loc(wsb=1024) == 3
    assert loc(ws=None) == 3
    assert loc(ws=ws + 16) == 1                  # workspace not 256-aligned
    assert loc(M=FAKE * 3) == 1                  # M over v
    assert loc(St=FAKE * 8) == 1                 # S~ over M
    # finish: the chain again over the kept records
    fin = lambda **kw: L.kda_cp_finish(kw.get("v", FAKE * 3), kw.get("Sin", FAKE * 8), kw.get("T", 64),
                                       kw.get("H", 1), kw.get("dk", 128), kw.get("dv", 128),
                                       kw.get("dt", BF16), kw.get("o", FAKE * 16), kw.get("fs", None),
                                       kw.get("ws", ws), kw.get("wsb", big), None)
    assert fin(T=0) == 1
    assert fin(dv=64) == 2
    assert fin(o=None) == 1
    assert fin(o=FAKE * 16 + 4) == 1
    assert fin(wsb=16) == 3
    assert fin(ws=ws + 64) == 1
    assert fin(o=FAKE * 3) == 1                  # o over v
    assert fin(fs=FAKE * 16 + 1024) == 1         # final state inside o


def test_layer_prefill_rejects_on_host(L):
    """kda_layer_prefill: the two-kernel tensor-core path only (bf16, d = 128,
    at least the prefill's workspace), A_log required, eps >= 0, the output
    gate not under o; all decided on the host."""
    T, H = 64, 1
    big = 1 << 40
    ws = FAKE * 1024

    def lay(**kw):
        a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, z=FAKE * 4, A=FAKE * 5, bl=FAKE * 6, og=None, nw=None,
                 qe=1e-6, ne=1e-6, s0=None, cu=None, n=1, T=T, H=H, dk=128, dv=128, dt=BF16,
                 o=FAKE * 16, fs=None, ws=ws, wsb=big)
        a.update(kw)
        return L.kda_layer_prefill(a["q"], a["k"], a["v"], a["z"], a["A"], a["bl"], a["og"], a["nw"],
                                   a["qe"], a["ne"], a["s0"], a["cu"], a["n"], a["T"], a["H"], a["dk"],
                                   a["dv"], a["dt"], a["o"], a["fs"], a["ws"], a["wsb"], None)
    assert lay(n=0) == 1
    assert lay(dt=FP32) == 2                     # the layer has no fp32 path
    assert lay(dk=64, dv=64) == 2
    assert lay(A=None) == 1
    assert lay(A=FAKE * 5 + 2) == 1              # A_log not 4-byte aligned
    assert lay(nw=FAKE * 7 + 1) == 1
    assert lay(og=FAKE * 8 + 8) == 1             # out_gate not 16-byte aligned
    assert lay(og=FAKE * 16 + 4096) == 1         # out_gate under o
    assert lay(qe=-1.0) == 1
    assert lay(ne=float("nan")) == 1
    assert lay(wsb=1024) == 3
    assert lay(ws=ws + 128) == 1                 # workspace not 256-aligned


def test_noalloc_refuses_more_sequences_than_its_array_holds(L):
    """kda_prefill_noalloc keeps its scratch in a fixed array sized for
    KDA_NOALLOC_MAX_SEQS sequences; more is refused before any CUDA call."""
    text = open(os.path.join(ROOT, "include", "kda.h")).read()
    cap = int(re.search(r"#define KDA_NOALLOC_MAX_SEQS (\d+)", text).group(1))
    st = L.kda_prefill_noalloc(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5, None, FAKE * 6,
                               cap + 1, 64 * (cap + 1), 1, 128, 128, BF16, FAKE * 16, None, None)
    assert st == 2


def test_layer_decode_rejects_on_host(L):
    """kda_layer_decode_step: kda_decode_step's checks plus the layer's own
    (A_log required and 4-byte aligned, eps >= 0, the output gate aligned and
    not under o)."""
    def lay(**kw):
        a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, z=FAKE * 4, A=FAKE * 5, bl=FAKE * 6, og=None, nw=None,
                 qe=1e-6, ne=1e-6, s=FAKE * 16, B=4, H=2, dk=16, dv=16, dt=FP32, o=FAKE * 64)
        a.update(kw)
        return L.kda_layer_decode_step(a["q"], a["k"], a["v"], a["z"], a["A"], a["bl"], a["og"], a["nw"],
                                       a["qe"], a["ne"], a["s"], a["B"], a["H"], a["dk"], a["dv"],
                                       a["dt"], a["o"], None)
    assert lay(B=0) == 0                         # empty batch: no-op
    assert lay(B=-1) == 1
    assert lay(dk=48) == 2
    assert lay(A=None) == 1
    assert lay(A=FAKE * 5 + 2) == 1
    assert lay(nw=FAKE * 7 + 2) == 1
    assert lay(og=FAKE * 8 + 2) == 1             # fp32 gate not 4-byte aligned
    assert lay(og=FAKE * 64 + 64) == 1           # out_gate under o
    assert lay(qe=-0.5) == 1
    assert lay(ne=float("nan")) == 1
    assert lay(s=FAKE * 16 + 8) == 1             # state not 16-byte aligned


def test_binding_checks_chunked_backward_gate_shape():
    import torch
    from gated_delta_rule_69_b200 import kda
    x = torch.zeros(4, 2, 128, dtype=torch.bfloat16)
    b = torch.zeros(4, 2, dtype=torch.bfloat16)
    with pytest.raises(ValueError):   # per-head gate given to the per-channel entry
        kda.kda_backward_chunked(x, x, x, b, b, x)
    with pytest.raises(ValueError):   # per-channel gate given to the Gated DeltaNet entry
        kda.gdn_backward_chunked(x, x, x, x, b, x)
