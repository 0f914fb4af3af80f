"""The operator with the layer prologue / epilogue fused in (kda_layer_prefill,
kda_layer_decode_step) against the fp64 oracle's prologue -> recurrence ->
epilogue, through the C ABI.

Error measure for o.  The epilogue rescales every output row to unit RMS, so
a row whose o is small (q nearly orthogonal to what the state holds) has its
bf16-level error scaled up with it, and the plain operator's measure (worst
|error| over the (sequence, head) slice's largest |o|) would be applied to a
different quantity.  The tests take the kernel's output back to the scale of
o with the oracle's own per-row factor (o = y * rms_ref / (w sigmoid(g))) and
apply the plain measure and tolerance to that; a wrong normalisation factor,
weight or gate shows up there as it would in y.  Beside it, y itself is
checked element by element against a bound derived from that tolerance
(``y_within_bound``).  The final state is compared directly."""
import numpy as np
import pytest
import torch

from gated_delta_rule_69_b200 import inputs as kin
from parity_util import TOL, o_err, state_err

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


def kda():
    from gated_delta_rule_69_b200 import kda as k
    return k


def f64(t):
    return None if t is None else t.detach().cpu().double().numpy()


def layer_case(T, H, dk, dv, dtype="bf16", seed=0, lengths=None, init_std=0.02, A_mean=0.0,
               z_mean=-1.0, gates=True):
    """Raw activations: q, k ~ N(0, 2^2) (not normalised), gate pre-activation
    z ~ N(z_mean, 1), A_log ~ N(A_mean, 0.25^2) per head, beta logits and
    output-gate pre-activations ~ N(0, 1), RMSNorm weight ~ 1 + N(0, 0.1^2)."""
    w = kin.Workload("layer", "prefill", H=H, d_k=dk, d_v=dv, dtype=dtype, seed=seed, T=T,
                     init_std=init_std)
    inp = kin.generate(w, device=DEV, lengths=lengths)
    g = torch.Generator(device="cpu").manual_seed(seed + 7)
    io = inp["q"].dtype
    Tt = inp["q"].shape[0]
    inp["q"] = (torch.randn(Tt, H, dk, generator=g) * 2.0).to(io).to(DEV)
    inp["k"] = (torch.randn(Tt, H, dk, generator=g) * 2.0).to(io).to(DEV)
    inp["gate_z"] = (torch.randn(Tt, H, dk, generator=g) + z_mean).to(io).to(DEV)
    inp["A_log"] = (torch.randn(H, generator=g) * 0.25 + A_mean).float().to(DEV)
    inp["beta_logit"] = torch.randn(Tt, H, generator=g).to(io).to(DEV)
    inp["out_gate"] = torch.randn(Tt, H, dv, generator=g).to(io).to(DEV) if gates else None
    inp["norm_weight"] = (1.0 + 0.1 * torch.randn(dv, generator=g)).float().to(DEV) if gates else None
    return inp


def oracle_layer(inp, qk_eps=1e-6, norm_eps=1e-6):
    """Returns (o before the epilogue, final state, cu, to_o): to_o maps an
    output y of the fused op back to o's scale with the oracle's factors."""
    import oracle
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    o_pre, fs = oracle.kda_recurrence(
        oracle.l2_normalize(f64(inp["q"]), qk_eps), oracle.l2_normalize(f64(inp["k"]), qk_eps),
        f64(inp["v"]), oracle.kimi_log_alpha(f64(inp["gate_z"]), f64(inp["A_log"])),
        oracle.sigmoid(f64(inp["beta_logit"])), f64(inp["init_state"]), cu)
    y_ref = oracle.rms_norm_gate(o_pre, f64(inp["out_gate"]), f64(inp["norm_weight"]), norm_eps)
    # y = o * factor per element (factor = w sigmoid(g) / rms): o = y / factor
    factor = y_ref / np.where(o_pre == 0.0, 1.0, o_pre)
    factor = np.where(o_pre == 0.0, 1.0, factor)

    def to_o(y):
        return y / factor
    return o_pre, fs, cu, to_o


def y_within_bound(y, inp, tol, norm_eps=1e-6):
    """The fused op's output y checked directly, row by row, against a bound
    derived from the plain operator's tolerance.

    Per (sequence, head) slice let S = max |o_ref| (o before the epilogue).
    The operator's tolerance allows |do_j| <= tol S on every element.  With
    r = rms(o_ref row) (eps included) and y_j = c_j o_j / r, c_j = w_j
    sigmoid(g_j): the row's rms moves by at most max |do| (rms is 1-Lipschitz
    in the max norm), so |dy_j| <= |c_j| tol S (1 + |o_ref_j| / r) / (r - tol S)
    for r > tol S, plus the rounding of y itself to its dtype (2^-8 |y_j| in
    bf16, 2^-23 |y_j| in fp32).  A row
    whose rms is within 2 tol S of zero carries only the operator's noise,
    which the epilogue scales up to unit rms: such rows are left out and
    counted (about 8 % of the rows of the layer cases below; the
    rescaled-o measure still covers them).  Returns (worst ratio of error to bound, rows left out, rows)."""
    import oracle
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    o_pre, _ = oracle.kda_recurrence(
        oracle.l2_normalize(f64(inp["q"]), 1e-6), oracle.l2_normalize(f64(inp["k"]), 1e-6),
        f64(inp["v"]), oracle.kimi_log_alpha(f64(inp["gate_z"]), f64(inp["A_log"])),
        oracle.sigmoid(f64(inp["beta_logit"])), f64(inp["init_state"]), cu)
    y_ref = oracle.rms_norm_gate(o_pre, f64(inp["out_gate"]), f64(inp["norm_weight"]), norm_eps)
    c = np.ones_like(o_pre)
    if inp["norm_weight"] is not None:
        c = c * f64(inp["norm_weight"])
    if inp["out_gate"] is not None:
        c = c * oracle.sigmoid(f64(inp["out_gate"]))
    yk = f64(y)
    rnd = 2.0 ** -8 if y.dtype == torch.bfloat16 else 2.0 ** -23
    H = o_pre.shape[1]
    worst, skipped, rows = 0.0, 0, 0
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        for h in range(H):
            o_s = o_pre[a:b, h]
            if o_s.size == 0:
                continue
            S = np.max(np.abs(o_s))
            r = np.sqrt(np.mean(o_s * o_s, axis=-1) + norm_eps)
            keep = r > 2.0 * tol * S
            skipped += int((~keep).sum())
            rows += r.size
            if not keep.any():
                continue
            rk = r[keep][:, None]
            bound = (np.abs(c[a:b, h][keep]) * tol * S * (1.0 + np.abs(o_s[keep]) / rk) / (rk - tol * S)
                     + rnd * np.abs(y_ref[a:b, h][keep]))
            err = np.abs(yk[a:b, h][keep] - y_ref[a:b, h][keep])
            if not np.all(np.isfinite(err)):
                return float("inf"), skipped, rows
            worst = max(worst, float(np.max(err / bound)))
    return worst, skipped, rows


def run_layer(inp, workspace=None):
    T, H, _ = inp["q"].shape
    dv = inp["v"].shape[-1]
    n = inp["cu_seqlens"].numel() - 1
    o = torch.full((T, H, dv), float("nan"), dtype=inp["q"].dtype, device=DEV)
    o, fs = kda().kda_layer_prefill(inp["q"], inp["k"], inp["v"], inp["gate_z"], inp["A_log"],
                                    inp["beta_logit"], out_gate=inp["out_gate"],
                                    norm_weight=inp["norm_weight"], init_state=inp["init_state"],
                                    cu_seqlens=inp["cu_seqlens"], num_seqs=n, o=o,
                                    workspace=workspace)
    torch.cuda.synchronize()
    return o, fs


@pytest.mark.parametrize("lengths,gates", [(None, True), ([1, 64, 130, 200, 63], True),
                                           ([100, 37], False)])
def test_layer_prefill(lengths, gates):
    T = 300 if lengths is None else sum(lengths)
    inp = layer_case(T, 3, 128, 128, seed=31, lengths=lengths, gates=gates)
    o, fs = run_layer(inp)
    ref_o, ref_s, cu, to_o = oracle_layer(inp)
    assert o_err(to_o(f64(o)), ref_o, cu, 3) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]
    ratio, skipped, rows = y_within_bound(o, inp, TOL["bf16"])
    assert ratio <= 1.0, ratio
    assert skipped <= rows // 5, (skipped, rows)


@pytest.mark.parametrize("A_mean", [0.0, 2.6])
def test_layer_prefill_prologue_inside_the_preparation(A_mean):
    """A workspace of kda_prefill_workspace_size bytes (no room for the
    prologue's outputs): the prologue runs inside the chunk preparation."""
    lengths = [1, 64, 130, 200, 63]
    inp = layer_case(sum(lengths), 3, 128, 128, seed=36, lengths=lengths, A_mean=A_mean)
    n = len(lengths)
    T, H = inp["q"].shape[:2]
    need = kda().kda_prefill_workspace_size(n, T, H, 128, 128)
    assert kda().kda_layer_prefill_workspace_size(n, T, H, 128, 128) > need
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    o, fs = run_layer(inp, workspace=ws)
    ref_o, ref_s, cu, to_o = oracle_layer(inp)
    assert o_err(to_o(f64(o)), ref_o, cu, 3) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]
    ratio, skipped, rows = y_within_bound(o, inp, TOL["bf16"])
    assert ratio <= 1.0, ratio


@pytest.mark.parametrize("A_mean", [1.3, 2.6])
def test_layer_prefill_fast_decay(A_mean):
    """e^A softplus(z) near 2.5 and 10 per token: chunks that take the
    one-reference-per-16-token-block path and the pairwise path, both with
    the normalisation factors applied to the raw rows they reload."""
    inp = layer_case(256, 2, 128, 128, seed=32, A_mean=A_mean, z_mean=0.5)
    o, fs = run_layer(inp)
    ref_o, ref_s, cu, to_o = oracle_layer(inp)
    assert o_err(to_o(f64(o)), ref_o, cu, 2) <= TOL["bf16"]
    assert state_err(f64(fs), ref_s) <= TOL["bf16"]


def test_layer_prefill_rejects_other_paths():
    k = kda()
    inp = layer_case(64, 1, 64, 64, dtype="fp32", seed=33)
    with pytest.raises(k.KdaError):
        run_layer(inp)
    inp = layer_case(64, 1, 128, 128, seed=34)
    small = torch.empty(512, dtype=torch.uint8, device=DEV)
    with pytest.raises(k.KdaError):
        run_layer(inp, workspace=small)


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, "bf16"), (16, 32, "fp32"), (64, 64, "fp32")])
def test_layer_decode_step(dk, dv, dtype):
    B, H = 5, 3
    inp = layer_case(B, H, dk, dv, dtype=dtype, seed=35 + dk, lengths=[1] * B)
    state = inp["init_state"].clone()
    o = torch.full((B, H, dv), float("nan"), dtype=inp["q"].dtype, device=DEV)
    kda().kda_layer_decode_step(inp["q"], inp["k"], inp["v"], inp["gate_z"], inp["A_log"],
                                inp["beta_logit"], state, out_gate=inp["out_gate"],
                                norm_weight=inp["norm_weight"], o=o)
    torch.cuda.synchronize()
    ref_o, ref_s, cu, to_o = oracle_layer(inp)
    tol = TOL[dtype]
    assert o_err(to_o(f64(o)), ref_o, cu, H) <= tol
    assert state_err(f64(state), ref_s) <= tol
    ratio, skipped, rows = y_within_bound(o, inp, tol)
    assert ratio <= 1.0, ratio
    assert skipped == 0, (skipped, rows)


def test_layer_prefill_then_decode():
    T1, T2, H = 130, 3, 2
    inp = layer_case(T1 + T2, H, 128, 128, seed=36)
    ref_o, ref_s, cu, to_o = oracle_layer(inp)
    k = kda()
    sl = slice(0, T1)
    o1, st = k.kda_layer_prefill(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["gate_z"][sl],
                                 inp["A_log"], inp["beta_logit"][sl], out_gate=inp["out_gate"][sl],
                                 norm_weight=inp["norm_weight"], init_state=inp["init_state"])
    outs = [o1]
    for t in range(T1, T1 + T2):
        s1 = slice(t, t + 1)
        outs.append(k.kda_layer_decode_step(inp["q"][s1], inp["k"][s1], inp["v"][s1],
                                            inp["gate_z"][s1], inp["A_log"], inp["beta_logit"][s1],
                                            st, out_gate=inp["out_gate"][s1],
                                            norm_weight=inp["norm_weight"]))
    torch.cuda.synchronize()
    o = torch.cat(outs)
    assert o_err(to_o(f64(o)), ref_o, cu, H) <= TOL["bf16"]
    assert state_err(f64(st), ref_s) <= TOL["bf16"]
