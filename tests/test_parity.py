"""GPU parity: libcattn (through its C ABI) against the fp64 oracle on the
same seeded bf16 inputs, for the five workloads and for ragged/edge shapes.

The oracle always receives the bf16-rounded inputs the GPU receives, so the
difference measured is the kernels' own error.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import check_bf16, check_bf16_beyond_rounding, check_lse, errors
from workloads import (WORKLOADS, as_f64, bf16_inputs, draw_extra,
                       sample_heads, seed_for, workload_inputs)

pytestmark = pytest.mark.gpu


def run_gpu(lib, q, k, v, do, scale, residual=True):
    """Forward + backward through the C ABI.  residual=True uses the
    extended calls (the forward's O_lo feeds the backward's Delta);
    residual=False the plain attn_fwd / attn_bwd."""
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    if residual:
        o, lse, o_lo = lib.attn_fwd_ex(qd, kd, vd, scale)
        dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, lse, dod, scale, o_lo=o_lo)
    else:
        o, lse = lib.attn_fwd(qd, kd, vd, scale)
        dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, lse, dod, scale)
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    return {n: as_f64(t) for n, t in
            (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}


def full_oracle(q, k, v, do, scale):
    qn, kn, vn, don = (as_f64(t) for t in (q, k, v, do))
    o, lse = oracle.attention_forward(qn, kn, vn, scale)
    dq, dk, dv = oracle.attention_backward(qn, kn, vn, don, scale)
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def check_all(got, ref, report=None):
    for n in ("o", "dq", "dk", "dv"):
        ma, rl = check_bf16(n, got[n], ref[n])
        if report is not None:
            report[n] = (ma, rl)
    ma = check_lse(got["lse"], ref["lse"])
    if report is not None:
        report["lse"] = ma


@pytest.mark.parametrize("index", [0, 1, 2, 3])
def test_workload_full_oracle(lib, index):
    w = WORKLOADS[index]
    q, k, v, do = workload_inputs(index)
    got = run_gpu(lib, q, k, v, do, w.scale)
    ref = full_oracle(q, k, v, do, w.scale)
    rep = {}
    check_all(got, ref, rep)
    print(w.name, rep)


@pytest.mark.parametrize("index", [0, 1, 2, 3])
def test_workload_plain_entry_points(lib, index):
    """attn_fwd / attn_bwd without the residual: Delta from the bf16 O."""
    w = WORKLOADS[index]
    q, k, v, do = workload_inputs(index)
    got = run_gpu(lib, q, k, v, do, w.scale, residual=False)
    ref = full_oracle(q, k, v, do, w.scale)
    rep = {}
    check_all(got, ref, rep)
    print(w.name, "plain", rep)


def bf16_floor(ref):
    """max |bf16(ref) - ref|: the error of a perfect kernel with bf16 output."""
    return float(np.abs(as_f64(torch.tensor(ref).to(torch.bfloat16)) - ref).max())


def test_long_context_sampled_heads(lib):
    """T = 8192, D = 128, logit std 4: two whole heads through the full
    oracle (fwd + bwd), plus single rows of O/LSE on eight more heads.

    On these heads |dQ| and |dK| exceed 8, where bf16's own rounding (half
    an ulp, up to 0.031) is above the 2e-2 max-abs bar.  So: the bf16
    gradients are held to 2e-2 beyond their own rounding (the stated
    figures are printed as they are), and the same call with fp32 gradient
    outputs is held to the stated 2e-2 / 1e-2 exactly."""
    index = 4
    w = WORKLOADS[index]
    q, k, v, do = workload_inputs(index)
    heads = sample_heads(w.BH, 2, seed=seed_for(index))
    qn, kn, vn, don = (as_f64(t) for t in (q, k, v, do))
    ro, rl = oracle.attention_forward_heads(qn, kn, vn, w.scale, heads)
    rq, rk, rv = oracle.attention_backward_heads(qn, kn, vn, don, w.scale, heads)
    refs = (("o", ro), ("dq", rq), ("dk", rk), ("dv", rv))

    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse, o_lo = lib.attn_fwd_ex(qd, kd, vd, w.scale)
    bf = lib.attn_bwd(qd, kd, vd, o, lse, dod, w.scale, o_lo=o_lo)
    f32 = lib.attn_bwd(qd, kd, vd, o, lse, dod, w.scale, o_lo=o_lo, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    got_bf = dict(o=as_f64(o), dq=as_f64(bf[0]), dk=as_f64(bf[1]), dv=as_f64(bf[2]))
    got_32 = dict(dq=as_f64(f32[0]), dk=as_f64(f32[1]), dv=as_f64(f32[2]))

    def head_view(x):
        return x.reshape(w.BH, w.T, -1)[heads]

    check_bf16("o", head_view(got_bf["o"]), ro)
    check_lse(as_f64(lse).reshape(w.BH, w.T)[heads], rl)
    for n, ref in refs[1:]:
        stated = errors(head_view(got_bf[n]), ref)
        print(f"{w.name} {n} bf16: max-abs {stated[0]:.4f} rel-L2 {stated[1]:.2e} "
              f"(bf16 floor {bf16_floor(ref):.4f})")
        check_bf16_beyond_rounding(n, head_view(got_bf[n]), ref)
        ma, rl2 = check_bf16(n + " fp32", head_view(got_32[n]), ref)
        print(f"{w.name} {n} fp32: max-abs {ma:.2e} rel-L2 {rl2:.2e}")
    # The plain entry points (attn_fwd / attn_bwd, the pages' signatures) on
    # the same heads.  attn_bwd receives O in bf16, and its row term Delta
    # carries that rounding: even the exact gradient given bf16(O) misses
    # the exact one by more than 2e-2 beyond rounding here (`forced`, from
    # the oracle alone).  So:
    # (a) attn_fwd's O and LSE: the stated tolerance;
    # (b) attn_bwd's own error: fed the oracle's bf16 O and LSE on the
    #     sampled heads (heads are independent), against the exact gradient
    #     given that O, at the stated 2e-2 beyond bf16 rounding;
    # (c) attn_fwd then attn_bwd, end to end, against the exact gradient, at
    #     2e-2 beyond rounding plus `forced`.
    plain = run_gpu(lib, q, k, v, do, w.scale, residual=False)
    check_bf16("o plain", head_view(plain["o"]), ro)
    check_lse(plain["lse"].reshape(w.BH, w.T)[heads], rl)
    ro_bf16 = as_f64(torch.tensor(ro).to(torch.bfloat16))
    given = oracle.attention_backward_given_o(qn, kn, vn, don, ro_bf16, w.scale, heads)
    o_in, lse_in = lib.attn_fwd(qd, kd, vd, w.scale)
    torch.cuda.synchronize()
    o_view = o_in.view(w.BH, w.T, w.D)
    lse_view = lse_in.view(w.BH, w.T)
    for n_, f in enumerate(heads):
        o_view[f] = torch.tensor(ro[n_]).to(torch.bfloat16).to(dev)
        lse_view[f] = torch.tensor(rl[n_], dtype=torch.float32).to(dev)
    fed = lib.attn_bwd(qd, kd, vd, o_in, lse_in, dod, w.scale)
    torch.cuda.synchronize()
    assert lib.cattn_get_device_status() == lib.OK
    for (n, ref), ref_given, g_fed in zip(refs[1:], given, fed):
        forced = float((np.abs(as_f64(torch.tensor(ref_given).to(torch.bfloat16)) - ref)
                        - 2.0 ** -8 * np.abs(ref)).max())
        excess_b, _ = check_bf16_beyond_rounding(n + " plain bwd vs exact given bf16 O",
                                                 head_view(as_f64(g_fed)), ref_given)
        got = head_view(plain[n])
        excess, _ = check_bf16_beyond_rounding(n + " plain fwd+bwd vs exact", got, ref,
                                               max_abs=2e-2 + max(forced, 0.0))
        stated = errors(got, ref)
        print(f"{w.name} {n} plain: max-abs {stated[0]:.4f} rel-L2 {stated[1]:.2e}; beyond "
              f"bf16 rounding: fwd+bwd {excess:.4f} vs exact (the bf16 O alone forces "
              f"{forced:.4f}), bwd {excess_b:.4f} vs exact given bf16 O")
    rows = [0, 1, 127, 128, 4095, 8191]
    for f in sample_heads(w.BH, 8, seed=seed_for(index) + 1):
        b, h = divmod(f, w.H)
        o_rows, lse_rows = oracle.attention_rows(qn, kn, vn, w.scale, b, h, rows)
        check_bf16("o rows", got_bf["o"][b, h, rows], o_rows)
        check_lse(as_f64(lse)[b, h, rows], lse_rows)


@pytest.mark.parametrize("index", [1, 2, 3])
def test_workload_fp32_gradients(lib, index):
    """The fp32-gradient option on the GPT-shaped workloads: stated
    tolerance with no output rounding."""
    w = WORKLOADS[index]
    q, k, v, do = workload_inputs(index)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse, o_lo = lib.attn_fwd_ex(qd, kd, vd, w.scale)
    dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, lse, dod, w.scale, o_lo=o_lo,
                              grad_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = full_oracle(q, k, v, do, w.scale)
    for n, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        ma, rl = check_bf16(n + " fp32", as_f64(g), ref[n])
        print(w.name, n, "fp32", ma, rl)


RAGGED_T = [1, 17, 63, 64, 65, 127, 128, 129, 255, 1000]


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("T", RAGGED_T)
def test_ragged_lengths(lib, T, D):
    B, H = 2, 1
    q, k, v, do = bf16_inputs(B, H, T, D, seed=7000 + 10 * T + D)
    scale = 1.0 / math.sqrt(D)
    check_all(run_gpu(lib, q, k, v, do, scale), full_oracle(q, k, v, do, scale))


@pytest.mark.parametrize("scale", [0.02, 0.25, 0.5])
def test_other_scales_and_peaked_logits(lib, scale):
    """q, k with std 2: logits with std 0.64 .. 16.  At the larger scales
    |dQ|, |dK| reach 12..24, where bf16's half-ulp alone is 0.03..0.06, so
    the bf16 outputs are bounded beyond that rounding; the same gradients
    as fp32 outputs (residual forward, no final rounding) are held to the
    stated 2e-2 / 1e-2 exactly."""
    B, H, T, D = 1, 3, 300, 64
    q, k, v, do = bf16_inputs(B, H, T, D, seed=91, qk_std=2.0)
    got = run_gpu(lib, q, k, v, do, scale)
    ref = full_oracle(q, k, v, do, scale)
    for n in ("o", "dq", "dk", "dv"):
        check_bf16_beyond_rounding(n, got[n], ref[n])
    check_lse(got["lse"], ref["lse"])
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse, o_lo = lib.attn_fwd_ex(qd, kd, vd, scale)
    f32 = lib.attn_bwd(qd, kd, vd, o, lse, dod, scale, o_lo=o_lo, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    for n, g in zip(("dq", "dk", "dv"), f32):
        check_bf16(n + " fp32", as_f64(g), ref[n])


def test_preprocess_delta(lib):
    """The Delta step on its own: synthetic O and dO (independent draws)."""
    B, H, T, D = 3, 4, 333, 64
    o = draw_extra((B, H, T, D), seed=501)
    do = draw_extra((B, H, T, D), seed=502)
    delta = lib.attn_bwd_preprocess(o.cuda(), do.cuda())
    torch.cuda.synchronize()
    ref = oracle.delta_from_o(as_f64(o), as_f64(do))
    err = np.abs(as_f64(delta) - ref).max()
    assert err <= 1e-4 * max(1.0, np.abs(ref).max()), err
    for D2 in (16, 32, 128):
        o2 = draw_extra((1, 2, 77, D2), seed=503 + D2)
        do2 = draw_extra((1, 2, 77, D2), seed=504 + D2)
        d2 = lib.attn_bwd_preprocess(o2.cuda(), do2.cuda())
        ref2 = oracle.delta_from_o(as_f64(o2), as_f64(do2))
        assert np.abs(as_f64(d2) - ref2).max() <= 1e-4 * max(1.0, np.abs(ref2).max())


def test_outputs_stay_in_bounds(lib):
    """Canary-padded outputs: every byte outside the tensors is untouched,
    and a NaN-poisoned workspace does not leak into the results."""
    B, H, T, D = 2, 3, 200, 64
    q, k, v, do = bf16_inputs(B, H, T, D, seed=333)
    scale = 1.0 / math.sqrt(D)
    dev = torch.device("cuda:0")
    n = B * H * T * D
    pad = 4096
    sentinel = torch.tensor(1234.0, dtype=torch.bfloat16)

    def padded(numel, dtype):
        buf = torch.full((numel + 2 * pad,), float(sentinel) if dtype == torch.bfloat16
                         else -777.0, dtype=dtype, device=dev)
        return buf, buf[pad:pad + numel]

    ob, o = padded(n, torch.bfloat16)
    lb, lse = padded(B * H * T, torch.float32)
    outs = [padded(n, torch.bfloat16) for _ in range(3)]
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    lib.attn_fwd(qd, kd, vd, scale, o=o.view(B, H, T, D), lse=lse.view(B, H, T))
    wsn = lib.attn_bwd_workspace_bytes(B, H, T, D)
    ws = torch.full((wsn,), 0xFF, dtype=torch.uint8, device=dev)   # NaN floats
    lib.attn_bwd(qd, kd, vd, o.view(B, H, T, D), lse.view(B, H, T), dod, scale,
                 dq=outs[0][1].view(B, H, T, D), dk=outs[1][1].view(B, H, T, D),
                 dv=outs[2][1].view(B, H, T, D), workspace=ws)
    torch.cuda.synchronize()
    for buf in [ob] + [b for b, _ in outs]:
        assert (buf[:pad] == sentinel).all() and (buf[-pad:] == sentinel).all()
    assert (lb[:pad] == -777.0).all() and (lb[-pad:] == -777.0).all()
    got = dict(o=as_f64(o.view(B, H, T, D)), lse=as_f64(lse.view(B, H, T)),
               dq=as_f64(outs[0][1].view(B, H, T, D)), dk=as_f64(outs[1][1].view(B, H, T, D)),
               dv=as_f64(outs[2][1].view(B, H, T, D)))
    check_all(got, full_oracle(q, k, v, do, scale))


def test_forward_is_deterministic(lib):
    q, k, v, _ = (t.cuda() for t in bf16_inputs(2, 4, 700, 64, seed=44))
    o1, l1 = lib.attn_fwd(q, k, v)
    o2, l2 = lib.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_empty_sequence(lib):
    q = torch.empty(2, 3, 0, 64, dtype=torch.bfloat16, device="cuda")
    o, lse = lib.attn_fwd(q, q, q)
    dq, dk, dv = lib.attn_bwd(q, q, q, o, lse, q)
    assert o.shape == (2, 3, 0, 64) and dq.shape == (2, 3, 0, 64)


def test_autograd_wrapper(lib):
    B, H, T, D = 1, 2, 150, 64
    q, k, v, do = bf16_inputs(B, H, T, D, seed=12)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    out = lib.CausalAttention.apply(qd, kd, vd, None)
    out.backward(do.cuda())
    ref = full_oracle(q, k, v, do, 1.0 / math.sqrt(D))
    check_bf16("o", as_f64(out), ref["o"])
    check_bf16("dq", as_f64(qd.grad), ref["dq"])
    check_bf16("dk", as_f64(kd.grad), ref["dk"])
    check_bf16("dv", as_f64(vd.grad), ref["dv"])


def test_hang_guard_times_out_cleanly(lib):
    """A wait on a barrier nothing arrives on gives up after its limit,
    records CATTN_ERR_TIMEOUT, and leaves the context usable."""
    st = lib.cattn_selftest_wait_timeout(2000)
    assert st == lib.ERR_TIMEOUT
    assert lib.cattn_get_device_status() == lib.OK   # the self-test cleared it
    q, k, v, do = bf16_inputs(1, 2, 130, 64, seed=5)
    got = run_gpu(lib, q, k, v, do, 0.125)
    check_all(got, full_oracle(q, k, v, do, 0.125))


def test_status_words_are_per_workspace(lib):
    """A wait that runs out is recorded in the status words of the
    workspace of the call it belongs to, on that call's stream, and not in
    another workspace used meanwhile on another stream; a backward call
    that reuses the workspace starts its record afresh."""
    B, H, T, D = 1, 2, 130, 64
    wsn = lib.attn_bwd_workspace_bytes(B, H, T, D)
    ws_a = torch.zeros(wsn, dtype=torch.uint8, device="cuda")
    ws_b = torch.zeros(wsn, dtype=torch.uint8, device="cuda")
    q, k, v, do = (t.cuda() for t in bf16_inputs(B, H, T, D, seed=6))
    o, lse = lib.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    # stream A: a wait that nothing ends, limit 2 ms, recorded in ws_a
    assert lib.cattn_selftest_wait_timeout(2000, stream=sa, workspace=ws_a) == lib.ERR_TIMEOUT
    # stream B: an ordinary backward with ws_b
    with torch.cuda.stream(sb):
        dq, dk, dv = lib.attn_bwd(q, k, v, o, lse, do, workspace=ws_b, stream=sb)
    assert lib.cattn_last_device_status(ws_b, stream=sb) == lib.OK
    assert lib.cattn_last_device_status(ws_a, stream=sa) == lib.ERR_TIMEOUT
    assert lib.cattn_get_device_status() == lib.OK   # the self-test left the global word clear
    check_bf16("dq", as_f64(dq), full_oracle(q.cpu(), k.cpu(), v.cpu(), do.cpu(), 0.125)["dq"])
    # the next backward on ws_a clears the record before it runs
    torch.cuda.synchronize()
    with torch.cuda.stream(sa):
        lib.attn_bwd(q, k, v, o, lse, do, workspace=ws_a, stream=sa)
    assert lib.cattn_last_device_status(ws_a, stream=sa) == lib.OK


def test_errors_reported_on_device(lib):
    q = torch.zeros(1, 1, 8, 48, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.CattnError) as e:
        lib.attn_fwd(q, q, q)
    assert e.value.status == lib.ERR_UNSUPPORTED
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    o, lse = lib.attn_fwd(q, q, q)
    with pytest.raises(lib.CattnError):
        lib.attn_bwd(q, q, q, o, lse, q,
                     workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert errors(as_f64(o), np.zeros((1, 1, 8, 64)))[0] == 0.0


def test_many_items_alternating_passes(lib):
    """9,600 forward work items (B*H = 9,600 heads of one query-tile pair):
    more passes over 148 CTAs than the planned codes cover, so the forward
    deals them in plain alternating passes.  Every head is computed; a
    seeded sample of them is checked against the oracle."""
    B, H, T, D = 150, 64, 130, 16
    assert lib.LIB.cattn_plan_passes(0, B * H, (T + 127) // 128, 148, None, 0) == 0
    q, k, v, do = bf16_inputs(B, H, T, D, seed=9100)
    scale = 1.0 / math.sqrt(D)
    got = run_gpu(lib, q, k, v, do, scale, residual=False)
    rng = np.random.default_rng(9101)
    for b, h in zip(rng.integers(0, B, 12), rng.integers(0, H, 12)):
        sl = (slice(int(b), int(b) + 1), slice(int(h), int(h) + 1))
        ref = full_oracle(q[sl], k[sl], v[sl], do[sl], scale)
        part = {n: got[n][sl] for n in got}
        for n in ("o", "dq", "dk", "dv"):
            check_bf16(n, part[n], ref[n])
        check_lse(part["lse"], ref["lse"])
