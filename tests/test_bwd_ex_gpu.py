"""Parity of the backward pass with the fused extras (m3_scan_bwd_ex: output gate, BCNorm and
BC biases, MIMO lightweight expansion) with the fp64 oracle's scan_bwd_ex, through the C ABI,
on the same rounded inputs.

The GPU forms the effective inputs in the io dtype (as the fused forward kernels use them),
reruns the ungated forward for the gate's derivative, runs the recurrence backward (the
chunked tensor-core one for bf16 P 64 with SISO N 64 / 128 or MIMO R 2 / 4 N 64, the sequential
fp32 one otherwise) and maps the gradients back.  Bars: 2e-2 of each gradient's largest value
for bf16 inputs, 2e-4 for fp32.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import KEYS, f64
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu

EPS = 1e-5


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


CASES = [
    # (b, H, G, P, N, R, T, io, gate, bias, eps, x_exp, tol)   gate: None | "plain" | "exp"
    (1, 4, 1, 64, 128, 1, 100, torch.bfloat16, "plain", False, 0.0, False, 2e-2),
    (1, 4, 1, 64, 128, 1, 130, torch.bfloat16, None, True, EPS, False, 2e-2),
    (1, 4, 2, 64, 128, 1, 90, torch.bfloat16, "exp", True, EPS, True, 2e-2),
    (1, 4, 1, 64, 64, 4, 70, torch.bfloat16, "exp", True, EPS, True, 2e-2),
    (1, 4, 2, 64, 64, 2, 90, torch.bfloat16, "plain", True, EPS, False, 2e-2),
    (1, 4, 2, 8, 6, 2, 40, torch.float32, "exp", True, EPS, True, 2e-4),
    (2, 2, 1, 16, 16, 1, 33, torch.float32, "plain", True, 0.0, False, 2e-4),
]


def _id(c):
    return (f"b{c[0]}H{c[1]}G{c[2]}P{c[3]}N{c[4]}R{c[5]}T{c[6]}"
            f"{'f32' if c[7] == torch.float32 else 'bf16'}-{c[8] or 'nogate'}"
            f"{'-bias' if c[9] else ''}{'-norm' if c[10] else ''}{'-xexp' if c[11] else ''}")


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_bwd_ex_matches_oracle(case):
    b, H, G, P, N, R, T, io, gate, bias, eps, x_exp, tol = case
    seed = 71
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=io, theta_max=1.0, seed=seed,
                                  h0_random=True, carry_prev=True)
    wx, wz = inputs.make_expand(H, R, P, seed=seed)
    bb, cb = inputs.make_bc_bias(H, N, seed=seed)
    x = inp["x"][:, :, :, 0, :].contiguous() if x_exp else inp["x"]
    z = None
    if gate == "plain":
        z = inputs.make_gate((b, T, H, R, P), io_dtype=io, seed=seed)
    elif gate == "exp":
        z = inputs.make_gate((b, T, H, P), io_dtype=io, seed=seed)
    gen = torch.Generator().manual_seed(seed + 5)
    dy = torch.randn((b, T, H, R, P), generator=gen).to(io)
    dh = torch.randn((b, H, N, P), generator=gen)

    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    g = {k: v.cuda() for k, v in inp.items()}
    ex = m3.Extras(z=None if z is None else z.cuda(),
                   B_bias=bb.cuda() if bias else None, C_bias=cb.cuda() if bias else None,
                   bc_norm_eps=eps, x_expand=wx.cuda() if x_exp else None,
                   z_expand=wz.cuda() if gate == "exp" else None)
    st = m3.State(d)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    gr = m3.alloc_grads(d, T)
    if x_exp:
        gr["dx"] = torch.empty((b, T, H, P), dtype=torch.float32, device="cuda")
    xg = m3.alloc_extra_grads(d, T, ex)
    for v in list(gr.values()) + list(xg.values()):
        v.fill_(float("nan"))
    ws = m3.alloc_bwd_workspace_ex(d, T, ex)
    m3.m3_scan_bwd_ex(d, T, x.cuda(), g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"],
                      g["D"], st, ex, dy.cuda(), dh.cuda(), gr, xg, ws)
    assert m3.m3_query_status(ws) == m3.M3_OK
    torch.cuda.synchronize()
    # the call reads the starting state only
    assert torch.equal(st.h.cpu(), inp["h0"]) and torch.equal(st.B_prev.cpu(), inp["B_prev"])

    ref = oracle.scan_bwd_ex(f64(x), *(f64(inp[k]) for k in KEYS[1:]), f64(dy), D=f64(inp["D"]),
                             h0=f64(inp["h0"]), x_prev=f64(inp["x_prev"]),
                             B_prev=f64(inp["B_prev"]), dhT=f64(dh),
                             z=None if z is None else f64(z),
                             B_bias=f64(bb) if bias else None, C_bias=f64(cb) if bias else None,
                             bc_eps=eps, x_expand=f64(wx) if x_exp else None,
                             z_expand=f64(wz) if gate == "exp" else None)
    errs = {}
    for k, v in list(gr.items()) + list(xg.items()):
        got = f64(v)
        assert np.all(np.isfinite(got)), k
        assert got.shape == ref[k].shape, (k, got.shape, ref[k].shape)
        errs[k] = _rel(got, ref[k])
    assert all(e <= tol for e in errs.values()), errs


def test_bwd_ex_without_extras_is_the_plain_backward():
    """An all-zero extras block runs m3_scan_bwd itself: the same gradients (dx and the
    starting state's bit for bit; the scalar chains up to the order of shared-memory sums)."""
    b, H, G, P, N, R, T = 1, 2, 1, 64, 128, 1, 80
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=72,
                                  h0_random=True, carry_prev=True)
    dy = torch.randn((b, T, H, R, P), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    g = {k: v.cuda() for k, v in inp.items()}
    outs = []
    for use_ex in (False, True):
        st = m3.State(d)
        st.h.copy_(g["h0"])
        st.x_prev.copy_(g["x_prev"])
        st.B_prev.copy_(g["B_prev"])
        gr = m3.alloc_grads(d, T)
        ws = m3.alloc_bwd_workspace(d, T)
        args = (d, T, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"], g["D"], st)
        if use_ex:
            m3.m3_scan_bwd_ex(*args, m3.Extras(), dy.cuda(), None, gr, {}, ws)
        else:
            m3.m3_scan_bwd(*args, dy.cuda(), None, gr, ws)
        assert m3.m3_query_status(ws) == m3.M3_OK
        outs.append({k: v.cpu() for k, v in gr.items()})
    for k in ("dx", "dh0", "dx_prev"):
        assert torch.equal(outs[0][k], outs[1][k]), k
    for k in ("ddt", "dA", "dlam", "dB", "dC", "dtheta"):
        assert _rel(f64(outs[1][k]), f64(outs[0][k])) <= 1e-5, k
