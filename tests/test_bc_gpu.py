"""Parity of the fused BC map (Mamba-3 paper summary, "Technical Approach": BCNorm then
head-specific BC biases) on the tcgen05 prefill, the sequential fp32 prefill and the
decode step, through m3_scan_fwd_ex / m3_decode_step_ex, against the fp64 oracle with the
same map; also with the output gate on, and across a call split (the carried raw B_prev
must go through the map)."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import KEYS, f64, rel_slices
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu
EPS = 1e-6


def _run(inp, d, T, Q, ex_args, flags=0, calls=1, dev="cuda"):
    g = {k: v.to(dev) for k, v in inp.items()}
    st = m3.State(d, dev)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    y = torch.full_like(g["x"], float("nan"))
    bounds = np.linspace(0, T, calls + 1).astype(int)
    for c in range(calls):
        lo, hi = int(bounds[c]), int(bounds[c + 1])
        sl = {k: g[k][:, lo:hi].contiguous() for k in KEYS}
        z = ex_args.get("z")
        ex = m3.Extras(z=None if z is None else z.to(dev)[:, lo:hi].contiguous(),
                       B_bias=ex_args.get("B_bias"), C_bias=ex_args.get("C_bias"),
                       bc_norm_eps=ex_args.get("bc_norm_eps", 0.0))
        ws = m3.alloc_workspace_ex(d, hi - lo, Q, ex, dev)
        yc = torch.empty_like(sl["x"])
        m3.m3_scan_fwd_ex(d, hi - lo, Q, *(sl[k] for k in KEYS), g["D"], ex, st, yc, ws, flags)
        assert m3.m3_query_status(ws) == m3.M3_OK
        y[:, lo:hi] = yc
    torch.cuda.synchronize()
    return f64(y), f64(st.h), f64(st.B_prev)


CASES = [
    # (b, H, G, P, N, R, T, chunk, io, tol, flags, parts)
    (2, 4, 1, 64, 128, 1, 300, 64, torch.bfloat16, 2e-2, 0, "norm+bias"),
    (1, 4, 1, 64, 128, 1, 200, 64, torch.bfloat16, 2e-2, 0, "bias"),
    (1, 4, 1, 64, 128, 1, 200, 64, torch.bfloat16, 2e-2, 0, "norm"),
    (1, 4, 1, 64, 128, 1, 257, 128, torch.bfloat16, 2e-2, 0, "norm+bias+gate"),
    (1, 4, 1, 64, 64, 4, 150, 32, torch.bfloat16, 2e-2, 0, "norm+bias"),
    (1, 4, 2, 64, 64, 2, 90, 32, torch.bfloat16, 2e-2, 0, "norm+bias+gate"),
    (1, 4, 1, 64, 128, 1, 140, 64, torch.bfloat16, 2e-2, m3.M3_FLAG_FORCE_SIMT, "norm+bias"),
    (1, 2, 1, 16, 16, 1, 256, 64, torch.float32, 1e-5, 0, "norm+bias+gate"),
    (1, 3, 3, 8, 6, 3, 40, 16, torch.float32, 1e-5, 0, "norm+bias"),
]


def _parts(case, seed):
    b, H, G, P, N, R, T, Q, io, tol, flags, parts = case
    bb, cb = inputs.make_bc_bias(H, N, seed=seed)
    ex = {}
    if "bias" in parts:
        ex["B_bias"], ex["C_bias"] = bb, cb
    if "norm" in parts:
        ex["bc_norm_eps"] = EPS
    if "gate" in parts:
        ex["z"] = inputs.make_gate((b, T, H, R, P), io_dtype=io, seed=seed)
    return ex


def _oracle(inp, ex):
    z = ex.get("z")
    return oracle.scan(*(f64(inp[k]) for k in KEYS), D=f64(inp["D"]), h0=f64(inp["h0"]),
                       x_prev=f64(inp["x_prev"]), B_prev=f64(inp["B_prev"]),
                       z=None if z is None else f64(z),
                       B_bias=None if "B_bias" not in ex else f64(ex["B_bias"]),
                       C_bias=None if "C_bias" not in ex else f64(ex["C_bias"]),
                       bc_eps=ex.get("bc_norm_eps", 0.0))


def _ids(c):
    return f"N{c[4]}R{c[5]}T{c[6]}Q{c[7]}{'f32' if c[8] == torch.float32 else ''}{'S' if c[10] else ''}-{c[11]}"


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_bc_scan_matches_oracle(case):
    b, H, G, P, N, R, T, Q, io, tol, flags, parts = case
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=io, theta_max=math.pi / 8,
                                  seed=31, h0_random=True, carry_prev=True)
    ex = _parts(case, 31)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    gex = {k: (v.cuda() if k in ("B_bias", "C_bias") else v) for k, v in ex.items()}
    yg, hg, bpg = _run(inp, d, T, Q, gex, flags)
    yo, ho, _, bpo = _oracle(inp, ex)
    assert np.all(np.isfinite(yg)) and np.all(np.isfinite(hg))
    assert rel_slices(yg, yo, (1, 3, 4)) <= tol
    assert rel_slices(hg, ho, (2, 3)) <= tol
    assert np.array_equal(bpg, bpo)        # the state keeps the raw previous-token B


@pytest.mark.parametrize("chunk", [64, 128])
def test_bc_call_split(chunk):
    """Three chained calls equal one oracle pass: the carried raw B_prev is mapped."""
    b, H, G, P, N, R, T = 1, 4, 1, 64, 128, 1, 384
    case = (b, H, G, P, N, R, T, chunk, torch.bfloat16, 2e-2, 0, "norm+bias")
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=32,
                                  carry_prev=True)
    ex = _parts(case, 32)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    gex = {k: v.cuda() for k, v in ex.items() if k != "bc_norm_eps"}
    gex["bc_norm_eps"] = EPS
    yg, hg, _ = _run(inp, d, T, chunk, gex, calls=3)
    yo, ho, _, _ = _oracle(inp, ex)
    assert rel_slices(yg, yo, (1, 3, 4)) <= 2e-2 and rel_slices(hg, ho, (2, 3)) <= 2e-2


@pytest.mark.parametrize("shape,io,tol,parts", [
    ((4, 8, 1, 64, 128, 1), torch.bfloat16, 2e-2, "norm+bias"),    # SISO half-heads
    ((2, 4, 1, 64, 128, 1), torch.bfloat16, 2e-2, "bias"),
    ((2, 4, 1, 64, 128, 1), torch.bfloat16, 2e-2, "norm+gate"),
    ((2, 4, 2, 64, 128, 1), torch.float32, 1e-5, "norm+bias+gate"),
    ((4, 8, 2, 64, 64, 4), torch.bfloat16, 2e-2, "norm+bias+gate"),
    ((2, 6, 3, 8, 6, 3), torch.float32, 1e-5, "norm+bias+gate"),
    ((2, 4, 1, 16, 16, 2), torch.float32, 1e-5, "bias"),
    ((2, 4, 2, 64, 64, 2), torch.float32, 1e-5, "norm+bias+gate"),
])
def test_bc_decode_matches_oracle(shape, io, tol, parts):
    b, H, G, P, N, R = shape
    steps = 5
    inp = inputs.make_decode_inputs(b, H, G, P, N, R, tokens=steps, io_dtype=io, seed=33)
    bb, cb = inputs.make_bc_bias(H, N, seed=33)
    z = inputs.make_gate((steps, b, H, R, P), io_dtype=io, seed=33) if "gate" in parts else None
    eps = EPS if "norm" in parts else 0.0
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    st = m3.State(d)
    st.h.copy_(inp["h0"])
    st.x_prev.copy_(inp["x_prev"])
    st.B_prev.copy_(inp["B_prev"])
    g = {k: inp[k].cuda() for k in KEYS}
    D, bbg, cbg = inp["D"].cuda(), bb.cuda(), cb.cuda()
    h, xp, bp = f64(inp["h0"]), f64(inp["x_prev"]), f64(inp["B_prev"])
    for t in range(steps):
        y = torch.empty_like(g["x"][t])
        ex = m3.Extras(z=None if z is None else z[t].cuda(), B_bias=bbg, C_bias=cbg,
                       bc_norm_eps=eps)
        m3.m3_decode_step_ex(d, *(g[k][t] for k in KEYS), D, ex, st, y)
        yo, h, xp, bp = oracle.decode_step(*(f64(inp[k][t]) for k in KEYS), f64(inp["D"]), h,
                                           xp, bp, z=None if z is None else f64(z[t]),
                                           B_bias=f64(bb), C_bias=f64(cb), bc_eps=eps)
        assert rel_slices(f64(y), yo, (2, 3)) <= tol
    assert rel_slices(f64(st.h), h, (2, 3)) <= tol
    assert np.array_equal(f64(st.B_prev), bp)
