"""Parity of the fused output gate (y * SiLU(z) after the skip; Mamba-3 paper summary,
"Technical Approach", output gating) on every kernel: the tcgen05 prefill, the sequential
fp32 prefill and the decode step, all through the C ABI, against the gated fp64 oracle.
The gate must leave the state untouched: the gated call's final state equals the
ungated call's up to the rounding of the kernel's own tiling."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import KEYS, f64, rel_slices
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu


def _scan(inp, z, d, T, Q, flags=0, gated=True, dev="cuda"):
    g = {k: v.to(dev) for k, v in inp.items()}
    st = m3.State(d, dev)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    y = torch.full_like(g["x"], float("nan"))
    ws = m3.alloc_workspace(d, T, Q, dev)
    args = [g[k] for k in KEYS] + [g["D"]]
    if gated:
        m3.m3_scan_fwd_gated(d, T, Q, *args, z.to(dev), st, y, ws, flags)
    else:
        m3.m3_scan_fwd(d, T, Q, *args, st, y, ws, flags)
    assert m3.m3_query_status(ws) == m3.M3_OK
    torch.cuda.synchronize()
    return f64(y), f64(st.h)


def _oracle(inp, z):
    return oracle.scan(*(f64(inp[k]) for k in KEYS), D=f64(inp["D"]), h0=f64(inp["h0"]),
                       x_prev=f64(inp["x_prev"]), B_prev=f64(inp["B_prev"]), z=f64(z))


CASES = [
    # (b, H, G, P, N, R, T, chunk, io, tol, flags)
    (2, 4, 1, 64, 128, 1, 300, 64, torch.bfloat16, 2e-2, 0),        # tensor cores, ragged tail
    (1, 4, 1, 64, 128, 1, 257, 128, torch.bfloat16, 2e-2, 0),       # chunk 128
    (1, 4, 1, 64, 64, 4, 150, 64, torch.bfloat16, 2e-2, 0),         # MIMO R = 4 (32-token tiles)
    (1, 4, 2, 64, 64, 2, 90, 32, torch.bfloat16, 2e-2, 0),          # MIMO R = 2, G = 2
    (1, 4, 1, 64, 128, 1, 200, 64, torch.bfloat16, 2e-2, m3.M3_FLAG_FORCE_SIMT),
    (1, 2, 1, 16, 16, 1, 256, 64, torch.float32, 1e-5, 0),          # fp32 sequential kernel
    (1, 3, 3, 8, 6, 3, 40, 16, torch.float32, 1e-5, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[f"N{c[4]}R{c[5]}T{c[6]}Q{c[7]}{'f32' if c[8] == torch.float32 else 'bf16'}{'S' if c[10] else ''}" for c in CASES])
def test_gated_scan_matches_oracle(case):
    b, H, G, P, N, R, T, Q, io, tol, flags = case
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=io, theta_max=math.pi / 8,
                                  seed=21, h0_random=True, carry_prev=True)
    z = inputs.make_gate((b, T, H, R, P), io_dtype=io, seed=21)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    yg, hg = _scan(inp, z, d, T, Q, flags)
    yo, ho, _, _ = _oracle(inp, z)
    assert np.all(np.isfinite(yg))
    assert rel_slices(yg, yo, (1, 3, 4)) <= tol
    assert rel_slices(hg, ho, (2, 3)) <= tol
    # the gate touches y only: the state matches the ungated call's, bit for bit where the
    # z ring leaves the kernel's tiling unchanged, else within the bf16 rounding of the MMA
    # operands (a different raw sub-chunk split rounds a few rotated B values differently)
    _, hu = _scan(inp, z, d, T, Q, flags, gated=False)
    assert rel_slices(hg, hu, (2, 3)) <= (2.0 ** -9 if io == torch.bfloat16 else 1e-6)


def test_gated_scan_extreme_gate_values():
    """Saturated gates: z = +-60 (bf16) pass y through (times z) or close it, without NaN."""
    b, H, G, P, N, R, T, Q = 1, 4, 1, 64, 128, 1, 130, 64
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=22)
    z = torch.where(torch.rand(b, T, H, R, P, generator=torch.Generator().manual_seed(1)) < 0.5,
                    torch.tensor(-60.0), torch.tensor(60.0)).to(torch.bfloat16)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    yg, _ = _scan(inp, z, d, T, Q)
    yo, _, _, _ = _oracle(inp, z)
    assert np.all(np.isfinite(yg))
    assert rel_slices(yg, yo, (1, 3, 4)) <= 2e-2


@pytest.mark.parametrize("shape,io,tol", [
    ((4, 8, 1, 64, 128, 1), torch.bfloat16, 2e-2),
    ((4, 8, 2, 64, 64, 4), torch.bfloat16, 2e-2),
    ((2, 6, 3, 8, 6, 3), torch.float32, 1e-5),
])
def test_gated_decode_matches_oracle(shape, io, tol):
    b, H, G, P, N, R = shape
    steps = 6
    inp = inputs.make_decode_inputs(b, H, G, P, N, R, tokens=steps, io_dtype=io, seed=23)
    z = inputs.make_gate((steps, b, H, R, P), io_dtype=io, seed=23)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    st = m3.State(d)
    st.h.copy_(inp["h0"])
    st.x_prev.copy_(inp["x_prev"])
    st.B_prev.copy_(inp["B_prev"])
    g = {k: inp[k].cuda() for k in KEYS}
    D, zg = inp["D"].cuda(), z.cuda()
    h, xp, bp = f64(inp["h0"]), f64(inp["x_prev"]), f64(inp["B_prev"])
    for t in range(steps):
        y = torch.empty_like(g["x"][t])
        m3.m3_decode_step_gated(d, *(g[k][t] for k in KEYS), D, zg[t], st, y)
        yo, h, xp, bp = oracle.decode_step(*(f64(inp[k][t]) for k in KEYS), f64(inp["D"]), h,
                                           xp, bp, z=f64(z[t]))
        assert rel_slices(f64(y), yo, (2, 3)) <= tol      # per (batch, head): [R][P]
    assert rel_slices(f64(st.h), h, (2, 3)) <= tol
