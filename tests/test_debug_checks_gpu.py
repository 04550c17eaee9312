"""M3_FLAG_DEBUG_CHECKS: the non-trapping device scan of the caller's value ranges.

The recurrence's coefficients have ranges ("Technical Approach", Proposition 1): the step
dt > 0 (after softplus), A <= 0 (alpha = exp(dt A) <= 1) and the trapezoid weight lam in
[0, 1] (after sigmoid); every other input must be finite.  With the flag, a host-made
out-of-range value is reported by m3_query_status as M3_ERR_RANGE, clean inputs give M3_OK,
and the flag changes no result."""
import math

import pytest
import torch

from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu


def _setup(io=torch.bfloat16, N=128, P=64, H=4):
    b, G, R, T, Q = 1, 1, 1, 200, 64
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=io, theta_max=math.pi / 8,
                                  seed=41)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    g = {k: v.cuda() for k, v in inp.items()}
    return d, g, T, Q


def _scan(d, g, T, Q, flags):
    st = m3.State(d)
    y = torch.empty_like(g["x"])
    ws = m3.alloc_workspace(d, T, Q)
    m3.m3_scan_fwd(d, T, Q, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"],
                   g["D"], st, y, ws, flags=flags)
    return m3.m3_query_status(ws), y, st.h


@pytest.mark.parametrize("io,N,P", [(torch.bfloat16, 128, 64), (torch.float32, 16, 16)],
                         ids=["tensor_core", "sequential"])
def test_clean_inputs_pass_and_results_unchanged(io, N, P):
    d, g, T, Q = _setup(io, N, P)
    s0, y0, h0 = _scan(d, g, T, Q, 0)
    s1, y1, h1 = _scan(d, g, T, Q, m3.M3_FLAG_DEBUG_CHECKS)
    assert s0 == m3.M3_OK and s1 == m3.M3_OK
    assert torch.equal(y0, y1) and torch.equal(h0, h1)


@pytest.mark.parametrize("key,index,value", [
    ("lam", (0, 17, 2), 1.5),        # trapezoid weight above 1
    ("lam", (0, 199, 3), -0.25),     # ... and below 0
    ("dt", (0, 5, 0), 0.0),          # step not positive
    ("A", (0, 100, 1), 0.1),         # growing mode: alpha > 1
    ("theta", (0, 3, 0, 7), float("inf")),
    ("x", (0, 150, 2, 0, 9), float("nan")),
    ("C", (0, 1, 0, 0, 100), float("inf")),
])
def test_out_of_range_value_is_reported(key, index, value):
    d, g, T, Q = _setup()
    g[key][index] = value
    status, _, _ = _scan(d, g, T, Q, m3.M3_FLAG_DEBUG_CHECKS)
    assert status == m3.M3_ERR_RANGE
    # without the flag nothing is scanned (the caller's contract)
    status, _, _ = _scan(d, g, T, Q, 0)
    assert status == m3.M3_OK


def test_backward_scan_reports_range():
    b, H, G, P, N, R, T = 1, 2, 1, 16, 16, 1, 64
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.float32, seed=42)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_F32)
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    dy = torch.ones_like(g["x"])
    gr = m3.alloc_grads(d, T)
    ws = m3.alloc_bwd_workspace(d, T)
    args = (d, T, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"], g["D"], st, dy,
            None, gr, ws)
    m3.m3_scan_bwd(*args, flags=m3.M3_FLAG_DEBUG_CHECKS)
    assert m3.m3_query_status(ws) == m3.M3_OK
    g["lam"][0, 10, 1] = 2.0
    m3.m3_scan_bwd(*args, flags=m3.M3_FLAG_DEBUG_CHECKS)
    assert m3.m3_query_status(ws) == m3.M3_ERR_RANGE
