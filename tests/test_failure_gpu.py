"""Failure path of the tensor-core prefill: a bounded device-side wait that runs out.

The test hook M3_FLAG_TEST_STALL makes one wait in the kernel target a barrier that
nothing completes; the wait gives up after 50 ms, the kernel aborts cleanly and the
host reads M3_ERR_TIMEOUT from the workspace status word.  No trap, no fault: the CUDA
context stays usable, which the follow-up call checks against the oracle."""
import numpy as np
import pytest
import torch

from gpu_helpers import gpu_scan, oracle_scan, scan_errors
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu


def test_stalled_wait_reports_timeout_and_context_survives():
    b, H, G, P, N, R, T, Q = 1, 4, 1, 64, 128, 1, 256, 64
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=31)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    y = torch.empty_like(g["x"])
    ws = m3.alloc_workspace(d, T, Q)
    m3.m3_scan_fwd(d, T, Q, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"],
                   g["D"], st, y, ws, flags=m3.M3_FLAG_TEST_STALL)
    assert m3.m3_query_status(ws) == m3.M3_ERR_TIMEOUT
    # the context is still usable and a normal call is correct
    yg, hg, _, _ = gpu_scan(inp, d, T, Q)
    yo, ho, _, _ = oracle_scan(inp)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert ey <= 2e-2 and eh <= 2e-2


def test_status_is_cleared_by_the_next_call():
    b, H, G, P, N, R, T, Q = 1, 4, 1, 64, 64, 1, 128, 64
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=32)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    y = torch.empty_like(g["x"])
    ws = m3.alloc_workspace(d, T, Q)
    args = (d, T, Q, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"], g["D"], st,
            y, ws)
    m3.m3_scan_fwd(*args, flags=m3.M3_FLAG_TEST_STALL)
    assert m3.m3_query_status(ws) == m3.M3_ERR_TIMEOUT
    m3.m3_state_init(d, st)
    m3.m3_scan_fwd(*args)
    assert m3.m3_query_status(ws) == m3.M3_OK
    assert np.all(np.isfinite(y.float().cpu().numpy()))
