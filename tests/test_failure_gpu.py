"""Failure path of the tensor-core prefill and of the chunked tensor-core backward: a bounded
device-side wait that runs out.

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


@pytest.mark.parametrize("N,R", [(128, 1), (64, 4)], ids=["siso", "mimo_r4"])
def test_backward_stalled_wait_reports_timeout_and_context_survives(N, R):
    """The chunked backward's chunk-gradient kernel under the test hook: its issuing thread
    waits (50 ms) on a barrier nothing completes before it issues any MMA; the CTAs abort,
    drain their copies and release tensor memory; the status reads M3_ERR_TIMEOUT and a
    normal backward call right after is correct (SISO N 128 and MIMO rank 4 N 64)."""
    import oracle
    from gpu_helpers import KEYS, f64
    b, H, G, P, T = 1, 2, 1, 64, 100
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=34,
                                  h0_random=True, carry_prev=True)
    dy = torch.randn((b, T, H, R, P), generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    gr = m3.alloc_grads(d, T)
    ws = m3.alloc_bwd_workspace(d, T)
    args = (d, T, *(g[k] for k in KEYS), g["D"], st, dy.cuda(), None, gr, ws)
    m3.m3_scan_bwd(*args, flags=m3.M3_FLAG_TEST_STALL)
    assert m3.m3_query_status(ws) == m3.M3_ERR_TIMEOUT
    m3.m3_scan_bwd(*args)
    assert m3.m3_query_status(ws) == m3.M3_OK
    ref = oracle.scan_bwd(*(f64(inp[k]) for k in KEYS), f64(dy), D=f64(inp["D"]),
                          h0=f64(inp["h0"]), x_prev=f64(inp["x_prev"]), B_prev=f64(inp["B_prev"]))
    for k in m3.GRAD_NAMES:
        got = f64(gr[k])
        err = float(np.max(np.abs(got - ref[k])) / max(np.max(np.abs(ref[k])), 1e-30))
        assert err <= 2e-2, (k, err)
