"""Prefill parity of the tcgen05 tensor-core kernel (bf16 io) against the fp64 oracle.

Tolerance: max relative error per (batch, head) slice <= 2e-2 on y and on the final
state, with the oracle fed the already-rounded bf16 inputs."""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import f64, gpu_scan, oracle_scan, rel_slices, scan_errors
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu
TOL = 2e-2


def dims_of(b, H, G, P, N, R):
    return m3.Dims(b, H, G, P, N, R, m3.M3_BF16)


CASES = [
    # (b, H, G, P, N, R, T, chunk, theta_max)
    (2, 4, 1, 64, 128, 1, 300, 64, math.pi / 8),     # SISO, ragged tail
    (1, 4, 4, 64, 128, 1, 257, 128, math.pi),        # SISO chunk 128, G = H, fast rotation
    (2, 8, 2, 64, 64, 1, 200, 64, math.pi / 8),      # SISO N = 64
    (1, 4, 1, 64, 64, 1, 130, 128, math.pi / 8),
    (2, 4, 1, 64, 64, 4, 130, 32, math.pi / 8),      # MIMO R = 4, Q*R = 128
    (1, 4, 1, 64, 64, 4, 77, 16, math.pi / 8),       # MIMO R = 4, Q*R = 64
    (1, 4, 2, 64, 64, 2, 150, 64, math.pi / 8),      # MIMO R = 2, Q*R = 128
    (1, 4, 1, 64, 64, 2, 33, 32, math.pi / 8),       # MIMO R = 2, Q*R = 64
    (1, 4, 1, 64, 128, 1, 1, 64, math.pi / 8),       # T = 1
    (1, 4, 1, 64, 128, 1, 64, 64, math.pi / 8),      # exactly one chunk
    (1, 4, 1, 64, 128, 1, 100, 32, math.pi / 8),     # chunk 32 runs as 64-token tiles
    (1, 4, 1, 64, 64, 4, 150, 64, math.pi / 8),      # R = 4, chunk 64 runs as 32-token tiles
    (1, 4, 1, 64, 64, 2, 90, 16, math.pi / 8),       # R = 2, chunk 16 runs as 32-token tiles
]


@pytest.mark.parametrize("case", CASES, ids=[f"N{c[4]}R{c[5]}T{c[6]}Q{c[7]}G{c[2]}" for c in CASES])
def test_tc_matches_oracle(case):
    b, H, G, P, N, R, T, Q, tmax = case
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, theta_max=tmax,
                                  seed=11, h0_random=True, carry_prev=True)
    d = dims_of(b, H, G, P, N, R)
    yg, hg, xpg, bpg = gpu_scan(inp, d, T, Q)
    yo, ho, xpo, bpo = oracle_scan(inp)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert np.all(np.isfinite(yg)) and np.all(np.isfinite(hg))
    assert ey <= TOL and eh <= TOL, (ey, eh)
    assert np.array_equal(xpg, xpo) and np.array_equal(bpg, bpo)


def test_tc_call_split_carry():
    """Four chained calls of the tensor-core kernel equal one oracle pass."""
    b, H, G, P, N, R, T, Q = 1, 8, 1, 64, 128, 1, 512, 128
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16,
                                  theta_max=math.pi, seed=12)
    d = dims_of(b, H, G, P, N, R)
    yg, hg, _, bpg = gpu_scan(inp, d, T, Q, calls=4)
    yo, ho, _, bpo = oracle_scan(inp)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert ey <= TOL and eh <= TOL, (ey, eh)
    assert np.array_equal(bpg, bpo)


@pytest.mark.parametrize("Q", [64, 128])
def test_tc_agrees_with_sequential_kernel(Q):
    """Chunked tensor-core result vs the sequential fp32 kernel on the same inputs."""
    b, H, G, P, N, R, T = 1, 4, 1, 64, 128, 1, 384
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=13)
    d = dims_of(b, H, G, P, N, R)
    yt, ht, _, _ = gpu_scan(inp, d, T, Q)
    ys, hs, _, _ = gpu_scan(inp, d, T, Q, flags=m3.M3_FLAG_FORCE_SIMT)
    assert rel_slices(yt, ys, (1, 3, 4)) <= TOL and rel_slices(ht, hs, (2, 3)) <= TOL


def test_tc_batch_row_slices_equal_one_call():
    """Calls on slices of the batch rows (State.rows views of one state) give exactly the
    results of one call over the whole batch: the rows are independent.  (The pipelined
    end-to-end bench leg runs the batch this way.)"""
    b, H, G, P, N, R, T, Q = 4, 4, 1, 64, 128, 1, 200, 64
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=14,
                                  h0_random=True, carry_prev=True)
    d = dims_of(b, H, G, P, N, R)
    g = {k: v.cuda() for k, v in inp.items()}
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")   # unsegmented either way

    def fresh():
        st = m3.State(d)
        st.h.copy_(g["h0"])
        st.x_prev.copy_(g["x_prev"])
        st.B_prev.copy_(g["B_prev"])
        return st

    st1, y1 = fresh(), torch.empty_like(g["x"])
    m3.m3_scan_fwd(d, T, Q, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"],
                   g["D"], st1, y1, ws)
    st2, y2 = fresh(), torch.empty_like(g["x"])
    for lo, hi in ((0, 1), (1, 3), (3, 4)):
        sv = st2.rows(lo, hi)
        m3.m3_scan_fwd(sv.dims, T, Q, *(g[k][lo:hi] for k in ("x", "B", "C", "dt", "A", "lam", "theta")),
                       g["D"], sv, y2[lo:hi], ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(st1.h, st2.h) and torch.equal(st1.x_prev, st2.x_prev)
    assert torch.equal(st1.B_prev, st2.B_prev)
