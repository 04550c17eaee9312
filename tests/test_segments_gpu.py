"""Segment-parallel prefill of the tensor-core path.

With few (batch, head) streams per call (long sequences at small batch), the call splits
every sequence into segments run side by side: a segment pass from no entry state, a
chain step that composes the segments' affine maps ("Parallel representation under
SSD": the carried state is decay x rotation x entry state plus the segment's own part),
and the output pass.  Checked here: parity with the fp64 oracle (the same 2e-2 bf16 bar
as the unsegmented kernel), agreement with the unsegmented run of the same inputs (a
workspace without room for the segment records), and the carried state between calls.
"""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import KEYS, f64, oracle_scan, rel_slices, scan_errors
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu
TOL = 2e-2

CASES = [
    # (b, H, G, P, N, R, T, chunk, theta_max)
    (1, 4, 1, 64, 128, 1, 1000, 64, math.pi / 8),    # 16 chunks: 8 segments, ragged tail
    (1, 8, 1, 64, 128, 1, 1000, 128, math.pi),       # chunk 128, fast rotation
    (2, 4, 2, 64, 64, 1, 517, 64, math.pi / 8),      # N 64, two groups
    (1, 4, 1, 64, 64, 2, 300, 32, math.pi / 8),      # MIMO R 2
    (1, 4, 1, 64, 64, 4, 200, 16, math.pi / 8),      # MIMO R 4
]


def _run(inp, d, T, Q, ws, calls=1):
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    y = torch.full_like(g["x"], float("nan"))
    bounds = np.linspace(0, T, calls + 1).astype(int)
    for c in range(calls):
        lo, hi = int(bounds[c]), int(bounds[c + 1])
        sl = {k: g[k][:, lo:hi].contiguous() for k in KEYS}
        yc = torch.empty_like(sl["x"])
        m3.m3_scan_fwd(d, hi - lo, Q, sl["x"], sl["B"], sl["C"], sl["dt"], sl["A"], sl["lam"],
                       sl["theta"], g["D"], st, yc, ws)
        assert m3.m3_query_status(ws) == m3.M3_OK
        y[:, lo:hi] = yc
    torch.cuda.synchronize()
    return f64(y), f64(st.h), f64(st.x_prev), f64(st.B_prev)


@pytest.mark.parametrize("case", CASES, ids=[f"N{c[4]}R{c[5]}T{c[6]}Q{c[7]}b{c[0]}H{c[1]}" for c in CASES])
def test_segmented_matches_oracle_and_unsegmented(case):
    b, H, G, P, N, R, T, Q, tmax = case
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    full = m3.m3_scan_workspace_bytes(d, T, Q)
    assert full > 256, "this shape should run in segments"
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, theta_max=tmax,
                                  seed=31, h0_random=True, carry_prev=True)
    seg = _run(inp, d, T, Q, m3.alloc_workspace(d, T, Q))
    one = _run(inp, d, T, Q, torch.zeros(256, dtype=torch.uint8, device="cuda"))
    yo, ho, xpo, bpo = oracle_scan(inp)
    for got in (seg, one):
        assert np.all(np.isfinite(got[0])) and np.all(np.isfinite(got[1]))
        ey, eh = scan_errors(got[0], got[1], yo, ho)
        assert ey <= TOL and eh <= TOL, (ey, eh)
        assert np.array_equal(got[2], xpo) and np.array_equal(got[3], bpo)
    # the two runs differ only in rounding
    assert rel_slices(seg[0], one[0], (1, 3, 4)) <= TOL
    assert rel_slices(seg[1], one[1], (2, 3)) <= TOL


def test_segmented_chained_calls():
    """Four chained segmented calls (state carried between them) equal one oracle pass."""
    b, H, G, P, N, R, T, Q = 1, 8, 1, 64, 128, 1, 2048, 128
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    assert m3.m3_scan_workspace_bytes(d, T // 4, Q) > 256
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16,
                                  theta_max=math.pi, seed=32, h0_random=True, carry_prev=True)
    got = _run(inp, d, T, Q, m3.alloc_workspace(d, T // 4, Q), calls=4)
    yo, ho, xpo, bpo = oracle_scan(inp)
    ey, eh = scan_errors(got[0], got[1], yo, ho)
    assert ey <= TOL and eh <= TOL, (ey, eh)
    assert np.array_equal(got[2], xpo) and np.array_equal(got[3], bpo)


def test_long_call_with_few_heads():
    """A long call (batch 1, 16 heads, 4096 tokens, chunk 128) runs in segments; sampled
    heads against the oracle."""
    b, H, G, P, N, R, T, Q = 1, 16, 1, 64, 128, 1, 4096, 128
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    assert m3.m3_scan_workspace_bytes(d, T, Q) > 256
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16,
                                  theta_max=math.pi, seed=33, h0_random=True, carry_prev=True)
    got = _run(inp, d, T, Q, m3.alloc_workspace(d, T, Q))
    heads = [0, 7, 15]
    sub = {k: (v[:, :, heads].contiguous() if k in ("x", "dt", "A", "lam") else v)
           for k, v in inp.items()}
    sub["h0"] = inp["h0"][:, heads].contiguous()
    sub["x_prev"] = inp["x_prev"][:, heads].contiguous()
    sub["D"] = inp["D"][heads].contiguous()
    yo, ho, _, _ = oracle_scan(sub)
    ey, eh = scan_errors(got[0][:, :, heads], got[1][:, heads], yo, ho)
    assert ey <= TOL and eh <= TOL, (ey, eh)
