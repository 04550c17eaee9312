"""Prefill parity at the full sizes of the measured workloads.

The GPU runs the whole workload in the launch configuration the bench uses; the fp64
oracle recomputes sampled (batch, head) slices one by one (heads are independent, and
with one group every head reads the same B, C, theta), and every output is checked to
be finite."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import KEYS, f64, rel_slices
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu
TOL = 2e-2


def run_workload(w, chunk=None, calls=1, seed=0, flags=0):
    Q = chunk or w.chunk
    inp = inputs.make_scan_inputs(w.batch, w.seqlen, w.nheads, w.ngroups, w.headdim, w.dstate,
                                  w.rank, io_dtype=w.io_dtype, theta_max=w.theta_max, seed=seed)
    d = m3.Dims(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                m3.io_dtype_of(w.io_dtype))
    st = m3.State(d)
    m3.m3_state_init(d, st)
    D = inp["D"].cuda()
    Tc = w.seqlen // calls
    ws = m3.alloc_workspace(d, Tc, Q)
    ys = []
    for c in range(calls):
        sl = {k: inp[k][:, c * Tc:(c + 1) * Tc].contiguous().cuda() for k in KEYS}
        y = torch.empty_like(sl["x"])
        m3.m3_scan_fwd(d, Tc, Q, sl["x"], sl["B"], sl["C"], sl["dt"], sl["A"], sl["lam"],
                       sl["theta"], D, st, y, ws, flags=flags)
        assert m3.m3_query_status(ws) == m3.M3_OK
        ys.append(y.cpu())
        del sl
    torch.cuda.synchronize()
    return inp, torch.cat(ys, dim=1), st.h.cpu()


def oracle_slices(inp, bsel, hsel):
    """The oracle on batch rows bsel and heads hsel (one group: B, C, theta shared)."""
    sub = {}
    for k in KEYS:
        v = inp[k][bsel]
        if k in ("x", "dt", "A", "lam"):
            v = v[:, :, hsel]
        sub[k] = f64(v)
    return oracle.scan(*(sub[k] for k in KEYS), D=f64(inp["D"])[hsel])


def check(inp, yg, hg, bsel, hsel):
    assert bool(torch.isfinite(yg).all()) and bool(torch.isfinite(hg).all())
    yo, ho, _, _ = oracle_slices(inp, bsel, hsel)
    ys = f64(yg[bsel][:, :, hsel])
    hs = f64(hg[bsel][:, hsel])
    assert rel_slices(ys, yo, (1, 3, 4)) <= TOL
    assert rel_slices(hs, ho, (2, 3)) <= TOL


def test_siso_prefill_1p5b_full():
    w = inputs.WORKLOADS["siso_prefill_1p5b"]
    inp, yg, hg = run_workload(w)
    check(inp, yg, hg, [0, 7], [0, 37, 63])


@pytest.mark.parametrize("chunk,flags", [(64, 0), (32, 0), (64, m3.M3_FLAG_FORCE_SIMT)],
                         ids=["chunk64", "chunk32", "chunk64_sequential"])
def test_mimo_prefill_r4_full(chunk, flags):
    """R = 4 on the tensor-core kernel (chunk 64 runs as 32-token tiles, chunk * R = 128
    rows) and on the sequential fp32 kernel."""
    w = inputs.WORKLOADS["mimo_prefill_r4"]
    inp, yg, hg = run_workload(w, chunk=chunk, seed=1, flags=flags)
    check(inp, yg, hg, [3], [5, 60])


def test_longctx_carry_full():
    """65536 tokens as 16 chained calls of 4096 (state and previous token carried),
    chunk 128, fast rotation theta ~ U(-pi, pi)."""
    w = inputs.WORKLOADS["siso_longctx_carry"]
    inp, yg, hg = run_workload(w, calls=w.calls, seed=2)
    check(inp, yg, hg, [0], [11, 50])
