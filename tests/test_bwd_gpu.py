"""Parity of the backward pass (m3_scan_bwd, reverse-mode gradients of the recurrence) with
the fp64 oracle's backward, through the C ABI, on the same rounded inputs: the sequential fp32
kernel (every shape it covers; the bf16 P 64 shapes of the chunked tensor-core path, SISO
N 64 / 128 and MIMO ranks 2 / 4 with N 64, through M3_FLAG_FORCE_SIMT, since they would
otherwise take that path, checked in test_bwd_tc_gpu.py).

The kernel computes in fp32 (checkpoints every 16 tokens, recomputed segments), so the
bar is fp32 accumulation error: max |gpu - ref| / max |ref| per gradient tensor.  The full
1.5B-scale workload is checked on sampled heads: per-head gradients (dx, ddt, dA, dlam,
dh0, dx_prev) of two heads of batch row 0 against the oracle run on exactly those heads."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import KEYS, f64
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu

TOL = 2e-4


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _problem(b, H, G, P, N, R, T, io, seed, dhT=True):
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=io, theta_max=1.0, seed=seed,
                                  h0_random=True, carry_prev=True)
    gen = torch.Generator().manual_seed(seed + 5)
    dy = torch.randn((b, T, H, R, P), generator=gen).to(io)
    dh = torch.randn((b, H, N, P), generator=gen) if dhT else None
    return inp, dy, dh


def _gpu_bwd(inp, dy, dh, d, T, flags=0):
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    gr = m3.alloc_grads(d, T)
    for v in gr.values():
        v.fill_(float("nan"))
    ws = m3.alloc_bwd_workspace(d, T)
    m3.m3_scan_bwd(d, T, *(g[k] for k in KEYS), g["D"], st, dy.cuda(),
                   None if dh is None else dh.cuda(), gr, ws, flags)
    assert m3.m3_query_status(ws) == m3.M3_OK
    torch.cuda.synchronize()
    # the call reads the starting state only
    assert torch.equal(st.h.cpu(), inp["h0"]) and torch.equal(st.x_prev.cpu(), inp["x_prev"])
    return {k: f64(v) for k, v in gr.items()}


def _oracle_bwd(inp, dy, dh, angle=False):
    return oracle.scan_bwd(*(f64(inp[k]) for k in KEYS), f64(dy), D=f64(inp["D"]),
                           h0=f64(inp["h0"]), x_prev=f64(inp["x_prev"]),
                           B_prev=f64(inp["B_prev"]), dhT=None if dh is None else f64(dh),
                           theta_is_angle=angle)


CASES = [
    # (b, H, G, P, N, R, T, io, flags, dhT)
    (2, 2, 1, 3, 4, 2, 37, torch.float32, 0, True),        # ragged last segment, shared group
    (1, 3, 3, 8, 6, 3, 40, torch.float32, 0, False),       # G = H, no dL/dh_T
    (1, 2, 1, 16, 16, 1, 256, torch.float32, 0, True),     # the small fp32 SISO workload
    (1, 2, 1, 16, 16, 1, 50, torch.float32, m3.M3_FLAG_THETA_IS_ANGLE, True),
    (1, 4, 1, 64, 128, 1, 100, torch.bfloat16, m3.M3_FLAG_FORCE_SIMT, True),   # 1.5B-scale
    #                                   SISO head shape, on the sequential kernel
    (1, 4, 2, 64, 64, 4, 70, torch.bfloat16, m3.M3_FLAG_FORCE_SIMT, True),   # MIMO R = 4
    (2, 2, 1, 40, 10, 2, 33, torch.float32, 0, True),      # two column blocks, partial warp
]


def _id(c):
    return (f"b{c[0]}H{c[1]}G{c[2]}P{c[3]}N{c[4]}R{c[5]}T{c[6]}"
            f"{'f32' if c[7] == torch.float32 else 'bf16'}{'A' if c[8] else ''}{'' if c[9] else 'nodh'}")


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_backward_matches_oracle(case):
    b, H, G, P, N, R, T, io, flags, with_dh = case
    inp, dy, dh = _problem(b, H, G, P, N, R, T, io, seed=51, dhT=with_dh)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    got = _gpu_bwd(inp, dy, dh, d, T, flags)
    ref = _oracle_bwd(inp, dy, dh, angle=bool(flags & m3.M3_FLAG_THETA_IS_ANGLE))
    for k in m3.GRAD_NAMES:
        assert np.all(np.isfinite(got[k])), k
        assert _rel(got[k], ref[k]) <= TOL, (k, _rel(got[k], ref[k]))


def test_backward_rejects_bad_arguments():
    d = m3.Dims(1, 2, 1, 128, 16, 1, m3.M3_F32)     # P = 128: no backward kernel
    assert m3.m3_scan_bwd_workspace_bytes(d, 64) > 0
    inp, dy, dh = _problem(1, 2, 1, 16, 16, 1, 20, torch.float32, seed=3)
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_F32)
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    gr = m3.alloc_grads(d, 20)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(m3.M3Error):
        m3.m3_scan_bwd(d, 20, *(g[k] for k in KEYS), g["D"], st, dy.cuda(), None, gr, small)


def test_backward_fullsize_sampled_heads():
    """The 1.5B-scale SISO prefill workload (b8 H64 T4096 P64 N128, bf16), backward at full
    size; heads 0 and 37 of batch row 0 against the oracle on those two heads."""
    w = inputs.WORKLOADS["siso_prefill_1p5b"]
    b, H, G, P, N, R, T = w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank, w.seqlen
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=w.io_dtype, seed=7)
    gen = torch.Generator().manual_seed(12)
    dy = torch.randn((b, T, H, R, P), generator=gen).to(w.io_dtype)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    got = _gpu_bwd(inp, dy, None, d, T, m3.M3_FLAG_FORCE_SIMT)
    heads = [0, 37]
    sub = {k: inp[k][:1] for k in KEYS}
    for k in ("x", "dt", "A", "lam"):
        sub[k] = sub[k][:, :, heads]
    ref = oracle.scan_bwd(*(f64(sub[k]) for k in KEYS), f64(dy[:1, :, heads]),
                          D=f64(inp["D"][heads]), h0=f64(inp["h0"][:1, heads]),
                          x_prev=f64(inp["x_prev"][:1, heads]), B_prev=f64(inp["B_prev"][:1]))
    for k in ("dx", "ddt", "dA", "dlam"):
        assert _rel(got[k][:1, :, heads], ref[k]) <= TOL, k
    for k in ("dh0", "dx_prev"):
        assert _rel(got[k][:1, heads], ref[k]) <= TOL, k
    for k in ("dB", "dC", "dtheta", "dD"):
        assert np.all(np.isfinite(got[k])), k
