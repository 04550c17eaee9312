"""Prefill parity: m3_scan_fwd (CUDA, through the C ABI) vs the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import f64, gpu_scan, oracle_scan, scan_errors
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_TOL = 2e-2


def dims_of(b, H, G, P, N, R, io):
    return m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))


@pytest.mark.parametrize("G", [1, 2])
def test_siso_f32_small_config(G):
    """The fp32 oracle-scale configuration: b1, H2, T256, P16, N16, chunk 64."""
    w = inputs.WORKLOADS["siso_f32_small"]
    inp = inputs.make_scan_inputs(w.batch, w.seqlen, w.nheads, G, w.headdim, w.dstate, w.rank,
                                  io_dtype=w.io_dtype, theta_max=w.theta_max, seed=0)
    d = dims_of(w.batch, w.nheads, G, w.headdim, w.dstate, w.rank, w.io_dtype)
    yg, hg, xpg, bpg = gpu_scan(inp, d, w.seqlen, w.chunk)
    yo, ho, xpo, bpo = oracle_scan(inp)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert ey <= F32_TOL and eh <= F32_TOL, (ey, eh)
    assert np.array_equal(xpg, xpo) and np.array_equal(bpg, bpo)


@pytest.mark.parametrize("shape", [
    (2, 4, 2, 16, 16, 2, 100),      # MIMO R=2, ragged T
    (1, 3, 3, 12, 6, 3, 37),        # odd P, N=6, R=3, G=H
    (2, 2, 1, 32, 64, 1, 1),        # T = 1
    (1, 2, 1, 8, 256, 4, 50),       # large N
])
def test_f32_shapes(shape):
    b, H, G, P, N, R, T = shape
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.float32, seed=3,
                                  h0_random=True, carry_prev=True)
    d = dims_of(b, H, G, P, N, R, torch.float32)
    yg, hg, xpg, bpg = gpu_scan(inp, d, T, 64)
    yo, ho, xpo, bpo = oracle_scan(inp)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert ey <= F32_TOL and eh <= F32_TOL, (ey, eh)
    assert np.array_equal(xpg, xpo) and np.array_equal(bpg, bpo)


def test_f32_theta_is_angle_and_no_skip():
    b, H, G, P, N, R, T = 1, 2, 1, 16, 16, 1, 64
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.float32, theta_max=2.0,
                                  seed=4)
    d = dims_of(b, H, G, P, N, R, torch.float32)
    yg, hg, _, _ = gpu_scan(inp, d, T, 64, flags=m3.M3_FLAG_THETA_IS_ANGLE, D=False)
    yo, ho, _, _ = oracle_scan(inp, D=False, theta_is_angle=True)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert ey <= F32_TOL and eh <= F32_TOL, (ey, eh)


def test_f32_call_split_carries_state():
    """Three chained calls (h, x_prev, B_prev carried) equal one oracle pass."""
    b, H, G, P, N, R, T = 2, 2, 1, 16, 16, 2, 150
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.float32, theta_max=math.pi,
                                  seed=5)
    d = dims_of(b, H, G, P, N, R, torch.float32)
    yg, hg, xpg, bpg = gpu_scan(inp, d, T, 64, calls=3)
    yo, ho, xpo, bpo = oracle_scan(inp)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert ey <= F32_TOL and eh <= F32_TOL, (ey, eh)
    assert np.array_equal(bpg, bpo)


def test_seqlen_zero_is_noop():
    b, H, G, P, N, R = 1, 2, 1, 16, 16, 1
    d = dims_of(b, H, G, P, N, R, torch.float32)
    st = m3.State(d)
    st.h.normal_()
    h_before = st.h.clone()
    x = torch.empty(b, 0, H, R, P, device="cuda")
    Bt = torch.empty(b, 0, G, R, N, device="cuda")
    s = torch.empty(b, 0, H, device="cuda")
    th = torch.empty(b, 0, G, N // 2, device="cuda")
    ws = m3.alloc_workspace(d, 0, 64)
    m3.m3_scan_fwd(d, 0, 64, x, Bt, Bt, s, s, s, th, None, st, x, ws)
    torch.cuda.synchronize()
    assert torch.equal(st.h, h_before)


@pytest.mark.parametrize("shape,chunk", [
    ((2, 4, 1, 64, 128, 1, 300), 64),
    ((1, 4, 4, 64, 128, 1, 257), 128),
    ((2, 4, 1, 64, 64, 4, 130), 64),
    ((2, 4, 1, 64, 64, 4, 96), 32),
    ((1, 2, 1, 32, 32, 1, 70), 16),
])
def test_bf16_simt_path(shape, chunk):
    """bf16 io forced onto the sequential CUDA-core kernel."""
    b, H, G, P, N, R, T = shape
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=6,
                                  carry_prev=True)
    d = dims_of(b, H, G, P, N, R, torch.bfloat16)
    yg, hg, xpg, bpg = gpu_scan(inp, d, T, chunk, flags=m3.M3_FLAG_FORCE_SIMT)
    yo, ho, xpo, bpo = oracle_scan(inp)
    ey, eh = scan_errors(yg, hg, yo, ho)
    assert ey <= BF16_TOL and eh <= BF16_TOL, (ey, eh)
    assert np.array_equal(xpg, xpo) and np.array_equal(bpg, bpo)
