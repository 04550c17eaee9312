"""Decode parity: m3_decode_step (CUDA, through the C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import f64, rel_slices
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu
KEYS = ("x", "B", "C", "dt", "A", "lam", "theta")


def run_decode(inp, d, steps, dev="cuda"):
    st = m3.State(d, dev)
    st.h.copy_(inp["h0"])
    st.x_prev.copy_(inp["x_prev"])
    st.B_prev.copy_(inp["B_prev"])
    g = {k: inp[k].to(dev) for k in KEYS}
    D = inp["D"].to(dev)
    ys = []
    for t in range(steps):
        y = torch.empty_like(g["x"][t])
        m3.m3_decode_step(d, *(g[k][t] for k in KEYS), D, st, y)
        ys.append(y)
    torch.cuda.synchronize()
    return np.stack([f64(y) for y in ys]), f64(st.h), f64(st.x_prev), f64(st.B_prev)


def oracle_decode(inp, steps, bsel=slice(None), hsel=slice(None)):
    h = f64(inp["h0"])[bsel][:, hsel]
    xp = f64(inp["x_prev"])[bsel][:, hsel]
    bp = f64(inp["B_prev"])[bsel]
    ys = []
    for t in range(steps):
        one = []
        for k in KEYS:
            v = f64(inp[k][t])[bsel]
            if k in ("x", "dt", "A", "lam"):
                v = v[:, hsel]
            one.append(v)
        y, h, xp, bp = oracle.decode_step(*one, f64(inp["D"])[hsel], h, xp, bp)
        ys.append(y)
    return np.stack(ys), h, xp, bp


@pytest.mark.parametrize("shape,io,tol", [
    ((4, 8, 1, 64, 128, 1), torch.bfloat16, 2e-2),
    ((4, 8, 2, 64, 64, 4), torch.bfloat16, 2e-2),
    ((3, 4, 4, 16, 16, 2), torch.float32, 1e-5),
    ((2, 4, 1, 32, 256, 1), torch.float32, 1e-5),
    ((2, 6, 3, 8, 6, 3), torch.float32, 1e-5),
    # P = 64 at several batch / group / rank mixes, fp32 and bf16 io
    ((40, 8, 8, 64, 64, 2), torch.bfloat16, 2e-2),
    ((3, 4, 2, 64, 128, 1), torch.float32, 1e-5),
    ((2, 4, 1, 64, 128, 2), torch.bfloat16, 2e-2),
    ((5, 6, 3, 64, 64, 4), torch.float32, 1e-5),
])
def test_decode_steps(shape, io, tol):
    b, H, G, P, N, R = shape
    steps = 12
    inp = inputs.make_decode_inputs(b, H, G, P, N, R, tokens=steps, io_dtype=io, seed=7)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    yg, hg, xpg, bpg = run_decode(inp, d, steps)
    yo, ho, xpo, bpo = oracle_decode(inp, steps)
    assert rel_slices(yg, yo, (0, 3, 4)) <= tol
    assert rel_slices(hg, ho, (2, 3)) <= tol
    assert np.array_equal(xpg, xpo) and np.array_equal(bpg, bpo)


@pytest.mark.parametrize("name", ["decode_siso_b256", "decode_mimo_b256"])
def test_decode_full_size_sampled(name):
    """The batch-256 decode configurations at full size, a few steps, checked on
    sampled (batch, head) slices that the oracle computes one by one."""
    w = inputs.WORKLOADS[name]
    steps = 3
    inp = inputs.make_decode_inputs(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                                    tokens=steps, io_dtype=w.io_dtype, theta_max=w.theta_max,
                                    seed=8)
    d = m3.Dims(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank, m3.M3_BF16)
    yg, hg, _, bpg = run_decode(inp, d, steps)
    bsel = np.array([0, 1, 77, 200, 255])
    hsel = np.array([0, 13, 63])
    yo, ho, _, _ = oracle_decode(inp, steps, bsel, hsel)
    assert rel_slices(yg[:, bsel][:, :, hsel], yo, (0, 3, 4)) <= 2e-2
    assert rel_slices(hg[bsel][:, hsel], ho, (2, 3)) <= 2e-2
    assert np.all(np.isfinite(yg)) and np.all(np.isfinite(hg))
    assert np.array_equal(bpg, f64(inp["B"][steps - 1]))


@pytest.mark.parametrize("name", ["decode_siso_b256", "decode_mimo_b256"])
def test_decode_full_size_1000_tokens(name):
    """The batch-256 decode configurations over their stated horizon: 1000 sequential steps,
    each with a fresh token, at full size in the launch configuration the bench times.  The
    oracle recomputes sampled (batch, head) slices over all 1000 steps (every y and the final
    state); every output of every step is checked to be finite.  The fp32 state must stay
    within the bf16 bar after 1000 updates, not only after a few."""
    w = inputs.WORKLOADS[name]
    steps = w.extra["tokens"]
    inp = inputs.make_decode_inputs(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                                    tokens=steps, io_dtype=w.io_dtype, theta_max=w.theta_max,
                                    seed=9, device="cuda")
    d = m3.Dims(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank, m3.M3_BF16)
    bsel = torch.tensor([0, 5, 128, 201, 255])
    hsel = torch.tensor([0, 21, 63])
    st = m3.State(d)
    st.h.copy_(inp["h0"])
    st.x_prev.copy_(inp["x_prev"])
    st.B_prev.copy_(inp["B_prev"])
    y = torch.empty_like(inp["x"][0])
    ysel = torch.empty((steps, len(bsel), len(hsel), w.rank, w.headdim), dtype=y.dtype,
                       device="cuda")
    finite = torch.ones((), dtype=torch.bool, device="cuda")
    bs, hs = bsel.cuda(), hsel.cuda()
    for t in range(steps):
        m3.m3_decode_step(d, *(inp[k][t] for k in KEYS), inp["D"], st, y)
        ysel[t] = y[bs][:, hs]
        finite &= torch.isfinite(y).all()
    torch.cuda.synchronize()
    assert bool(finite) and bool(torch.isfinite(st.h).all())
    # the oracle on the sampled slices, fed the same (already rounded) inputs
    # (only the sampled slices come back to the host: the full inputs are gigabytes)
    sub = {k: f64(inp[k][:, bs]) for k in ("B", "C", "theta")}
    sub.update({k: f64(inp[k][:, bs][:, :, hs]) for k in ("x", "dt", "A", "lam")})
    h = f64(inp["h0"][bs][:, hs])
    xp = f64(inp["x_prev"][bs][:, hs])
    bp = f64(inp["B_prev"][bs])
    Dh = f64(inp["D"][hs])
    yo = []
    for t in range(steps):
        yt, h, xp, bp = oracle.decode_step(*(sub[k][t] for k in KEYS), Dh, h, xp, bp)
        yo.append(yt)
    yo = np.stack(yo)
    assert rel_slices(f64(ysel), yo, (0, 3, 4)) <= 2e-2
    assert rel_slices(f64(st.h[bs][:, hs]), h, (2, 3)) <= 2e-2
    assert torch.equal(st.B_prev, inp["B"][steps - 1])
