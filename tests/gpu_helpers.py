"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the
fp64 oracle on the same (already rounded) inputs, and measure the error the way the
tolerance is stated: per (batch, head) slice, max |gpu - ref| / max |ref|."""
import numpy as np
import torch

import oracle
from state_space_model_06_b200 import m3

KEYS = ("x", "B", "C", "dt", "A", "lam", "theta")


def f64(t):
    return t.double().cpu().numpy()


def rel_slices(gpu, ref, axes):
    err = np.abs(gpu - ref).max(axis=axes)
    scale = np.maximum(np.abs(ref).max(axis=axes), 1e-30)
    return float((err / scale).max())


def scan_errors(yg, hg, yo, ho):
    """y [b,T,H,R,P] per (b,h); h [b,H,N,P] per (b,h)."""
    return rel_slices(yg, yo, (1, 3, 4)), rel_slices(hg, ho, (2, 3))


def gpu_scan(inp, dims, seqlen, chunk, flags=0, calls=1, D=True, dev="cuda"):
    """Run m3_scan_fwd over `seqlen` tokens split into `calls` chained calls."""
    g = {k: v.to(dev) for k, v in inp.items()}
    st = m3.State(dims, dev)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    y = torch.full_like(g["x"], float("nan"))
    bounds = np.linspace(0, seqlen, calls + 1).astype(int)
    ws = m3.alloc_workspace(dims, int(max(np.diff(bounds).max(), 1)), chunk, dev)
    for c in range(calls):
        lo, hi = int(bounds[c]), int(bounds[c + 1])
        sl = {k: g[k][:, lo:hi].contiguous() for k in KEYS}
        yc = torch.empty_like(sl["x"])
        m3.m3_scan_fwd(dims, hi - lo, chunk, sl["x"], sl["B"], sl["C"], sl["dt"], sl["A"],
                       sl["lam"], sl["theta"], g["D"] if D else None, st, yc, ws, flags)
        assert m3.m3_query_status(ws) == m3.M3_OK
        y[:, lo:hi] = yc
    torch.cuda.synchronize()
    return f64(y), f64(st.h), f64(st.x_prev), f64(st.B_prev)


def oracle_scan(inp, D=True, theta_is_angle=False):
    return oracle.scan(*(f64(inp[k]) for k in KEYS), D=f64(inp["D"]) if D else None,
                       h0=f64(inp["h0"]), x_prev=f64(inp["x_prev"]), B_prev=f64(inp["B_prev"]),
                       theta_is_angle=theta_is_angle)
