"""The no-allocation prefill entry point (m3_scan_fwd_noalloc) gives the same results as
m3_scan_fwd with a caller-provided workspace.

It serves callers that cannot allocate device memory themselves; the library lends
them a fixed scratch array instead.  Two calls in a row share that array, so the
second call also checks that the leftovers of the first one do no harm.  This file
sorts last so that a run stopping at the first failure has run every other test.
"""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import f64
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu


def _run(fn, inp, d, T, Q, **kw):
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    y = torch.empty_like(g["x"])
    fn(d, T, Q, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"], g["D"], st, y,
       **kw)
    torch.cuda.synchronize()
    return f64(y), f64(st.h), f64(st.x_prev), f64(st.B_prev)


@pytest.mark.parametrize("shape", [
    (2, 8, 1, 64, 128, 1, 300, 64, torch.bfloat16),     # tensor-core kernel
    (1, 2, 1, 16, 16, 1, 256, 64, torch.float32),        # sequential fp32 kernel
])
def test_noalloc_matches_workspace_entry_point(shape):
    b, H, G, P, N, R, T, Q, io = shape
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    for call, seed in enumerate((21, 22)):           # two calls in a row on the shared scratch
        inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=io, theta_max=math.pi / 4,
                                      seed=seed, h0_random=True, carry_prev=True)
        # a workspace of the scratch's size (64 KiB): like the no-allocation call, no room
        # for sequence-segment records, so both run the same unsegmented kernels
        ws = torch.zeros(64 * 1024, dtype=torch.uint8, device="cuda")
        ref = _run(lambda *a: m3.m3_scan_fwd(*a[:-1], a[-1], ws), inp, d, T, Q)
        got = _run(m3.m3_scan_fwd_noalloc, inp, d, T, Q)
        # the same deterministic kernel on the same inputs: bit-identical results, so that
        # nothing left in the shared scratch by the previous call can hide
        for k in range(4):
            assert np.array_equal(got[k], ref[k]), (call, k)
        assert np.all(np.isfinite(got[0]))


def test_noalloc_on_a_side_stream():
    """A stream of the current device other than the default one works the same way."""
    b, H, G, P, N, R, T, Q = 1, 4, 1, 64, 128, 1, 130, 64
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=torch.bfloat16, seed=23)
    ws = torch.zeros(64 * 1024, dtype=torch.uint8, device="cuda")
    ref = _run(lambda *a: m3.m3_scan_fwd(*a[:-1], a[-1], ws), inp, d, T, Q)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        got = _run(lambda *a: m3.m3_scan_fwd_noalloc(*a, stream=side), inp, d, T, Q)
    for k in range(4):
        assert np.array_equal(got[k], ref[k]), k
