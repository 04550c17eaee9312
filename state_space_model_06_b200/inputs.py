"""Seeded synthetic inputs for the Mamba-3 mixer hot path.

This module is the only code that both the CUDA path's tests/bench and the CPU
oracle's callers share.  It draws random numbers and shapes them; it holds none
of the recurrence's arithmetic.

Distributions (a 1.5B-scale Mamba-3 layer: d_model 2048, expand 2, headdim 64,
so 64 heads; state size 128 -- the Mamba-3 paper summary, "Experimental
Analysis", Table 6 setting):

    x ~ N(0, 1);  B, C ~ N(0, 1/N)  (variance 1/N)
    dt  = softplus(z), z ~ N(-2, 1)          (step size, after softplus)
    A   = -exp(z),     z ~ N(0, 0.5)         (per token, per head; variance 0.5)
    lam = sigmoid(z),  z ~ N(0, 1)           (trapezoid weight, after sigmoid)
    theta ~ U(-theta_max, theta_max)         (per token, per group, N/2 angles)
    D ~ N(0, 1) per head;  h0 = 0 for prefill, N(0, 1) for decode

Draw order is fixed: x, B, C, dt, A, lam, theta, D, h0 (then x_prev, B_prev when
a carried previous token is requested), with a CPU ``torch.Generator`` seeded by
``seed``.  Large tensors are drawn one batch row at a time (a fixed, documented
order) and rounded to the io dtype right away, so host memory stays bounded.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    nheads: int
    ngroups: int
    headdim: int
    dstate: int
    rank: int
    seqlen: int
    chunk: int
    io_dtype: torch.dtype
    theta_max: float = math.pi / 8
    calls: int = 1                      # seqlen is split into this many chained calls
    extra: dict = field(default_factory=dict)


# The five measured configurations of the hot path.
WORKLOADS = {
    "siso_f32_small": Workload("siso_f32_small", 1, 2, 1, 16, 16, 1, 256, 64, torch.float32),
    "siso_prefill_1p5b": Workload("siso_prefill_1p5b", 8, 64, 1, 64, 128, 1, 4096, 64,
                                  torch.bfloat16),
    "mimo_prefill_r4": Workload("mimo_prefill_r4", 8, 64, 1, 64, 64, 4, 4096, 64, torch.bfloat16),
    "decode_siso_b256": Workload("decode_siso_b256", 256, 64, 1, 64, 128, 1, 1, 1, torch.bfloat16,
                                 extra={"tokens": 1000}),
    "decode_mimo_b256": Workload("decode_mimo_b256", 256, 64, 1, 64, 64, 4, 1, 1, torch.bfloat16,
                                 extra={"tokens": 1000}),
    "siso_longctx_carry": Workload("siso_longctx_carry", 1, 64, 1, 64, 128, 1, 65536, 128,
                                   torch.bfloat16, theta_max=math.pi, calls=16),
}


def _randn(g, shape, std=1.0, mean=0.0, dtype=torch.float32):
    """Draw N(mean, std^2) one leading row at a time, rounded to ``dtype`` (on the
    generator's device)."""
    out = torch.empty(shape, dtype=dtype, device=g.device)
    for i in range(shape[0]):
        r = torch.randn(shape[1:], generator=g, device=g.device)
        if std != 1.0:
            r.mul_(std)
        if mean != 0.0:
            r.add_(mean)
        out[i].copy_(r)
    return out


def make_scan_inputs(batch, seqlen, nheads, ngroups, headdim, dstate, rank=1,
                     io_dtype=torch.bfloat16, theta_max=math.pi / 8, seed=0,
                     h0_random=False, carry_prev=False):
    """Inputs of one prefill call, as CPU tensors in the library's layouts.

    x [b,T,H,R,P] and B, C [b,T,G,R,N] in ``io_dtype``; dt, A, lam [b,T,H],
    theta [b,T,G,N/2], D [H], h0 [b,H,N,P] in float32; x_prev [b,H,R,P] and
    B_prev [b,G,R,N] in ``io_dtype`` (zeros unless ``carry_prev``).
    """
    b, T, H, G, P, N, R = batch, seqlen, nheads, ngroups, headdim, dstate, rank
    g = torch.Generator("cpu").manual_seed(seed)
    inp = {}
    inp["x"] = _randn(g, (b, T, H, R, P), dtype=io_dtype)
    inp["B"] = _randn(g, (b, T, G, R, N), std=1.0 / math.sqrt(N), dtype=io_dtype)
    inp["C"] = _randn(g, (b, T, G, R, N), std=1.0 / math.sqrt(N), dtype=io_dtype)
    inp["dt"] = torch.nn.functional.softplus(torch.randn((b, T, H), generator=g) - 2.0)
    inp["A"] = -torch.exp(torch.randn((b, T, H), generator=g) * math.sqrt(0.5))
    inp["lam"] = torch.sigmoid(torch.randn((b, T, H), generator=g))
    inp["theta"] = (torch.rand((b, T, G, N // 2), generator=g) * 2.0 - 1.0) * theta_max
    inp["D"] = torch.randn((H,), generator=g)
    if h0_random:
        inp["h0"] = torch.randn((b, H, N, P), generator=g)
    else:
        inp["h0"] = torch.zeros((b, H, N, P))
    if carry_prev:
        inp["x_prev"] = torch.randn((b, H, R, P), generator=g).to(io_dtype)
        inp["B_prev"] = (torch.randn((b, G, R, N), generator=g) / math.sqrt(N)).to(io_dtype)
    else:
        inp["x_prev"] = torch.zeros((b, H, R, P), dtype=io_dtype)
        inp["B_prev"] = torch.zeros((b, G, R, N), dtype=io_dtype)
    return inp


def make_gate(shape, io_dtype=torch.bfloat16, seed=0, device="cpu"):
    """Output-gate input z ~ N(0, 1) of the given shape (the layout of y), rounded to the io
    dtype.  Drawn from its own generator (seed + 7919) so that adding a gate never changes
    the other inputs of a seeded workload; ``device`` as for ``make_decode_inputs``."""
    g = torch.Generator(device).manual_seed(seed + 7919)
    return _randn(g, tuple(shape), dtype=io_dtype)


def make_bc_bias(nheads, dstate, seed=0):
    """BC biases B_bias, C_bias [H][N] float32: the pages' all-ones initialisation plus a
    per-channel N(0, 0.3^2) spread (a trained layer's biases are not all equal).  Own
    generator (seed + 104729): adding biases never changes the other seeded inputs."""
    g = torch.Generator("cpu").manual_seed(seed + 104729)
    return (1.0 + 0.3 * torch.randn((nheads, dstate), generator=g),
            1.0 + 0.3 * torch.randn((nheads, dstate), generator=g))


def make_expand(nheads, rank, headdim, seed=0):
    """MIMO lightweight-expansion weights x_expand, z_expand [H][R][P] float32, N(0, 1) (the
    pages fix no initialisation; unit scale keeps X = x * w at the scale of x).  Own
    generator (seed + 15485863): adding them never changes the other seeded inputs.  The
    per-channel input x [.., H, P] of an expanded workload is rank column 0 of the drawn x."""
    g = torch.Generator("cpu").manual_seed(seed + 15485863)
    return (torch.randn((nheads, rank, headdim), generator=g),
            torch.randn((nheads, rank, headdim), generator=g))


def make_decode_inputs(batch, nheads, ngroups, headdim, dstate, rank=1, tokens=1,
                       io_dtype=torch.bfloat16, theta_max=math.pi / 8, seed=0, device="cpu"):
    """Per-token decode inputs stacked over ``tokens`` plus the starting state.

    x [tok,b,H,R,P], B, C [tok,b,G,R,N] (io dtype); dt, A, lam [tok,b,H];
    theta [tok,b,G,N/2]; D [H]; h0 [b,H,N,P] ~ N(0,1) float32;
    x_prev [b,H,R,P], B_prev [b,G,R,N] drawn like x and B (io dtype).

    ``device`` selects the generator: "cpu" (the default; a CPU ``torch.Generator``) or a
    CUDA device, where torch's seeded device generator draws the same distributions in the
    same order straight into device memory.  The two give different values for one seed.
    Long full-size decode horizons (1000 fresh tokens of batch 256 are gigabytes) are drawn
    on the device; a test that checks them against the oracle copies the slices it checks
    back to the host.
    """
    b, H, G, P, N, R, K = batch, nheads, ngroups, headdim, dstate, rank, tokens
    g = torch.Generator(device).manual_seed(seed)
    dev = g.device

    def rn(shape):
        return torch.randn(shape, generator=g, device=dev)

    inp = {}
    inp["x"] = _randn(g, (K, b, H, R, P), dtype=io_dtype)
    inp["B"] = _randn(g, (K, b, G, R, N), std=1.0 / math.sqrt(N), dtype=io_dtype)
    inp["C"] = _randn(g, (K, b, G, R, N), std=1.0 / math.sqrt(N), dtype=io_dtype)
    inp["dt"] = torch.nn.functional.softplus(rn((K, b, H)) - 2.0)
    inp["A"] = -torch.exp(rn((K, b, H)) * math.sqrt(0.5))
    inp["lam"] = torch.sigmoid(rn((K, b, H)))
    inp["theta"] = (torch.rand((K, b, G, N // 2), generator=g, device=dev) * 2.0 - 1.0) * theta_max
    inp["D"] = rn((H,))
    inp["h0"] = _randn(g, (b, H, N, P))
    inp["x_prev"] = rn((b, H, R, P)).to(io_dtype)
    inp["B_prev"] = (rn((b, G, R, N)) / math.sqrt(N)).to(io_dtype)
    return inp
