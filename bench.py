"""Benchmark of the Mamba-3 mixer hot path on B200.

One step = one m3_scan_fwd call over the SISO 1.5B-scale prefill workload
(batch 8, 64 heads, T 4096, P 64, N 128, chunk 64, bf16 x/B/C, fp32 dt/A/lam/theta/state),
i.e. every prefill step of the method.  Alongside, as sub-metrics: the batch-256 decode
workloads (SISO N 128 and MIMO R 4 N 64; 1000 sequential steps with fresh tokens, captured
once as a CUDA graph and replayed), the same prefill and decode with the fused output gate
("gated") and with BCNorm + BC biases ("bc"), the MIMO rank-4 prefill plain and with the
lightweight expansion of x and z, and its backward pass ("mimo"), the long-context workload of
16 chained calls
("longctx") and the fp32 parity workload ("small_f32"), the backward pass of the prefill
workload ("backward"), the end-to-end call through pinned host
buffers ("e2e"), and the CPU oracle on the workload's inputs ("cpu_baseline").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Profiling subsets (their lines are not measurements of the full set): --prefill-only,
--bwd-only (the prefill line and the SISO backward), --mimo-only (the prefill line and the
MIMO leg); --batch / --seqlen shrink the workloads for short ncu captures.

N > 1 runs one independent replica per GPU (the path has no cross-GPU exchange:
every (batch, head) recurrence is independent), launched with torch.distributed.run;
times are CUDA-event device times, max over ranks.  Rank 0 prints one JSON line.

`--impl reference` times the CPU oracle (plain fp64 C, OpenMP) on host cores on a
bounded sample of the same workload and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from state_space_model_06_b200 import inputs, m3  # noqa: E402

METRIC = ("prefill tokens/s/layer (% tensor peak); decode tok/s at batch 256 (% HBM BW)")
WORKLOAD = "siso_prefill_1p5b"
DECODES = ("decode_siso_b256", "decode_mimo_b256")
DECODE_TOKENS = 1000        # sequential decode steps, each with a fresh pre-generated token
BC_EPS = 1e-6              # BCNorm epsilon of the BC legs
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def peaks():
    """The measured peaks (HBM GB/s, bf16 TFLOP/s) of MEASURED_PEAKS.json where present, else
    the fallback figures; a key that is missing or not a number falls back on its own."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        return FALLBACK_PEAKS, "fallback"
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"
    out, kind = dict(FALLBACK_PEAKS), "measured"
    for k in FALLBACK_PEAKS:
        v = d.get(k) if isinstance(d, dict) else None
        if isinstance(v, dict):
            v = v.get("value")
        if isinstance(v, (int, float)) and v > 0:
            out[k] = float(v)
        else:
            kind = "measured (fallback for missing keys)"
    return out, kind


def scan_algorithmic(w):
    """Algorithmic bytes and FLOPs of one prefill call (each tensor read or written once;
    FLOPs of the four chunk contractions, causal half of the intra-chunk products)."""
    b, T, H, G, P, N, R, Q = w.batch, w.seqlen, w.nheads, w.ngroups, w.headdim, w.dstate, \
        w.rank, w.chunk
    e = 2
    per_head_tok = 2 * P * R * e + 3 * 4                  # x in, y out, dt/A/lam
    per_group_tok = 2 * N * R * e + (N // 2) * 4          # B, C, theta
    state = b * H * N * P * 4 * 2 + b * H * R * P * e * 2 + b * G * R * N * e * 2
    byts = b * T * (H * per_head_tok + G * per_group_tok) + state
    nchunk = math.ceil(T / Q)
    tri = Q * (Q + 1) // 2
    flops_chunk = tri * R * R * 2 * N + tri * R * R * 2 * P + 2 * N * P * Q * R + 2 * Q * R * N * P
    flops = b * H * nchunk * flops_chunk
    return byts, flops


def decode_algorithmic(w):
    b, H, G, P, N, R = w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank
    e = 2
    byts = (2 * b * H * N * P * 4            # state read + write
            + 4 * b * H * R * P * e          # x, x_prev in, x_prev out, y
            + 4 * b * G * R * N * e          # B, C, B_prev in, B_prev out
            + 3 * b * H * 4 + b * G * (N // 2) * 4 + H * 4)
    return byts


def source_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def committed_counters(kernel_src, workload):
    """The committed ncu figures of the workload's kernel (DRAM traffic per launch, tensor-pipe
    utilisation), if they were taken on the current kernel source (else an empty dict)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        d = json.load(f)
    ent = d.get(workload)
    if not ent or ent.get("source_sha256_16") != source_hash(kernel_src):
        return {}
    return ent


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running (read only)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, period=0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop, self._t = period, threading.Event(), None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: clocks reported as unknown
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = fn(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons - {"gpu_idle"})}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return ws, rank, local


def max_over_ranks(x, ws):
    """Maximum of a per-rank float over all ranks (device times are reported as the max)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, ms_per_rank, ws):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    ms = max_over_ranks(ms_per_rank, ws)
    return ws * units_per_rank / (ms / 1e3), ms


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- our arm
def prefill_setup(w, dev, seed):
    inp = inputs.make_scan_inputs(w.batch, w.seqlen, w.nheads, w.ngroups, w.headdim, w.dstate,
                                  w.rank, io_dtype=w.io_dtype, theta_max=w.theta_max, seed=seed)
    d = m3.Dims(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                m3.io_dtype_of(w.io_dtype))
    g = {k: v.to(dev) for k, v in inp.items()}
    st = m3.State(d, dev)
    y = torch.empty_like(g["x"])
    ws = m3.alloc_workspace(d, w.seqlen, w.chunk, dev)
    return inp, d, g, st, y, ws


def run_scan(w, d, g, st, y, ws, stream):
    m3.m3_scan_fwd(d, w.seqlen, w.chunk, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"],
                   g["theta"], g["D"], st, y, ws, stream=stream)


def time_prefill(w, d, g, st, y, ws, steps, warmup, stream, ws_world):
    for _ in range(warmup):
        m3.m3_state_init(d, st, stream=stream)
        run_scan(w, d, g, st, y, ws, stream)
    torch.cuda.synchronize()
    barrier(ws_world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        m3.m3_state_init(d, st, stream=stream)         # fresh sequence each step (memsets)
        ev[i][0].record(stream)
        run_scan(w, d, g, st, y, ws, stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(ws_world)
    torch.cuda.synchronize()
    status = m3.m3_query_status(ws, stream)
    per = [a.elapsed_time(b) for a, b in ev]
    return sum(per) / steps, status


def time_prefill_ex(w, d, g, ex, st, y, ws, steps, warmup, stream):
    """The same prefill step through m3_scan_fwd_ex with the fused parts in ``ex``."""
    def run():
        m3.m3_scan_fwd_ex(d, w.seqlen, w.chunk, g["x"], g["B"], g["C"], g["dt"], g["A"],
                          g["lam"], g["theta"], g["D"], ex, st, y, ws, stream=stream)
    for _ in range(warmup):
        m3.m3_state_init(d, st, stream=stream)
        run()
    torch.cuda.synchronize()
    per = []
    for _ in range(steps):
        m3.m3_state_init(d, st, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        per.append((e0, e1))
    torch.cuda.synchronize()
    status = m3.m3_query_status(ws, stream)
    if status != m3.M3_OK:
        raise RuntimeError(f"device status {m3.m3_status_string(status)}")
    return sum(a.elapsed_time(b) for a, b in per) / steps


def time_prefill_e2e(w, d, inp, st, ws, steps, stream, dev, slices=8):
    """Same call through host buffers: pinned H2D of the step's inputs, the call, D2H of y.

    The batch rows are independent, so a step runs as `slices` calls on row slices over three
    streams: the H2D copy of slice i + 1, the call on slice i and the D2H copy of slice i - 1
    overlap (PCIe is full duplex).  Every byte of the step's inputs and of y still crosses
    PCIe inside the timed region; a slice's buffers are reused only after the previous step's
    call (inputs) or copy (y) of that slice is done."""
    keys = ("x", "B", "C", "dt", "A", "lam", "theta")
    nb = d.batch
    S = max(1, min(slices, nb))
    bounds = [nb * i // S for i in range(S + 1)]
    host = {k: inp[k].pin_memory() for k in keys + ("D",)}
    devb = {k: torch.empty_like(inp[k], device=dev) for k in keys + ("D",)}
    y = torch.empty_like(devb["x"])
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y.numel() * y.element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    done_call = [None] * S   # the last call on each slice (its inputs may be overwritten after)
    done_copy = [None] * S   # the last D2H of each slice (its y may be overwritten after)

    def step():
        for i in range(S):
            lo, hi = bounds[i], bounds[i + 1]
            dsl = dataclasses.replace(d, batch=hi - lo)
            stv = st.rows(lo, hi)
            with torch.cuda.stream(s_in):
                if done_call[i] is not None:
                    s_in.wait_event(done_call[i])
                if i == 0:
                    devb["D"].copy_(host["D"], non_blocking=True)
                for k in keys:
                    devb[k][lo:hi].copy_(host[k][lo:hi], non_blocking=True)
                ein = torch.cuda.Event()
                ein.record(s_in)
            stream.wait_event(ein)
            if done_copy[i] is not None:
                stream.wait_event(done_copy[i])
            m3.m3_state_init(dsl, stv, stream=stream)
            m3.m3_scan_fwd(dsl, w.seqlen, w.chunk, devb["x"][lo:hi], devb["B"][lo:hi],
                           devb["C"][lo:hi], devb["dt"][lo:hi], devb["A"][lo:hi],
                           devb["lam"][lo:hi], devb["theta"][lo:hi], devb["D"], stv, y[lo:hi],
                           ws, stream=stream)
            ec = torch.cuda.Event()
            ec.record(stream)
            done_call[i] = ec
            s_out.wait_event(ec)
            with torch.cuda.stream(s_out):
                y_host[lo:hi].copy_(y[lo:hi], non_blocking=True)
                eo = torch.cuda.Event()
                eo.record(s_out)
            done_copy[i] = eo

    step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in range(steps):
        step()
    e1.record(s_out)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h, S


def time_decode(name, dev, stream, seed, tokens=DECODE_TOKENS, gated=False, bc=False):
    """`tokens` sequential decode steps of the workload, each with its own fresh token
    (drawn up front on the device by the seeded generator of ``inputs``).  The whole
    sequence is captured once as one CUDA graph and replayed: a step is ~0.2 ms of device
    time, about what a host launch through ctypes costs, so steps launched one by one would
    time the host.  The state is reset to the drawn starting state before each replay."""
    w = inputs.WORKLOADS[name]
    g = inputs.make_decode_inputs(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                                  tokens=tokens, io_dtype=w.io_dtype, theta_max=w.theta_max,
                                  seed=seed, device=dev)
    d = m3.Dims(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                m3.io_dtype_of(w.io_dtype))
    st = m3.State(d, dev)
    y = torch.empty_like(g["x"][0])
    keys = ("x", "B", "C", "dt", "A", "lam", "theta")
    z = None
    if gated:
        z = inputs.make_gate(g["x"].shape, io_dtype=w.io_dtype, seed=seed, device=dev)
    bias = [v.to(dev) for v in inputs.make_bc_bias(w.nheads, w.dstate, seed=seed)] if bc else None

    def step(t):   # on the current stream: the capture stream while the graph is recorded
        tok = [g[k][t] for k in keys]
        if bc:
            ex = m3.Extras(z=None if z is None else z[t], B_bias=bias[0], C_bias=bias[1],
                           bc_norm_eps=BC_EPS)
            m3.m3_decode_step_ex(d, *tok, g["D"], ex, st, y, stream=None)
        elif gated:
            m3.m3_decode_step_gated(d, *tok, g["D"], z[t], st, y, stream=None)
        else:
            m3.m3_decode_step(d, *tok, g["D"], st, y, stream=None)

    def reset():
        st.h.copy_(g["h0"])
        st.x_prev.copy_(g["x_prev"])
        st.B_prev.copy_(g["B_prev"])

    reset()
    for t in range(10):
        step(t)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for t in range(tokens):
            step(t)
    reset()
    graph.replay()                      # warm-up replay
    reset()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    e0.record(cur)
    graph.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / tokens
    del graph
    if torch.equal(st.h, g["h0"]):
        raise RuntimeError("decode graph replay left the state unchanged")
    finite = bool(torch.isfinite(st.h).all().item())
    byts = decode_algorithmic(w) + (w.batch * w.nheads * w.rank * w.headdim * 2 if gated else 0)
    del g, z
    return {"tokens_per_s": w.batch / (ms / 1e3), "us_per_step": ms * 1e3,
            "achieved_gbs": byts / (ms / 1e3) / 1e9, "alg_bytes_per_step": byts,
            "state_finite": finite,
            "config": {"batch": w.batch, "heads": w.nheads, "headdim": w.headdim,
                       "dstate": w.dstate, "rank": w.rank, "tokens": tokens,
                       "distinct_tokens": tokens}}


def mimo_leg(args, dev, stream, rank, ws_world, pk):
    """The MIMO prefill workload (rank 4, N 64, 32-token tiles): plain, with the
    lightweight expansion of x (x read as [b][T][H][P]), and with the expansion of x and z
    plus the fused gate; then its backward pass (16-token chunks of 64 (token, rank) rows).
    Algorithmic bytes count each tensor as the call reads it."""
    w = inputs.WORKLOADS["mimo_prefill_r4"]
    if args.batch or args.seqlen:   # profiler captures only, as for the prefill line
        w = dataclasses.replace(w, batch=args.batch or w.batch, seqlen=args.seqlen or w.seqlen)
    inp, d, g, st, y, ws = prefill_setup(w, dev, seed=200 + rank)
    del inp
    byts, _ = scan_algorithmic(w)
    b, T, H, R, P = w.batch, w.seqlen, w.nheads, w.rank, w.headdim
    xio = b * T * H * P * 2                      # one bf16 value per head channel and token
    x1 = g["x"][:, :, :, 0, :].contiguous()
    wx, wz = (v.to(dev) for v in inputs.make_expand(H, R, P, seed=200 + rank))
    z1 = inputs.make_gate((b, T, H, P), io_dtype=w.io_dtype, seed=200 + rank).to(dev)
    legs = (("prefill", g["x"], None, byts),
            ("prefill_expanded", x1, m3.Extras(x_expand=wx), byts - xio * (R - 1)),
            ("prefill_expanded_gated", x1, m3.Extras(z=z1, x_expand=wx, z_expand=wz),
             byts - xio * (R - 1) + xio))
    out = {}
    for key, x, ex, nbytes in legs:
        gx = dict(g)
        gx["x"] = x
        ms = time_prefill_ex(w, d, gx, ex, st, y, ws, min(args.steps, 20), 3, stream)
        val, ms_max = job_throughput(b * T, ms, ws_world)
        gbs = nbytes / (ms / 1e3) / 1e9
        out[key] = {"tokens_per_s": val, "ms_per_step": ms_max, "alg_bytes_per_step": nbytes,
                    "achieved_gbs": gbs, "hbm_frac": gbs / pk["hbm_gbs"]}
    if not args.no_bwd:
        out["backward"] = backward_leg(args, w, d, g, dev, stream, rank, ws_world, pk)
    out["config"] = {"workload": w.name, "batch": b, "heads": H, "seqlen": T, "headdim": P,
                     "dstate": w.dstate, "rank": R, "chunk": w.chunk}
    return out


def backward_leg(args, w, d, g, dev, stream, rank, ws_world, pk):
    """The backward pass (m3_scan_bwd) of the prefill workload: gradients of every input and
    of the starting state for a random dL/dy, inputs resident in HBM.  Algorithmic bytes: the
    forward inputs and dy read once, the fp32 gradients and dh0 written once."""
    T = w.seqlen
    st = m3.State(d, dev)
    m3.m3_state_init(d, st, stream=stream)
    gen = torch.Generator().manual_seed(300 + rank)
    dy = torch.randn(g["x"].shape, generator=gen).to(w.io_dtype).to(dev)
    gr = m3.alloc_grads(d, T, dev)
    ws = m3.alloc_bwd_workspace(d, T, dev)

    def run():
        m3.m3_scan_bwd(d, T, g["x"], g["B"], g["C"], g["dt"], g["A"], g["lam"], g["theta"],
                       g["D"], st, dy, None, gr, ws, stream=stream)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 3))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    if m3.m3_query_status(ws, stream) != m3.M3_OK:
        raise RuntimeError("backward: device status not OK")
    ms = e0.elapsed_time(e1) / steps
    b, H, G, P, N, R = w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank
    e = 2
    reads = b * T * (2 * H * R * P * e + 12 * H + G * (2 * R * N * e + 2 * N)) + b * H * N * P * 4
    writes = sum(v.numel() * 4 for v in gr.values())
    val, ms_max = job_throughput(b * T, ms, ws_world)
    gbs = (reads + writes) / (ms / 1e3) / 1e9
    del ws, gr, dy
    return {"tokens_per_s": val, "ms_per_step": ms_max, "alg_bytes_per_step": reads + writes,
            "achieved_gbs": gbs, "hbm_frac": gbs / pk["hbm_gbs"], "steps": steps,
            "kernel": "chunked tensor-core backward: bwd_vu_kernel (chunk products), "
                      "bwd_scan_kernel (chunk states and adjoints), bwd_grads_kernel "
                      "(chunk gradients), bwd_finish_kernel (angle carries)"}


def longctx_leg(args, dev, stream, rank, ws_world, pk):
    """The long-context workload: batch 1, 64 heads, 65536 tokens as 16 chained calls of 4096
    (state and previous token carried from call to call), chunk 128, fast rotation.  One step
    is the 16 calls; the state is reset outside the timed interval."""
    w = inputs.WORKLOADS["siso_longctx_carry"]
    Tc = w.seqlen // w.calls
    inp = inputs.make_scan_inputs(w.batch, w.seqlen, w.nheads, w.ngroups, w.headdim, w.dstate,
                                  w.rank, io_dtype=w.io_dtype, theta_max=w.theta_max,
                                  seed=400 + rank)
    d = m3.Dims(w.batch, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                m3.io_dtype_of(w.io_dtype))
    keys = ("x", "B", "C", "dt", "A", "lam", "theta")
    calls = [{k: inp[k][:, c * Tc:(c + 1) * Tc].contiguous().to(dev) for k in keys}
             for c in range(w.calls)]
    D = inp["D"].to(dev)
    del inp
    st = m3.State(d, dev)
    ys = [torch.empty_like(c["x"]) for c in calls]
    ws = m3.alloc_workspace(d, Tc, w.chunk, dev)

    def run():
        for c, y in zip(calls, ys):
            m3.m3_scan_fwd(d, Tc, w.chunk, c["x"], c["B"], c["C"], c["dt"], c["A"], c["lam"],
                           c["theta"], D, st, y, ws, stream=stream)
    for _ in range(3):
        m3.m3_state_init(d, st, stream=stream)
        run()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 10))
    per = []
    for _ in range(steps):
        m3.m3_state_init(d, st, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        per.append((e0, e1))
    torch.cuda.synchronize()
    if m3.m3_query_status(ws, stream) != m3.M3_OK:
        raise RuntimeError("longctx: device status not OK")
    ms = sum(a.elapsed_time(b) for a, b in per) / steps
    # bytes and flops per call; flops of the contractions as run: with N = 128 the kernel
    # runs chunk 128 as 64-token tiles
    wc = dataclasses.replace(w, seqlen=Tc, chunk=64 if w.dstate == 128 else w.chunk)
    byts, flops = scan_algorithmic(wc)
    byts, flops = byts * w.calls, flops * w.calls
    val, ms_max = job_throughput(w.batch * w.seqlen, ms, ws_world)
    gbs = byts / (ms / 1e3) / 1e9
    return {"tokens_per_s": val, "ms_per_step": ms_max, "calls_per_step": w.calls,
            "alg_bytes_per_step": byts, "achieved_gbs": gbs, "hbm_frac": gbs / pk["hbm_gbs"],
            "tensor_frac": flops / (ms / 1e3) / 1e12 / pk["bf16_tflops"],
            "config": {"workload": w.name, "batch": w.batch, "heads": w.nheads,
                       "seqlen": w.seqlen, "calls": w.calls, "headdim": w.headdim,
                       "dstate": w.dstate, "chunk": w.chunk, "theta_max": w.theta_max}}


def small_f32_leg(args, dev, stream, rank, ws_world):
    """The fp32 parity workload (batch 1, 2 heads, T 256, P 16, N 16): the sequential fp32
    CUDA-core kernel; latency-bound by design (one call is a few microseconds of work)."""
    w = inputs.WORKLOADS["siso_f32_small"]
    inp, d, g, st, y, ws = prefill_setup(w, dev, seed=500 + rank)
    del inp
    for _ in range(5):
        m3.m3_state_init(d, st, stream=stream)
        run_scan(w, d, g, st, y, ws, stream)
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 50))
    per = []
    for _ in range(steps):
        m3.m3_state_init(d, st, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run_scan(w, d, g, st, y, ws, stream)
        e1.record(stream)
        per.append((e0, e1))
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in per) / steps
    val, ms_max = job_throughput(w.batch * w.seqlen, ms, ws_world)
    return {"tokens_per_s": val, "us_per_call": ms_max * 1e3, "kernel": "scan_simt_kernel (fp32)",
            "config": {"workload": w.name, "batch": w.batch, "heads": w.nheads,
                       "seqlen": w.seqlen, "headdim": w.headdim, "dstate": w.dstate,
                       "chunk": w.chunk, "io": "fp32"}}


def w_dec_batch(name):
    return inputs.WORKLOADS[name].batch


def oracle_workload(w, inp, rows):
    """Time the CPU oracle on the first `rows` batch rows of the workload's own inputs (all
    heads, all tokens), one row per call so that host memory stays bounded."""
    import oracle
    threads = min(oracle.max_threads(), w.nheads)
    secs = 0.0
    for b in range(rows):
        arr = {k: inp[k][b:b + 1].double().numpy() for k in ("x", "B", "C", "dt", "A", "lam",
                                                              "theta")}
        D = inp["D"].double().numpy()
        t0 = time.perf_counter()
        oracle.scan(arr["x"], arr["B"], arr["C"], arr["dt"], arr["A"], arr["lam"], arr["theta"],
                    D=D, nthreads=threads)
        secs += time.perf_counter() - t0
    return rows * w.seqlen / secs, threads, secs


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_one_thread(w, inp):
    """The CPU oracle on one (batch, head) slice of the workload (batch row 0, head 0, all
    tokens) on a single thread: tokens per second of one sequential recurrence."""
    import oracle
    keys = ("x", "B", "C", "dt", "A", "lam", "theta")
    arr = {k: inp[k][:1].double().numpy() for k in keys}
    for k in ("x", "dt", "A", "lam"):
        arr[k] = arr[k][:, :, :1].copy()
    for k in ("B", "C", "theta"):
        arr[k] = arr[k][:, :, :1].copy()   # head 0 reads group 0
    D = inp["D"][:1].double().numpy()
    t0 = time.perf_counter()
    oracle.scan(*(arr[k] for k in keys), D=D, nthreads=1)
    secs = time.perf_counter() - t0
    return w.seqlen / secs, secs


def oracle_sample(w, seqlen, seed=0):
    """Time the CPU oracle on batch row 0, all heads, the first `seqlen` tokens."""
    import oracle
    inp = inputs.make_scan_inputs(1, seqlen, w.nheads, w.ngroups, w.headdim, w.dstate, w.rank,
                                  io_dtype=w.io_dtype, theta_max=w.theta_max, seed=seed)
    arr = {k: inp[k].double().numpy() for k in ("x", "B", "C", "dt", "A", "lam", "theta", "D")}
    threads = min(oracle.max_threads(), w.nheads)
    t0 = time.perf_counter()
    oracle.scan(arr["x"], arr["B"], arr["C"], arr["dt"], arr["A"], arr["lam"], arr["theta"],
                D=arr["D"], nthreads=threads)
    dt = time.perf_counter() - t0
    return seqlen / dt, threads, dt


def ours(args):
    ws_world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    w = inputs.WORKLOADS[WORKLOAD]
    if args.batch or args.seqlen:
        # a smaller case of the same workload: only for short profiler captures
        w = dataclasses.replace(w, batch=args.batch or w.batch, seqlen=args.seqlen or w.seqlen)
    pk, pk_kind = peaks()

    inp, d, g, st, y, ws = prefill_setup(w, dev, seed=rank)
    with ClockSampler(local) as clk:
        ms, status = time_prefill(w, d, g, st, y, ws, args.steps, args.warmup, stream, ws_world)
    if status != m3.M3_OK:
        raise RuntimeError(f"device status {m3.m3_status_string(status)}")
    tokens = w.batch * w.seqlen
    value, ms_max = job_throughput(tokens, ms, ws_world)
    byts, flops = scan_algorithmic(w)
    achieved = byts / (ms / 1e3) / 1e9
    tflops = flops / (ms / 1e3) / 1e12
    kernel_src = os.path.join(ROOT, "state_space_model_06_b200", "csrc", "scan_tc.cu")
    # the committed counters describe the current kernel on the full workload only
    counters = {} if (args.batch or args.seqlen) else committed_counters(kernel_src, WORKLOAD)
    traffic = counters.get("dram_bytes_per_launch")

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of a 1.5B-scale Mamba-3 layer)",
        "config": {"workload": WORKLOAD, "batch": w.batch, "heads": w.nheads,
                   "groups": w.ngroups, "seqlen": w.seqlen, "headdim": w.headdim,
                   "dstate": w.dstate, "rank": w.rank, "chunk": w.chunk,
                   "io": "bf16 x/B/C/y, fp32 dt/A/lam/theta/state",
                   "l2": f"inputs larger than L2 ({byts / 1e6:.0f} MB touched per step)",
                   "parallelism": f"replicas x{ws_world} (independent (batch, head) work)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                     "peak_source": pk_kind, "kernel": "scan_tc_kernel<128,64,1>",
                     "alg_bytes_per_launch": byts,
                     "tensor": {"achieved_tflops": tflops, "peak_tflops": pk["bf16_tflops"],
                                "frac": tflops / pk["bf16_tflops"],
                                "alg_flops_per_launch": flops,
                                "pipe_active_ncu_pct": counters.get("tensor_pipe_active_pct"),
                                "pipe_active_ncu_how": counters.get("tensor_pipe_how")}},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }

    if args.prefill_only or args.bwd_only or args.mimo_only:
        args.no_decode = args.no_e2e = args.no_cpu = args.no_gate = args.no_mimo = True
        args.no_bwd = args.no_longctx = True
        args.no_bwd = not (args.bwd_only or args.mimo_only)
        args.no_mimo = not args.mimo_only
    if not args.no_decode:
        line["decode"] = {}
        for name in (args.decode or DECODES):
            r = time_decode(name, dev, stream, seed=100 + rank, tokens=args.decode_tokens)
            r["hbm_frac"] = r["achieved_gbs"] / pk["hbm_gbs"]
            r["tokens_per_s"], _ = job_throughput(w_dec_batch(name), r["us_per_step"] / 1e3,
                                                  ws_world)
            line["decode"][name] = r

    if not args.no_gate:
        # the fused output gate (y * SiLU(z)): the same prefill step plus z read once
        z = inputs.make_gate(g["x"].shape, io_dtype=w.io_dtype, seed=rank).to(dev)
        gms = time_prefill_ex(w, d, g, m3.Extras(z=z), st, y, ws, min(args.steps, 20), 3, stream)
        gval, gms_max = job_throughput(tokens, gms, ws_world)
        gbytes = byts + z.numel() * z.element_size()
        line["gated"] = {"prefill": {"tokens_per_s": gval, "ms_per_step": gms_max,
                                     "alg_bytes_per_step": gbytes,
                                     "achieved_gbs": gbytes / (gms / 1e3) / 1e9,
                                     "hbm_frac": gbytes / (gms / 1e3) / 1e9 / pk["hbm_gbs"]}}
        del z
        if not args.no_decode:
            for name in (args.decode or DECODES):
                r = time_decode(name, dev, stream, seed=100 + rank, tokens=args.decode_tokens,
                                gated=True)
                r["hbm_frac"] = r["achieved_gbs"] / pk["hbm_gbs"]
                r["tokens_per_s"], _ = job_throughput(w_dec_batch(name), r["us_per_step"] / 1e3,
                                                      ws_world)
                line["gated"][name] = r

    if not args.no_gate:
        # BCNorm + BC biases (and everything fused at once: norm, biases and the gate)
        bb, cb = (v.to(dev) for v in inputs.make_bc_bias(w.nheads, w.dstate, seed=rank))
        line["bc"] = {}
        zfull = inputs.make_gate(g["x"].shape, io_dtype=w.io_dtype, seed=rank).to(dev)
        for key, ex in (("prefill", m3.Extras(B_bias=bb, C_bias=cb, bc_norm_eps=BC_EPS)),
                        ("prefill_all", m3.Extras(z=zfull, B_bias=bb, C_bias=cb,
                                                  bc_norm_eps=BC_EPS))):
            wsx = m3.alloc_workspace_ex(d, w.seqlen, w.chunk, ex, dev)
            bms = time_prefill_ex(w, d, g, ex, st, y, wsx, min(args.steps, 20), 3, stream)
            bval, bms_max = job_throughput(tokens, bms, ws_world)
            line["bc"][key] = {"tokens_per_s": bval, "ms_per_step": bms_max}
            del wsx
        del zfull
        if not args.no_decode:
            for name in (args.decode or DECODES):
                r = time_decode(name, dev, stream, seed=100 + rank, tokens=args.decode_tokens,
                                bc=True)
                r["hbm_frac"] = r["achieved_gbs"] / pk["hbm_gbs"]
                r["tokens_per_s"], _ = job_throughput(w_dec_batch(name), r["us_per_step"] / 1e3,
                                                      ws_world)
                line["bc"][name] = r

    if not args.no_mimo:
        line["mimo"] = mimo_leg(args, dev, stream, rank, ws_world, pk)

    if not args.no_longctx:
        line["longctx"] = longctx_leg(args, dev, stream, rank, ws_world, pk)
        line["small_f32"] = small_f32_leg(args, dev, stream, rank, ws_world)

    if not args.no_bwd and not args.mimo_only:
        line["backward"] = backward_leg(args, w, d, g, dev, stream, rank, ws_world, pk)

    if not args.no_e2e:
        e2e_ms, h2d, d2h, e2e_slices = time_prefill_e2e(w, d, inp, st, ws, min(args.steps, 5),
                                                        stream, dev)
        e2e_value, e2e_ms = job_throughput(tokens, e2e_ms, ws_world)
        line["e2e"] = {"value": e2e_value, "unit": "tokens/s",
                       "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h,
                       "how": f"{e2e_slices} batch-row slices pipelined over three streams "
                              "(H2D, call, D2H overlap)"}

    if rank == 0 and ws_world == 1 and not args.no_cpu:
        rows = max(1, min(args.cpu_rows, w.batch))
        tps, cores, secs = oracle_workload(w, inp, rows)
        one_tps, one_secs = oracle_one_thread(w, inp)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"the workload's own inputs, batch rows 0..{rows - 1} of "
                                          f"{w.batch}, all {w.nheads} heads and {w.seqlen} tokens "
                                          f"({secs:.1f} s of fp64 CPU work)",
                                "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                                "one_thread": {"value": one_tps, "unit": "tokens/s per (batch, head)",
                                               "sample": f"batch row 0, head 0, {w.seqlen} tokens, "
                                                         f"1 thread ({one_secs:.2f} s)"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- reference arm
def reference(args):
    rank = int(os.environ.get("RANK", "0"))
    ws_world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = inputs.WORKLOADS[WORKLOAD]
    for _ in range(args.warmup):
        oracle_sample(w, args.ref_tokens, seed=1)
    times = []
    cores = 0
    for _ in range(args.steps):
        _, cores, secs = oracle_sample(w, args.ref_tokens, seed=1)
        times.append(secs)
    sec = sum(times) / len(times)
    value = args.ref_tokens / sec
    sample = (f"each step: batch row 0, all {w.nheads} heads, first {args.ref_tokens} of "
              f"{w.seqlen} tokens of the workload")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": ws_world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": w.batch, "heads": w.nheads,
                       "groups": w.ngroups, "seqlen": w.seqlen, "headdim": w.headdim,
                       "dstate": w.dstate, "rank": w.rank, "chunk": w.chunk},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-gate", action="store_true", help="skip the fused-output-gate legs")
    ap.add_argument("--no-mimo", action="store_true", help="skip the MIMO prefill legs")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward-pass leg")
    ap.add_argument("--no-longctx", action="store_true",
                    help="skip the long-context and fp32 small-workload legs")
    ap.add_argument("--cpu-rows", type=int, default=8,
                    help="batch rows of the workload timed on the CPU oracle (default: all)")
    ap.add_argument("--ref-tokens", type=int, default=256)
    ap.add_argument("--decode", action="append", choices=DECODES,
                    help="time only these decode workloads (profiling)")
    ap.add_argument("--decode-tokens", type=int, default=DECODE_TOKENS,
                    help="sequential decode tokens timed per workload")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling only)")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the sequence length (profiling only)")
    ap.add_argument("--prefill-only", action="store_true", help="skip decode, e2e and CPU legs")
    ap.add_argument("--bwd-only", action="store_true",
                    help="the prefill line and the backward leg only (profiling)")
    ap.add_argument("--mimo-only", action="store_true",
                    help="the prefill line and the MIMO leg (prefill and backward) only (profiling)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
