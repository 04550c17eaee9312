"""Thin ctypes binding of the C ABI in ``include/m3.h`` (libm3.so, built in-tree).

The functions keep the C names and only marshal arguments: torch tensors become
device pointers, dims become an ``m3_dims`` struct, the current torch stream is
passed as the cudaStream_t.  Every step of the computation runs in the CUDA
kernels of libm3.so; there is no fallback of any kind -- if the library is
missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, replace

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libm3.so")

M3_OK, M3_ERR_NULL, M3_ERR_SHAPE, M3_ERR_DTYPE, M3_ERR_ALIGN, M3_ERR_UNSUPPORTED, \
    M3_ERR_WORKSPACE, M3_ERR_LAUNCH, M3_ERR_TIMEOUT, M3_ERR_CUDA, M3_ERR_RANGE = range(11)
M3_F32, M3_BF16 = 0, 1
M3_FLAG_THETA_IS_ANGLE = 1
M3_FLAG_FORCE_SIMT = 2
M3_FLAG_TEST_STALL = 4
M3_FLAG_DEBUG_CHECKS = 8

EXPORTED = ("m3_state_bytes", "m3_state_init", "m3_scan_workspace_bytes", "m3_scan_fwd",
            "m3_decode_step", "m3_query_status", "m3_scan_fwd_noalloc", "m3_scan_fwd_gated",
            "m3_decode_step_gated", "m3_scan_workspace_bytes_ex", "m3_scan_fwd_ex",
            "m3_decode_step_ex", "m3_scan_bwd_workspace_bytes", "m3_scan_bwd",
            "m3_scan_bwd_workspace_bytes_ex", "m3_scan_bwd_ex", "m3_status_string")


class M3Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {m3_status_string(status)} (status {status})")


class m3_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("nheads", ctypes.c_int32),
                ("ngroups", ctypes.c_int32), ("headdim", ctypes.c_int32),
                ("dstate", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("io_dtype", ctypes.c_int32)]


class m3_state(ctypes.Structure):
    _fields_ = [("h", ctypes.c_void_p), ("x_prev", ctypes.c_void_p), ("B_prev", ctypes.c_void_p)]


class m3_grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dx", "dB", "dC", "ddt", "dA", "dlam", "dtheta",
                                               "dD", "dh0", "dx_prev", "dB_prev")]


class m3_extra_grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dz", "dB_bias", "dC_bias", "dx_expand",
                                                "dz_expand")]


class m3_extras(ctypes.Structure):
    _fields_ = [("z", ctypes.c_void_p), ("B_bias", ctypes.c_void_p), ("C_bias", ctypes.c_void_p),
                ("bc_norm_eps", ctypes.c_float), ("x_expand", ctypes.c_void_p),
                ("z_expand", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libm3.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path} (run __graft_entry__.build())")
        lib = ctypes.CDLL(path)
        vp, u32, i32, sz = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_int32, ctypes.c_size_t
        dp = ctypes.POINTER(m3_dims)
        sp = ctypes.POINTER(m3_state)
        szp = ctypes.POINTER(ctypes.c_size_t)
        lib.m3_state_bytes.argtypes = [dp, szp, szp, szp]
        lib.m3_state_init.argtypes = [dp, sp, vp, vp]
        lib.m3_scan_workspace_bytes.argtypes = [dp, i32, i32, szp]
        lib.m3_scan_fwd.argtypes = [dp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sp, vp, vp, sz,
                                    u32, vp]
        lib.m3_decode_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, sp, vp, u32, vp]
        lib.m3_scan_fwd_gated.argtypes = [dp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sp,
                                          vp, vp, sz, u32, vp]
        lib.m3_decode_step_gated.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sp, vp,
                                             u32, vp]
        ep = ctypes.POINTER(m3_extras)
        lib.m3_scan_workspace_bytes_ex.argtypes = [dp, i32, i32, ep, szp]
        lib.m3_scan_fwd_ex.argtypes = [dp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, ep, sp, vp,
                                       vp, sz, u32, vp]
        lib.m3_decode_step_ex.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, ep, sp, vp, u32, vp]
        lib.m3_scan_fwd_noalloc.argtypes = [dp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sp, vp,
                                            u32, vp]
        lib.m3_scan_bwd_workspace_bytes.argtypes = [dp, i32, szp]
        lib.m3_scan_bwd.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sp, vp, vp,
                                    ctypes.POINTER(m3_grads), vp, sz, u32, vp]
        lib.m3_scan_bwd_workspace_bytes_ex.argtypes = [dp, i32, ep, szp]
        lib.m3_scan_bwd_ex.argtypes = [dp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sp, ep, vp, vp,
                                       ctypes.POINTER(m3_grads), ctypes.POINTER(m3_extra_grads),
                                       vp, sz, u32, vp]
        lib.m3_query_status.argtypes = [vp, vp]
        lib.m3_status_string.argtypes = [ctypes.c_int]
        lib.m3_status_string.restype = ctypes.c_char_p
        for name in EXPORTED[:-1]:
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


@dataclass
class Dims:
    batch: int
    nheads: int
    ngroups: int
    headdim: int
    dstate: int
    rank: int = 1
    io_dtype: int = M3_BF16

    def c(self) -> m3_dims:
        return m3_dims(self.batch, self.nheads, self.ngroups, self.headdim, self.dstate,
                       self.rank, self.io_dtype)


def io_dtype_of(t: torch.dtype) -> int:
    return {torch.bfloat16: M3_BF16, torch.float32: M3_F32}[t]


def torch_dtype_of(io: int) -> torch.dtype:
    return {M3_BF16: torch.bfloat16, M3_F32: torch.float32}[io]


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != M3_OK:
        raise M3Error(status, where)


def m3_status_string(status: int) -> str:
    return load_library().m3_status_string(int(status)).decode()


class State:
    """Caller-owned resumable state (h fp32, previous token's x and B in io dtype)."""

    def __init__(self, dims: Dims, device="cuda"):
        io = torch_dtype_of(dims.io_dtype)
        self.dims = dims
        self.h = torch.zeros(dims.batch, dims.nheads, dims.dstate, dims.headdim,
                             dtype=torch.float32, device=device)
        self.x_prev = torch.zeros(dims.batch, dims.nheads, dims.rank, dims.headdim, dtype=io,
                                  device=device)
        self.B_prev = torch.zeros(dims.batch, dims.ngroups, dims.rank, dims.dstate, dtype=io,
                                  device=device)

    def c(self) -> m3_state:
        return m3_state(self.h.data_ptr(), self.x_prev.data_ptr(), self.B_prev.data_ptr())

    def rows(self, lo: int, hi: int) -> "State":
        """Batch rows [lo, hi) of this state (the same memory), for a call on a slice of
        the batch: every tensor of the state leads with the batch axis."""
        v = State.__new__(State)
        v.dims = replace(self.dims, batch=hi - lo)
        v.h, v.x_prev, v.B_prev = self.h[lo:hi], self.x_prev[lo:hi], self.B_prev[lo:hi]
        return v


def m3_state_bytes(dims: Dims):
    h, x, b = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().m3_state_bytes(ctypes.byref(dims.c()), ctypes.byref(h), ctypes.byref(x),
                                         ctypes.byref(b)), "m3_state_bytes")
    return h.value, x.value, b.value


def m3_state_init(dims: Dims, state: State, h0=None, stream=None):
    st = state.c()
    _check(load_library().m3_state_init(ctypes.byref(dims.c()), ctypes.byref(st), _ptr(h0),
                                        _stream(stream)), "m3_state_init")


def m3_scan_workspace_bytes(dims: Dims, seqlen: int, chunk: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().m3_scan_workspace_bytes(ctypes.byref(dims.c()), int(seqlen), int(chunk),
                                                  ctypes.byref(n)), "m3_scan_workspace_bytes")
    return n.value


def m3_scan_fwd(dims: Dims, seqlen: int, chunk: int, x, B, C, dt, A, lam, theta, D,
                state: State, y, workspace, flags: int = 0, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = state.c()
    _check(load_library().m3_scan_fwd(
        ctypes.byref(dims.c()), int(seqlen), int(chunk), _ptr(x), _ptr(B), _ptr(C), _ptr(dt),
        _ptr(A), _ptr(lam), _ptr(theta), _ptr(D), ctypes.byref(st), _ptr(y), _ptr(workspace),
        ws_bytes, int(flags), _stream(stream)), "m3_scan_fwd")


def m3_scan_fwd_noalloc(dims: Dims, seqlen: int, chunk: int, x, B, C, dt, A, lam, theta, D,
                        state: State, y, flags: int = 0, stream=None):
    """Prefill for callers that cannot allocate device memory: no workspace argument;
    the library lends its own fixed scratch (see include/m3.h)."""
    st = state.c()
    _check(load_library().m3_scan_fwd_noalloc(
        ctypes.byref(dims.c()), int(seqlen), int(chunk), _ptr(x), _ptr(B), _ptr(C), _ptr(dt),
        _ptr(A), _ptr(lam), _ptr(theta), _ptr(D), ctypes.byref(st), _ptr(y), int(flags),
        _stream(stream)), "m3_scan_fwd_noalloc")


def m3_scan_fwd_gated(dims: Dims, seqlen: int, chunk: int, x, B, C, dt, A, lam, theta, D, z,
                      state: State, y, workspace, flags: int = 0, stream=None):
    """Prefill with the fused output gate y * SiLU(z) (z in the layout and dtype of y)."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = state.c()
    _check(load_library().m3_scan_fwd_gated(
        ctypes.byref(dims.c()), int(seqlen), int(chunk), _ptr(x), _ptr(B), _ptr(C), _ptr(dt),
        _ptr(A), _ptr(lam), _ptr(theta), _ptr(D), _ptr(z), ctypes.byref(st), _ptr(y),
        _ptr(workspace), ws_bytes, int(flags), _stream(stream)), "m3_scan_fwd_gated")


@dataclass
class Extras:
    """Optional fused parts (see m3_extras in include/m3.h): output gate z, BC biases
    B_bias / C_bias [H][N] fp32, BCNorm epsilon (0: off), MIMO lightweight expansion
    weights x_expand / z_expand [H][R][P] fp32 (x, z then hold [..][H][P])."""
    z: object = None
    B_bias: object = None
    C_bias: object = None
    bc_norm_eps: float = 0.0
    x_expand: object = None
    z_expand: object = None

    def c(self) -> m3_extras:
        return m3_extras(_ptr(self.z), _ptr(self.B_bias), _ptr(self.C_bias),
                         float(self.bc_norm_eps), _ptr(self.x_expand), _ptr(self.z_expand))


def _ex_ref(ex):
    return ctypes.byref(ex.c()) if ex is not None else None


def m3_scan_workspace_bytes_ex(dims: Dims, seqlen: int, chunk: int, ex) -> int:
    n = ctypes.c_size_t()
    _check(load_library().m3_scan_workspace_bytes_ex(ctypes.byref(dims.c()), int(seqlen),
                                                     int(chunk), _ex_ref(ex), ctypes.byref(n)),
           "m3_scan_workspace_bytes_ex")
    return n.value


def m3_scan_fwd_ex(dims: Dims, seqlen: int, chunk: int, x, B, C, dt, A, lam, theta, D, ex,
                   state: State, y, workspace, flags: int = 0, stream=None):
    """Prefill with the optional fused parts in ``ex`` (an Extras, or None)."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = state.c()
    _check(load_library().m3_scan_fwd_ex(
        ctypes.byref(dims.c()), int(seqlen), int(chunk), _ptr(x), _ptr(B), _ptr(C), _ptr(dt),
        _ptr(A), _ptr(lam), _ptr(theta), _ptr(D), _ex_ref(ex), ctypes.byref(st), _ptr(y),
        _ptr(workspace), ws_bytes, int(flags), _stream(stream)), "m3_scan_fwd_ex")


def m3_decode_step_ex(dims: Dims, x, B, C, dt, A, lam, theta, D, ex, state: State, y,
                      flags: int = 0, stream=None):
    """Decode step with the optional fused parts in ``ex`` (an Extras, or None)."""
    st = state.c()
    _check(load_library().m3_decode_step_ex(
        ctypes.byref(dims.c()), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam),
        _ptr(theta), _ptr(D), _ex_ref(ex), ctypes.byref(st), _ptr(y), int(flags),
        _stream(stream)), "m3_decode_step_ex")


def alloc_workspace_ex(dims: Dims, seqlen: int, chunk: int, ex, device="cuda") -> torch.Tensor:
    """A workspace tensor of the size m3_scan_fwd_ex needs with these extras."""
    n = m3_scan_workspace_bytes_ex(dims, seqlen, chunk, ex)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def m3_decode_step_gated(dims: Dims, x, B, C, dt, A, lam, theta, D, z, state: State, y,
                         flags: int = 0, stream=None):
    """Decode step with the fused output gate y * SiLU(z)."""
    st = state.c()
    _check(load_library().m3_decode_step_gated(
        ctypes.byref(dims.c()), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam),
        _ptr(theta), _ptr(D), _ptr(z), ctypes.byref(st), _ptr(y), int(flags), _stream(stream)),
        "m3_decode_step_gated")


def m3_decode_step(dims: Dims, x, B, C, dt, A, lam, theta, D, state: State, y, flags: int = 0,
                   stream=None):
    st = state.c()
    _check(load_library().m3_decode_step(
        ctypes.byref(dims.c()), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(lam),
        _ptr(theta), _ptr(D), ctypes.byref(st), _ptr(y), int(flags), _stream(stream)),
        "m3_decode_step")


def m3_query_status(workspace, stream=None) -> int:
    """Synchronise the stream and return the device-side status word (M3_OK, M3_ERR_TIMEOUT or
    M3_ERR_RANGE)."""
    return int(load_library().m3_query_status(_ptr(workspace), _stream(stream)))


def alloc_workspace(dims: Dims, seqlen: int, chunk: int, device="cuda") -> torch.Tensor:
    """A workspace tensor of the size m3_scan_fwd needs (256-byte aligned by torch)."""
    n = m3_scan_workspace_bytes(dims, seqlen, chunk)
    return torch.zeros(n, dtype=torch.uint8, device=device)


GRAD_NAMES = ("dx", "dB", "dC", "ddt", "dA", "dlam", "dtheta", "dD", "dh0", "dx_prev", "dB_prev")


def alloc_grads(dims: Dims, seqlen: int, device="cuda") -> dict:
    """fp32 gradient tensors of m3_scan_bwd, in its layouts."""
    b, H, G, P, N, R, T = (dims.batch, dims.nheads, dims.ngroups, dims.headdim, dims.dstate,
                           dims.rank, seqlen)
    f = dict(dtype=torch.float32, device=device)
    return dict(dx=torch.empty(b, T, H, R, P, **f), dB=torch.empty(b, T, G, R, N, **f),
                dC=torch.empty(b, T, G, R, N, **f), ddt=torch.empty(b, T, H, **f),
                dA=torch.empty(b, T, H, **f), dlam=torch.empty(b, T, H, **f),
                dtheta=torch.empty(b, T, G, N // 2, **f), dD=torch.empty(H, **f),
                dh0=torch.empty(b, H, N, P, **f), dx_prev=torch.empty(b, H, R, P, **f),
                dB_prev=torch.empty(b, G, R, N, **f))


def m3_scan_bwd_workspace_bytes(dims: Dims, seqlen: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().m3_scan_bwd_workspace_bytes(ctypes.byref(dims.c()), int(seqlen),
                                                      ctypes.byref(n)),
           "m3_scan_bwd_workspace_bytes")
    return n.value


def alloc_bwd_workspace(dims: Dims, seqlen: int, device="cuda") -> torch.Tensor:
    return torch.zeros(m3_scan_bwd_workspace_bytes(dims, seqlen), dtype=torch.uint8,
                       device=device)


def m3_scan_bwd(dims: Dims, seqlen: int, x, B, C, dt, A, lam, theta, D, state0: State, dy,
                dhT, grads: dict, workspace, flags: int = 0, stream=None):
    """Backward pass of m3_scan_fwd: gradients into ``grads`` (see alloc_grads); state0 is
    the state the forward call started from (read only); dhT may be None."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = state0.c()
    g = m3_grads(*(_ptr(grads.get(k)) for k in GRAD_NAMES))
    _check(load_library().m3_scan_bwd(
        ctypes.byref(dims.c()), int(seqlen), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A),
        _ptr(lam), _ptr(theta), _ptr(D), ctypes.byref(st), _ptr(dy), _ptr(dhT), ctypes.byref(g),
        _ptr(workspace), ws_bytes, int(flags), _stream(stream)), "m3_scan_bwd")


EXTRA_GRAD_NAMES = ("dz", "dB_bias", "dC_bias", "dx_expand", "dz_expand")


def alloc_extra_grads(dims: Dims, seqlen: int, ex, device="cuda") -> dict:
    """fp32 gradient tensors of the parts of ``ex`` (an Extras) that are on."""
    b, H, P, N, R, T = dims.batch, dims.nheads, dims.headdim, dims.dstate, dims.rank, seqlen
    f = dict(dtype=torch.float32, device=device)
    out = {}
    if ex.z is not None:
        out["dz"] = torch.empty((b, T, H, P) if ex.z_expand is not None else (b, T, H, R, P), **f)
    if ex.B_bias is not None:
        out["dB_bias"] = torch.empty(H, N, **f)
    if ex.C_bias is not None:
        out["dC_bias"] = torch.empty(H, N, **f)
    if ex.x_expand is not None:
        out["dx_expand"] = torch.empty(H, R, P, **f)
    if ex.z_expand is not None:
        out["dz_expand"] = torch.empty(H, R, P, **f)
    return out


def m3_scan_bwd_workspace_bytes_ex(dims: Dims, seqlen: int, ex) -> int:
    n = ctypes.c_size_t()
    _check(load_library().m3_scan_bwd_workspace_bytes_ex(ctypes.byref(dims.c()), int(seqlen),
                                                         _ex_ref(ex), ctypes.byref(n)),
           "m3_scan_bwd_workspace_bytes_ex")
    return n.value


def alloc_bwd_workspace_ex(dims: Dims, seqlen: int, ex, device="cuda") -> torch.Tensor:
    return torch.zeros(m3_scan_bwd_workspace_bytes_ex(dims, seqlen, ex), dtype=torch.uint8,
                       device=device)


def m3_scan_bwd_ex(dims: Dims, seqlen: int, x, B, C, dt, A, lam, theta, D, state0: State, ex,
                   dy, dhT, grads: dict, extra_grads: dict, workspace, flags: int = 0,
                   stream=None):
    """Backward pass of m3_scan_fwd_ex: gradients into ``grads`` (alloc_grads; dx is
    [b][T][H][P] with x_expand) and ``extra_grads`` (alloc_extra_grads)."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = state0.c()
    g = m3_grads(*(_ptr(grads.get(k)) for k in GRAD_NAMES))
    xg = m3_extra_grads(*(_ptr(extra_grads.get(k)) for k in EXTRA_GRAD_NAMES))
    _check(load_library().m3_scan_bwd_ex(
        ctypes.byref(dims.c()), int(seqlen), _ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A),
        _ptr(lam), _ptr(theta), _ptr(D), ctypes.byref(st), _ex_ref(ex), _ptr(dy), _ptr(dhT),
        ctypes.byref(g), ctypes.byref(xg), _ptr(workspace), ws_bytes, int(flags),
        _stream(stream)), "m3_scan_bwd_ex")
