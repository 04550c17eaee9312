"""Plain fp64 CPU oracle for the Mamba-3 mixer recurrence.

TEST INFRASTRUCTURE ONLY.  The oracle is the slow, obviously correct reference
that the CUDA path is checked against; it is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py`` and by
nothing else.  It shares no code with the CUDA library in
``state_space_model_06_b200``, and neither side imports the other.

The arithmetic lives in ``m3_oracle.c`` (sequential fp64 loop over tokens,
OpenMP over independent (batch, head) pairs).  This module only builds that
file with gcc and marshals numpy float64 arrays into it.

Every function here follows the Mamba-3 paper summary, "Technical Approach":
Proposition 1 (exponential-trapezoidal recurrence), Propositions 2-4 (complex
transition as a data-dependent rotation of state pairs) and the MIMO
formulation (rank-R input and readout).  Parity pins for each part live in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3_oracle.c")
_LIB = os.path.join(_HERE, "libm3_oracle.so")

THETA_IS_ANGLE = 1


def build(force: bool = False) -> str:
    """Compile ``m3_oracle.c`` into ``libm3_oracle.so`` next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "nheads", "ngroups", "headdim", "dstate", "rank")]


_libs = {}


def _load(path=None):
    """Load the oracle library (``path`` lets a test load a deliberately broken copy)."""
    path = path or build()
    if path not in _libs:
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.m3o_scan.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int64, ctypes.c_uint32] + \
            [dp] * 12 + [ctypes.c_int]
        lib.m3o_scan.restype = ctypes.c_int
        lib.m3o_scan_ex.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int64, ctypes.c_uint32] + \
            [dp] * 10 + [ctypes.c_double] + [dp] * 4 + [ctypes.c_int]
        lib.m3o_scan_ex.restype = ctypes.c_int
        lib.m3o_max_threads.restype = ctypes.c_int
        lib.m3o_gate.argtypes = [ctypes.c_int64, dp, dp]
        lib.m3o_gate.restype = None
        lib.m3o_expand.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   dp, dp, dp]
        lib.m3o_expand.restype = None
        lib.m3o_scan_bwd.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int64, ctypes.c_uint32] + \
            [dp] * 24 + [ctypes.c_int]
        lib.m3o_scan_bwd.restype = ctypes.c_int
        _libs[path] = lib
    return _libs[path]


def max_threads() -> int:
    return int(_load().m3o_max_threads())


def _f64(a, shape, name):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if tuple(a.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {a.shape}")
    return a


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def expand(v, w, lib_path=None):
    """MIMO lightweight expansion: v [..., H, P] times w [H, R, P] gives [..., H, R, P]
    with out[..., h, r, p] = v[..., h, p] * w[h, r, p] (float64)."""
    w = np.asarray(w)
    H, R, P = w.shape
    v = np.asarray(v)
    lead = v.shape[:-2]
    v = _f64(v, tuple(lead) + (H, P), "expanded input")
    w = _f64(w, (H, R, P), "expansion weights")
    out = np.zeros(tuple(lead) + (H, R, P))
    rows = int(np.prod(lead)) if lead else 1
    _load(lib_path).m3o_expand(rows, H, R, P, _ptr(v), _ptr(w), _ptr(out))
    return out


def scan(x, B, C, dt, A, lam, theta, D=None, h0=None, x_prev=None, B_prev=None,
         theta_is_angle: bool = False, nthreads: int = 0, lib_path=None, z=None,
         B_bias=None, C_bias=None, bc_eps: float = 0.0, x_expand=None, z_expand=None):
    """Run the recurrence over T tokens.

    Shapes: x [b,T,H,R,P]; B, C [b,T,G,R,N]; dt, A, lam [b,T,H];
    theta [b,T,G,N/2]; D [H] or None; h0 [b,H,N,P] or None (zeros);
    x_prev [b,H,R,P] / B_prev [b,G,R,N] or None (fresh sequence: zeros);
    z [b,T,H,R,P] or None: output gate, y <- y * SiLU(z) after the skip
    ("Technical Approach", output gating).
    B_bias, C_bias [H,N] or None and bc_eps > 0: BC biases and BC normalisation
    ("Technical Approach", BCNorm and BC biases): per token, each rank column of B and
    C is scaled to unit RMS over N (when bc_eps > 0), then the head's bias is added.
    x_expand / z_expand [H,R,P] or None: MIMO lightweight expansion ("Multi-Input,
    Multi-Output (MIMO) Formulation", MIMO Parameterization Choices); x (z) is then
    [b,T,H,P] and the recurrence uses expand(x, x_expand) (the gate expand(z, z_expand)).
    x_prev stays the expanded [b,H,R,P] previous input.

    Returns (y [b,T,H,R,P], h_T, x_prev_out, B_prev_out), all float64.
    """
    if x_expand is not None:
        x = expand(x, x_expand, lib_path)
    if z is not None and z_expand is not None:
        z = expand(z, z_expand, lib_path)
    x = np.asarray(x)
    b, T, H, R, P = x.shape
    G, N = np.asarray(B).shape[2], np.asarray(B).shape[4]
    x = _f64(x, (b, T, H, R, P), "x")
    B = _f64(B, (b, T, G, R, N), "B")
    C = _f64(C, (b, T, G, R, N), "C")
    dt = _f64(dt, (b, T, H), "dt")
    A = _f64(A, (b, T, H), "A")
    lam = _f64(lam, (b, T, H), "lam")
    theta = _f64(theta, (b, T, G, N // 2), "theta")
    D = None if D is None else _f64(D, (H,), "D")
    h = np.zeros((b, H, N, P)) if h0 is None else _f64(h0, (b, H, N, P), "h0").copy()
    xp = np.zeros((b, H, R, P)) if x_prev is None else _f64(x_prev, (b, H, R, P), "x_prev").copy()
    bp = np.zeros((b, G, R, N)) if B_prev is None else _f64(B_prev, (b, G, R, N), "B_prev").copy()
    y = np.zeros((b, T, H, R, P))
    dims = _Dims(b, H, G, P, N, R)
    fl = THETA_IS_ANGLE if theta_is_angle else 0
    if B_bias is None and C_bias is None and bc_eps <= 0.0:
        rc = _load(lib_path).m3o_scan(ctypes.byref(dims), T, fl, _ptr(x), _ptr(B), _ptr(C),
                                      _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta), _ptr(D),
                                      _ptr(h), _ptr(xp), _ptr(bp), _ptr(y), int(nthreads))
    else:
        bb = None if B_bias is None else _f64(B_bias, (H, N), "B_bias")
        cb = None if C_bias is None else _f64(C_bias, (H, N), "C_bias")
        rc = _load(lib_path).m3o_scan_ex(ctypes.byref(dims), T, fl, _ptr(x), _ptr(B), _ptr(C),
                                         _ptr(dt), _ptr(A), _ptr(lam), _ptr(theta), _ptr(D),
                                         _ptr(bb), _ptr(cb), float(bc_eps), _ptr(h), _ptr(xp),
                                         _ptr(bp), _ptr(y), int(nthreads))
    if rc != 0:
        raise ValueError(f"m3o_scan rejected its arguments (code {rc})")
    if z is not None:
        z = _f64(z, (b, T, H, R, P), "z")
        _load(lib_path).m3o_gate(y.size, _ptr(z), _ptr(y))
    return y, h, xp, bp


def scan_bwd(x, B, C, dt, A, lam, theta, dy, D=None, h0=None, x_prev=None, B_prev=None,
             dhT=None, theta_is_angle: bool = False, nthreads: int = 0, lib_path=None):
    """Reverse-mode gradients of ``scan`` (no fused extras) for a loss with dL/dy = dy
    [b,T,H,R,P] and dL/dh_T = dhT [b,H,N,P] (None: zero).

    Returns a dict of float64 arrays: dx [b,T,H,R,P]; dB, dC [b,T,G,R,N] and dtheta
    [b,T,G,N/2] (summed over the heads of each group); ddt, dA, dlam [b,T,H]; dD [H] (summed
    over batch and tokens; None without D); dh0 [b,H,N,P]; dx_prev [b,H,R,P]; dB_prev
    [b,G,R,N].  The carried x_prev / B_prev outputs of the call get no gradient here.
    """
    x = np.asarray(x)
    b, T, H, R, P = x.shape
    G, N = np.asarray(B).shape[2], np.asarray(B).shape[4]
    ins = dict(
        x=_f64(x, (b, T, H, R, P), "x"), B=_f64(B, (b, T, G, R, N), "B"),
        C=_f64(C, (b, T, G, R, N), "C"), dt=_f64(dt, (b, T, H), "dt"),
        A=_f64(A, (b, T, H), "A"), lam=_f64(lam, (b, T, H), "lam"),
        theta=_f64(theta, (b, T, G, N // 2), "theta"))
    D = None if D is None else _f64(D, (H,), "D")
    h0 = None if h0 is None else _f64(h0, (b, H, N, P), "h0")
    xp = None if x_prev is None else _f64(x_prev, (b, H, R, P), "x_prev")
    bp = None if B_prev is None else _f64(B_prev, (b, G, R, N), "B_prev")
    dy = _f64(dy, (b, T, H, R, P), "dy")
    dhT = None if dhT is None else _f64(dhT, (b, H, N, P), "dhT")
    out = dict(dx=np.zeros((b, T, H, R, P)), dB=np.zeros((b, T, G, R, N)),
               dC=np.zeros((b, T, G, R, N)), ddt=np.zeros((b, T, H)), dA=np.zeros((b, T, H)),
               dlam=np.zeros((b, T, H)), dtheta=np.zeros((b, T, G, N // 2)),
               dD=np.zeros(H), dh0=np.zeros((b, H, N, P)), dx_prev=np.zeros((b, H, R, P)),
               dB_prev=np.zeros((b, G, R, N)))
    dims = _Dims(b, H, G, P, N, R)
    fl = THETA_IS_ANGLE if theta_is_angle else 0
    rc = _load(lib_path).m3o_scan_bwd(
        ctypes.byref(dims), T, fl, *(_ptr(ins[k]) for k in ("x", "B", "C", "dt", "A", "lam",
                                                           "theta")),
        _ptr(D), _ptr(h0), _ptr(xp), _ptr(bp), _ptr(dy), _ptr(dhT),
        *(_ptr(out[k]) for k in ("dx", "dB", "dC", "ddt", "dA", "dlam", "dtheta", "dD", "dh0",
                                 "dx_prev", "dB_prev")), int(nthreads))
    if rc != 0:
        raise ValueError(f"m3o_scan_bwd rejected its arguments (code {rc})")
    if D is None:
        out["dD"] = None
    return out


def decode_step(x, B, C, dt, A, lam, theta, D, h, x_prev, B_prev,
                theta_is_angle: bool = False, nthreads: int = 0, z=None, B_bias=None,
                C_bias=None, bc_eps: float = 0.0, x_expand=None, z_expand=None):
    """One decode token: x [b,H,R,P] ([b,H,P] with x_expand), B/C [b,G,R,N], dt/A/lam
    [b,H], theta [b,G,N/2]; z [b,H,R,P] ([b,H,P] with z_expand) or None (output gate).

    Identical to ``scan`` with T = 1; returns (y [b,H,R,P], h, x_prev, B_prev).
    """
    ins = [np.asarray(v)[:, None] for v in (x, B, C, dt, A, lam, theta)]
    y, h, xp, bp = scan(*ins, D=D, h0=h, x_prev=x_prev, B_prev=B_prev,
                        theta_is_angle=theta_is_angle, nthreads=nthreads,
                        z=None if z is None else np.asarray(z)[:, None], B_bias=B_bias,
                        C_bias=C_bias, bc_eps=bc_eps, x_expand=x_expand, z_expand=z_expand)
    return y[:, 0], h, xp, bp
