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


def _bc_map(v, bias, eps):
    """BC map of the columns v [..., N] (the same map m3o_bc_map applies): scale to unit RMS
    when eps > 0, then add the bias (None: 0).  Returns (map(v), scale [..., 1])."""
    if eps > 0.0:
        s = 1.0 / np.sqrt((v * v).mean(axis=-1, keepdims=True) + eps)
    else:
        s = np.ones(v.shape[:-1] + (1,))
    return v * s + (0.0 if bias is None else bias), s


def _bc_map_bwd(v, s, du, eps):
    """dL/dv of u = v s(v) + bias given du: s du - (s^3 / N) v <du, v> (RMS scale), or du."""
    if eps <= 0.0:
        return du
    return s * du - (s ** 3 / v.shape[-1]) * v * (du * v).sum(axis=-1, keepdims=True)


def scan_bwd_ex(x, B, C, dt, A, lam, theta, dy, D=None, h0=None, x_prev=None, B_prev=None,
                dhT=None, theta_is_angle=False, z=None, B_bias=None, C_bias=None,
                bc_eps: float = 0.0, x_expand=None, z_expand=None, nthreads: int = 0):
    """Reverse-mode gradients of ``scan`` with the fused extras (output gate, BC map, MIMO
    lightweight expansion), for dL/dy = dy [b,T,H,R,P] and dL/dh_T = dhT.

    Built on ``scan_bwd``: the extras' effective inputs are formed per head (X = x * x_expand,
    Z = z * z_expand; B, C, B_prev through the BC map with the head's bias; theta per head),
    the recurrence's backward runs with one group per head, and the chain goes back through
    the gate (SiLU'(Z) = sig(Z) (1 + Z (1 - sig(Z)))), the RMS scale's Jacobian and the
    expansion weights, summing over the heads of each group.  Layouts as in ``scan``.
    Returns the dict of ``scan_bwd`` plus dz, dB_bias, dC_bias, dx_expand, dz_expand (None
    where the part is off).
    """
    x = np.asarray(x, dtype=np.float64)
    X = expand(x, x_expand) if x_expand is not None else x
    b, T, H, R, P = X.shape
    B = np.asarray(B, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    G, N = B.shape[2], B.shape[4]
    gidx = np.arange(H) // (H // G)
    Bh, Ch = B[:, :, gidx], C[:, :, gidx]                       # [b,T,H,R,N]
    Bp = np.zeros((b, G, R, N)) if B_prev is None else np.asarray(B_prev, dtype=np.float64)
    Bph = Bp[:, gidx]                                           # [b,H,R,N]
    bb = None if B_bias is None else np.asarray(B_bias, dtype=np.float64)
    cb = None if C_bias is None else np.asarray(C_bias, dtype=np.float64)
    Be, sB = _bc_map(Bh, None if bb is None else bb[None, None, :, None, :], bc_eps)
    Ce, sC = _bc_map(Ch, None if cb is None else cb[None, None, :, None, :], bc_eps)
    Bpe, sP = _bc_map(Bph, None if bb is None else bb[None, :, None, :], bc_eps)
    th = np.asarray(theta, dtype=np.float64)[:, :, gidx]
    Z = None
    dy = np.asarray(dy, dtype=np.float64)
    dy_pre, dZ = dy, None
    if z is not None:
        z = np.asarray(z, dtype=np.float64)
        Z = expand(z, z_expand) if z_expand is not None else z
        y_pre = scan(X, Be, Ce, dt, A, lam, th, D=D, h0=h0, x_prev=x_prev, B_prev=Bpe,
                     theta_is_angle=theta_is_angle, nthreads=nthreads)[0]
        sig = 1.0 / (1.0 + np.exp(-Z))
        dy_pre = dy * Z * sig
        dZ = dy * y_pre * sig * (1.0 + Z * (1.0 - sig))
    g = scan_bwd(X, Be, Ce, dt, A, lam, th, dy_pre, D=D, h0=h0, x_prev=x_prev, B_prev=Bpe,
                 dhT=dhT, theta_is_angle=theta_is_angle, nthreads=nthreads)
    out = dict(g)

    def to_groups(v, axis):
        acc = np.zeros(v.shape[:axis] + (G,) + v.shape[axis + 1:])
        for hh in range(H):
            idx = [slice(None)] * v.ndim
            idx[axis] = hh
            oidx = list(idx)
            oidx[axis] = gidx[hh]
            acc[tuple(oidx)] += v[tuple(idx)]
        return acc

    out["dB"] = to_groups(_bc_map_bwd(Bh, sB, g["dB"], bc_eps), 2)
    out["dC"] = to_groups(_bc_map_bwd(Ch, sC, g["dC"], bc_eps), 2)
    out["dB_prev"] = to_groups(_bc_map_bwd(Bph, sP, g["dB_prev"], bc_eps), 1)
    out["dtheta"] = to_groups(g["dtheta"], 2)
    out["dB_bias"] = None if bb is None else g["dB"].sum(axis=(0, 1, 3)) + g["dB_prev"].sum(axis=(0, 2))
    out["dC_bias"] = None if cb is None else g["dC"].sum(axis=(0, 1, 3))
    if x_expand is not None:
        w = np.asarray(x_expand, dtype=np.float64)
        out["dx"] = (g["dx"] * w).sum(axis=-2)
        out["dx_expand"] = (g["dx"] * x[..., None, :]).sum(axis=(0, 1))
    else:
        out["dx_expand"] = None
    out["dz"], out["dz_expand"] = None, None
    if z is not None:
        if z_expand is not None:
            wz = np.asarray(z_expand, dtype=np.float64)
            out["dz"] = (dZ * wz).sum(axis=-2)
            out["dz_expand"] = (dZ * z[..., None, :]).sum(axis=(0, 1))
        else:
            out["dz"] = dZ
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
