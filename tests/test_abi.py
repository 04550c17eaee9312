"""The C-ABI library loads and exports every entry point the header declares;
host-side validation answers with status codes before touching the GPU (CPU only)."""
import ctypes
import os
import re

import pytest

from state_space_model_06_b200 import m3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "m3.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(m3_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(m3.LIB_PATH):
        import __graft_entry__
        __graft_entry__.build()
    return m3.load_library()


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("m3_state_init", "m3_scan_fwd", "m3_decode_step"):
        assert name in fns
    assert set(m3.EXPORTED) <= set(fns)


def test_every_declared_symbol_is_exported(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(10):
        assert m3.m3_status_string(s)
    assert "timed out" in m3.m3_status_string(m3.M3_ERR_TIMEOUT)


def test_state_bytes(lib):
    d = m3.Dims(8, 64, 1, 64, 128, 1, m3.M3_BF16)
    assert m3.m3_state_bytes(d) == (8 * 64 * 128 * 64 * 4, 8 * 64 * 64 * 2, 8 * 128 * 2)


def test_workspace_bytes_covers_status_block(lib):
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_F32)
    assert m3.m3_scan_workspace_bytes(d, 256, 64) >= 256


@pytest.mark.parametrize("dims,status", [
    (m3.Dims(1, 3, 2, 16, 16, 1, m3.M3_BF16), m3.M3_ERR_SHAPE),     # H % G != 0
    (m3.Dims(1, 2, 1, 16, 15, 1, m3.M3_BF16), m3.M3_ERR_SHAPE),     # odd N
    (m3.Dims(0, 2, 1, 16, 16, 1, m3.M3_BF16), m3.M3_ERR_SHAPE),     # empty batch
    (m3.Dims(1, 2, 1, 16, 16, 1, 7), m3.M3_ERR_DTYPE),
    (m3.Dims(1, 2, 1, 16, 16, 16, m3.M3_BF16), m3.M3_ERR_UNSUPPORTED),
])
def test_bad_dims_rejected(lib, dims, status):
    with pytest.raises(m3.M3Error) as e:
        m3.m3_state_bytes(dims)
    assert e.value.status == status


def _raw_scan(lib, dims, T=16, chunk=64, ptr=0x1000, state=None, ws=0x100000, ws_bytes=1 << 20,
              x=None):
    st = state if state is not None else m3.m3_state(0x2000, 0x3000, 0x4000)
    x = ptr if x is None else x
    return lib.m3_scan_fwd(ctypes.byref(dims.c()), T, chunk, x, ptr, ptr, ptr, ptr, ptr, ptr,
                           None, ctypes.byref(st), ptr, ws, ws_bytes, 0, None)


def test_scan_validation_before_launch(lib):
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_BF16)
    assert _raw_scan(lib, d, x=0) == m3.M3_ERR_NULL
    assert _raw_scan(lib, d, state=m3.m3_state(0, 0x3000, 0x4000)) == m3.M3_ERR_NULL
    assert _raw_scan(lib, d, x=0x1008) == m3.M3_ERR_ALIGN
    assert _raw_scan(lib, d, chunk=48) == m3.M3_ERR_SHAPE
    assert _raw_scan(lib, d, T=-1) == m3.M3_ERR_SHAPE
    assert _raw_scan(lib, d, ws=0) == m3.M3_ERR_WORKSPACE
    assert _raw_scan(lib, d, ws_bytes=16) == m3.M3_ERR_WORKSPACE
    assert _raw_scan(lib, d, ws=0x100010) == m3.M3_ERR_WORKSPACE
    # seqlen 0 is a validated no-op: nothing is launched
    assert _raw_scan(lib, d, T=0) == m3.M3_OK


def test_decode_validation_before_launch(lib):
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_BF16)
    st = m3.m3_state(0x2000, 0x3000, 0x4000)
    p = 0x1000
    args = lambda x, y, s: (ctypes.byref(d.c()), x, p, p, p, p, p, p, None, ctypes.byref(s), y, 0,
                            None)
    assert lib.m3_decode_step(*args(0, p, st)) == m3.M3_ERR_NULL
    assert lib.m3_decode_step(*args(p, p + 2, st)) == m3.M3_ERR_ALIGN
    assert lib.m3_decode_step(*args(p, p, m3.m3_state(0x2004, 0x3000, 0x4000))) == m3.M3_ERR_ALIGN
    d2 = m3.Dims(1, 2, 1, 18, 16, 1, m3.M3_BF16)       # P % 4 != 0: no decode kernel
    assert lib.m3_decode_step(ctypes.byref(d2.c()), p, p, p, p, p, p, p, None, ctypes.byref(st),
                              p, 0, None) == m3.M3_ERR_UNSUPPORTED


def test_gated_validation_before_launch(lib):
    """The gated entry points check z (present, 16-byte aligned) before anything else runs."""
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_BF16)
    st = m3.m3_state(0x2000, 0x3000, 0x4000)
    p, ws = 0x1000, 0x100000

    def scan(z, T=16):
        return lib.m3_scan_fwd_gated(ctypes.byref(d.c()), T, 64, p, p, p, p, p, p, p, None, z,
                                     ctypes.byref(st), p, ws, 1 << 20, 0, None)

    assert scan(None) == m3.M3_ERR_NULL
    assert scan(p + 8) == m3.M3_ERR_ALIGN
    assert scan(None, T=0) == m3.M3_OK        # seqlen 0: a validated no-op

    def dec(z):
        return lib.m3_decode_step_gated(ctypes.byref(d.c()), p, p, p, p, p, p, p, None, z,
                                        ctypes.byref(st), p, 0, None)

    assert dec(None) == m3.M3_ERR_NULL
    assert dec(p + 4) == m3.M3_ERR_ALIGN


def test_extras_validation_before_launch(lib):
    """m3_scan_fwd_ex / m3_decode_step_ex check the extras before anything runs, and the
    BCNorm scales are part of the workspace size."""
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_BF16)
    st = m3.m3_state(0x2000, 0x3000, 0x4000)
    p, ws = 0x1000, 0x100000
    base = m3.m3_scan_workspace_bytes(d, 64, 64)
    assert m3.m3_scan_workspace_bytes_ex(d, 64, 64, None) == base
    assert m3.m3_scan_workspace_bytes_ex(d, 64, 64, m3.Extras(B_bias=p)) == base
    with_norm = m3.m3_scan_workspace_bytes_ex(d, 64, 64, m3.Extras(bc_norm_eps=1e-6))
    assert with_norm >= base + 4 * (2 * 64 + 1)

    def scan(ex, ws_bytes=1 << 20):
        e = ex.c()
        return lib.m3_scan_fwd_ex(ctypes.byref(d.c()), 64, 64, p, p, p, p, p, p, p, None,
                                  ctypes.byref(e), ctypes.byref(st), p, ws, ws_bytes, 0, None)

    assert scan(m3.Extras(bc_norm_eps=-1.0)) == m3.M3_ERR_SHAPE
    assert scan(m3.Extras(bc_norm_eps=float("nan"))) == m3.M3_ERR_SHAPE
    assert scan(m3.Extras(B_bias=p + 2)) == m3.M3_ERR_ALIGN
    assert scan(m3.Extras(z=p + 8)) == m3.M3_ERR_ALIGN
    assert scan(m3.Extras(bc_norm_eps=1e-6), ws_bytes=base) == m3.M3_ERR_WORKSPACE

    def dec(ex):
        e = ex.c()
        return lib.m3_decode_step_ex(ctypes.byref(d.c()), p, p, p, p, p, p, p, None,
                                     ctypes.byref(e), ctypes.byref(st), p, 0, None)

    assert dec(m3.Extras(bc_norm_eps=-1.0)) == m3.M3_ERR_SHAPE
    assert dec(m3.Extras(C_bias=p + 1)) == m3.M3_ERR_ALIGN

    # MIMO lightweight expansion: 16-byte aligned weights; an expanded gate needs z
    for call in (scan, dec):
        assert call(m3.Extras(x_expand=p + 4)) == m3.M3_ERR_ALIGN
        assert call(m3.Extras(z_expand=p)) == m3.M3_ERR_NULL
        assert call(m3.Extras(z=p, z_expand=p + 8)) == m3.M3_ERR_ALIGN


def test_struct_layouts_match_the_header(tmp_path):
    """The binding's ctypes structs have the C header's sizes and field offsets."""
    import subprocess
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "m3.h"\n'
        'int main(void) {\n'
        '  printf("%zu %zu %zu\\n", sizeof(m3_dims), sizeof(m3_state), sizeof(m3_extras));\n'
        '  printf("%zu %zu %zu %zu %zu %zu\\n", offsetof(m3_extras, z), offsetof(m3_extras, B_bias),'
        ' offsetof(m3_extras, C_bias), offsetof(m3_extras, bc_norm_eps),'
        ' offsetof(m3_extras, x_expand), offsetof(m3_extras, z_expand));\n'
        '  return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    out = subprocess.check_output([str(exe)]).decode().split()
    sizes = [int(v) for v in out[:3]]
    offs = [int(v) for v in out[3:]]
    assert sizes == [ctypes.sizeof(m3.m3_dims), ctypes.sizeof(m3.m3_state),
                     ctypes.sizeof(m3.m3_extras)]
    assert offs == [getattr(m3.m3_extras, f).offset for f in
                    ("z", "B_bias", "C_bias", "bc_norm_eps", "x_expand", "z_expand")]


def test_binding_refuses_missing_library(tmp_path):
    old = m3._lib
    m3._lib = None
    try:
        with pytest.raises(RuntimeError):
            m3.load_library(str(tmp_path / "missing.so"))
    finally:
        m3._lib = old


def test_backward_validation_before_launch(lib):
    """m3_scan_bwd checks its arguments (nulls, alignment, supported shape, workspace size)
    before anything is launched."""
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_F32)
    st = m3.m3_state(0x2000, 0x3000, 0x4000)
    p, ws = 0x1000, 0x100000
    need = m3.m3_scan_bwd_workspace_bytes(d, 64)
    assert need >= 256 + 4 * (2 * 16 * 16 * 4)          # status block + a few states
    full = m3.m3_grads(*([p] * 11))

    def bwd(dims=d, grads=full, dy=p, ws_bytes=need, T=64, state=st):
        return lib.m3_scan_bwd(ctypes.byref(dims.c()), T, p, p, p, p, p, p, p, None,
                               ctypes.byref(state), dy, None,
                               ctypes.byref(grads) if grads is not None else None, ws, ws_bytes,
                               0, None)

    assert bwd(T=0) == m3.M3_OK                                   # nothing to do
    assert bwd(T=-1) == m3.M3_ERR_SHAPE
    assert bwd(grads=None) == m3.M3_ERR_NULL
    assert bwd(dy=None) == m3.M3_ERR_NULL
    assert bwd(grads=m3.m3_grads(*([p] * 10 + [None]))) == m3.M3_ERR_NULL   # dB_prev
    assert bwd(grads=m3.m3_grads(*([p + 2] + [p] * 10))) == m3.M3_ERR_ALIGN
    assert bwd(dy=p + 8) == m3.M3_ERR_ALIGN
    assert bwd(state=m3.m3_state(0x2000, 0, 0x4000)) == m3.M3_ERR_NULL
    assert bwd(ws_bytes=need - 256) == m3.M3_ERR_WORKSPACE
    assert bwd(dims=m3.Dims(1, 2, 1, 128, 16, 1, m3.M3_F32),
               ws_bytes=1 << 30) == m3.M3_ERR_UNSUPPORTED      # headdim 128: no kernel


def test_backward_ex_validation_before_launch(lib):
    """m3_scan_bwd_ex checks the extras and their gradient pointers (needed exactly when the
    part is on), alignment, epsilon and the workspace before anything is launched; an
    all-zero extras block is the plain backward."""
    d = m3.Dims(1, 2, 1, 16, 16, 2, m3.M3_F32)
    st = m3.m3_state(0x2000, 0x3000, 0x4000)
    p, ws = 0x1000, 0x100000
    full = m3.m3_grads(*([p] * 11))

    def ex_of(**kw):
        e = m3.m3_extras()
        for k, v in kw.items():
            setattr(e, k, v)
        return e

    gate = ex_of(z=p, z_expand=p, x_expand=p, B_bias=p, bc_norm_eps=1e-5)
    all_xg = m3.m3_extra_grads(p, p, None, p, p)
    n = ctypes.c_size_t()
    assert lib.m3_scan_bwd_workspace_bytes_ex(ctypes.byref(d.c()), 64, ctypes.byref(gate),
                                              ctypes.byref(n)) == m3.M3_OK
    need = n.value
    assert need > m3.m3_scan_bwd_workspace_bytes(d, 64)       # effective inputs, y_pre, ...
    bad = ex_of(bc_norm_eps=-1.0)
    assert lib.m3_scan_bwd_workspace_bytes_ex(ctypes.byref(d.c()), 64, ctypes.byref(bad),
                                              ctypes.byref(n)) == m3.M3_ERR_SHAPE

    def bwd(ex=gate, xg=all_xg, ws_bytes=need, T=64, dims=d):
        return lib.m3_scan_bwd_ex(ctypes.byref(dims.c()), T, p, p, p, p, p, p, p, None,
                                  ctypes.byref(st), ctypes.byref(ex) if ex is not None else None,
                                  p, None, ctypes.byref(full),
                                  ctypes.byref(xg) if xg is not None else None, ws, ws_bytes, 0,
                                  None)

    assert bwd(T=0) == m3.M3_OK
    assert bwd(T=-1) == m3.M3_ERR_SHAPE
    assert bwd(xg=None) == m3.M3_ERR_NULL
    assert bwd(xg=m3.m3_extra_grads(None, p, None, p, p)) == m3.M3_ERR_NULL        # dz
    assert bwd(xg=m3.m3_extra_grads(p, None, None, p, p)) == m3.M3_ERR_NULL        # dB_bias
    assert bwd(xg=m3.m3_extra_grads(p, p, None, None, p)) == m3.M3_ERR_NULL        # dx_expand
    assert bwd(xg=m3.m3_extra_grads(p, p, None, p, None)) == m3.M3_ERR_NULL        # dz_expand
    assert bwd(ex=ex_of(z_expand=p), xg=m3.m3_extra_grads(p, None, None, None, p)) == m3.M3_ERR_NULL
    assert bwd(ex=ex_of(C_bias=p, bc_norm_eps=float("nan"))) == m3.M3_ERR_SHAPE
    assert bwd(ex=ex_of(z=p + 2), xg=m3.m3_extra_grads(p, None, None, None, None)) == m3.M3_ERR_ALIGN
    assert bwd(ex=ex_of(x_expand=p + 4), xg=m3.m3_extra_grads(None, None, None, p, None)) == m3.M3_ERR_ALIGN
    assert bwd(ws_bytes=need - 256) == m3.M3_ERR_WORKSPACE
    assert bwd(dims=m3.Dims(1, 2, 1, 128, 16, 2, m3.M3_F32), ws_bytes=1 << 34) == m3.M3_ERR_UNSUPPORTED


def test_status_strings_cover_range_code(lib):
    assert "range" in m3.m3_status_string(m3.M3_ERR_RANGE)


def test_noalloc_validation_before_any_cuda_call(lib):
    """m3_scan_fwd_noalloc makes every host-side check of m3_scan_fwd before it asks the CUDA
    runtime for anything: bad arguments come back as the same status codes, here on a
    machine without a GPU."""
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_BF16)
    p = 0x1000

    def call(T=16, chunk=64, x=p, y=p, state=None, flags=0, dims=d):
        st = state if state is not None else m3.m3_state(0x2000, 0x3000, 0x4000)
        return lib.m3_scan_fwd_noalloc(ctypes.byref(dims.c()), T, chunk, x, p, p, p, p, p, p,
                                       None, ctypes.byref(st), y, flags, None)

    assert call(x=0) == m3.M3_ERR_NULL
    assert call(state=m3.m3_state(0x2000, 0, 0x4000)) == m3.M3_ERR_NULL
    assert call(y=p + 8) == m3.M3_ERR_ALIGN
    assert call(chunk=48) == m3.M3_ERR_SHAPE
    assert call(T=-1) == m3.M3_ERR_SHAPE
    assert call(dims=m3.Dims(1, 3, 2, 16, 16, 1, m3.M3_BF16)) == m3.M3_ERR_SHAPE
    assert call(T=0) == m3.M3_OK                        # validated no-op
    # the debug scan reports into a status word this entry point never reads back
    assert call(flags=m3.M3_FLAG_DEBUG_CHECKS) == m3.M3_ERR_UNSUPPORTED
    import torch
    if not torch.cuda.is_available():
        # valid arguments reach the device lookup, which fails cleanly without a GPU
        assert call() == m3.M3_ERR_CUDA


def test_decode_rejects_debug_checks(lib):
    """The decode step has no workspace status word for the debug scan to report into."""
    d = m3.Dims(1, 2, 1, 16, 16, 1, m3.M3_BF16)
    st = m3.m3_state(0x2000, 0x3000, 0x4000)
    p = 0x1000
    assert lib.m3_decode_step(ctypes.byref(d.c()), p, p, p, p, p, p, p, None, ctypes.byref(st),
                              p, m3.M3_FLAG_DEBUG_CHECKS, None) == m3.M3_ERR_UNSUPPORTED
