"""The seeded input generators (CPU): reproducible per seed, the documented shapes and
distributions, and the optional parts drawn from generators of their own."""
import math

import torch

from state_space_model_06_b200 import inputs


def test_scan_inputs_are_reproducible_and_shaped():
    a = inputs.make_scan_inputs(2, 33, 4, 2, 8, 6, 3, io_dtype=torch.float32, seed=5,
                                h0_random=True, carry_prev=True)
    b = inputs.make_scan_inputs(2, 33, 4, 2, 8, 6, 3, io_dtype=torch.float32, seed=5,
                                h0_random=True, carry_prev=True)
    shapes = dict(x=(2, 33, 4, 3, 8), B=(2, 33, 2, 3, 6), C=(2, 33, 2, 3, 6), dt=(2, 33, 4),
                  A=(2, 33, 4), lam=(2, 33, 4), theta=(2, 33, 2, 3), D=(4,), h0=(2, 4, 6, 8),
                  x_prev=(2, 4, 3, 8), B_prev=(2, 2, 3, 6))
    for k, shp in shapes.items():
        assert tuple(a[k].shape) == shp, k
        assert torch.equal(a[k], b[k]), k
    c = inputs.make_scan_inputs(2, 33, 4, 2, 8, 6, 3, io_dtype=torch.float32, seed=6)
    assert not torch.equal(a["x"], c["x"])


def test_value_ranges_of_the_recipe():
    v = inputs.make_scan_inputs(4, 512, 8, 1, 16, 64, 1, io_dtype=torch.float32, seed=1)
    assert bool((v["dt"] > 0).all())
    assert bool((v["A"] < 0).all())
    assert bool(((v["lam"] > 0) & (v["lam"] < 1)).all())
    assert float(v["theta"].abs().max()) <= math.pi / 8
    # B ~ N(0, 1/N): its variance is near 1/N
    assert abs(float(v["B"].var()) * 64 - 1.0) < 0.05
    assert bool((v["h0"] == 0).all()) and bool((v["x_prev"] == 0).all())


def test_optional_parts_do_not_disturb_the_other_inputs():
    """The gate, the BC biases and the expansion weights come from generators of their own:
    drawing them leaves every other input of the same seed unchanged."""
    base = inputs.make_scan_inputs(1, 20, 4, 1, 8, 6, 2, io_dtype=torch.float32, seed=3)
    z = inputs.make_gate((1, 20, 4, 2, 8), io_dtype=torch.float32, seed=3)
    bb, cb = inputs.make_bc_bias(4, 6, seed=3)
    wx, wz = inputs.make_expand(4, 2, 8, seed=3)
    again = inputs.make_scan_inputs(1, 20, 4, 1, 8, 6, 2, io_dtype=torch.float32, seed=3)
    for k in base:
        assert torch.equal(base[k], again[k]), k
    assert not torch.equal(z.reshape(-1)[:40], base["x"].reshape(-1)[:40])
    assert tuple(bb.shape) == (4, 6) and tuple(wx.shape) == (4, 2, 8)
    assert abs(float(bb.mean()) - 1.0) < 0.2          # all-ones initialisation plus a spread
    assert not torch.equal(wx, wz)


def test_bf16_workloads_round_at_the_source():
    v = inputs.make_scan_inputs(1, 16, 4, 1, 8, 6, 1, io_dtype=torch.bfloat16, seed=2)
    assert v["x"].dtype == torch.bfloat16 and v["B"].dtype == torch.bfloat16
    assert v["dt"].dtype == torch.float32 and v["theta"].dtype == torch.float32
