"""The seeded input generators: determinism, bf16 rounding, grids and shapes."""
import numpy as np
import torch

from int4_group_wise_b200 import inputs


def test_bf16_conversion_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 50,
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0, 3e-39], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(inputs.f32_to_bf16_bits(x), ref)
    back = inputs.bf16_bits_to_f32(ref)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_generators_are_deterministic_and_independent():
    a = inputs.gaussian((3, 1000), 0.02, seed=0, cfg=1, name="W/x")
    b = inputs.gaussian((3, 1000), 0.02, seed=0, cfg=1, name="W/x")
    c = inputs.gaussian((3, 1000), 0.02, seed=0, cfg=1, name="W/y")
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    assert abs(a.std() - 0.02) < 0.002
    x1 = inputs.activations(64, 256, seed=0, cfg=0, name="x", outliers=4)
    x2 = inputs.activations(64, 256, seed=0, cfg=0, name="x", outliers=4)
    np.testing.assert_array_equal(x1, x2)
    xf = inputs.bf16_bits_to_f32(x1)
    big = np.abs(xf).max(axis=0) > 10
    assert big.sum() == 4                       # exactly the 4 outlier columns stand out


def test_alpha_grids_by_index():
    a = inputs.alpha_grid(0.5, 0.005, 101)
    assert a.size == 101 and a[0] == np.float32(0.5) and a[-1] == np.float32(1.0)
    b = inputs.alpha_grid(0.30, 0.0035, 201)
    assert b.size == 201 and b[0] == np.float32(0.3) and b[-1] == np.float32(1.0)
    assert np.all(np.diff(a) > 0) and np.all(np.diff(b) > 0)


def test_workload_shapes():
    w3 = inputs.workload(3)
    assert len(w3.matrices) == 112 and len(w3.calib) == 64
    assert sum(m.d_out * m.d_in for m in w3.matrices) == 16 * (2048 * 2048 * 2 + 512 * 2048 * 2
                                                                + 8192 * 2048 * 2 + 2048 * 8192)
    w4 = inputs.workload(4)
    assert len(w4.matrices) == 224 and len(w4.searched) == 7
    assert sum(m.d_out * m.d_in for m in w4.matrices) == 6_979_321_856
    w0 = inputs.workload(0)
    assert w0.g_dtype == "f32" and w0.K == 101 and w0.matrices[0].d_in == 512
    assert inputs.workload(2).K == 201


def test_row_prefix_has_the_full_tensors_bytes():
    """weight(rows=r) / grad(rows=r) / activations(n=r) are the first r rows of the full tensors
    (the bounded CPU samples of the benchmark rely on it)."""
    w2 = inputs.workload(2)
    m2 = w2.matrices[0]
    full = w2.weight(m2)
    np.testing.assert_array_equal(w2.weight(m2, rows=100), full[:100])
    np.testing.assert_array_equal(w2.grad(m2, rows=64), w2.grad(m2)[:64])
    w0 = inputs.workload(0)
    np.testing.assert_array_equal(w0.activations("x", n=300), w0.activations("x")[:300])
    np.testing.assert_array_equal(w0.weight(w0.matrices[0], rows=17), w0.weight(w0.matrices[0])[:17])
