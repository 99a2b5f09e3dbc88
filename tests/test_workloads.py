"""The seeded synthetic inputs (workloads/) and two product-path guards.

The input recipe is shared by the tests, the bench and the oracle, so its
properties are pinned here on the CPU: the shapes and layouts of the five
workloads, reproducibility from the seed, the value distributions they state,
exact storage round trips, the layer-sweep adapter, and that the product
package never reaches the oracle or a CPU path.
"""
import ast
import os

import numpy as np
import pytest

import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_workload_shapes_layouts_and_activations():
    tiny, trunk, seg, many = (wl.spec(w) for w in range(4))
    assert (tiny.shape, tiny.layout, tiny.dtype, tiny.act) == ((2, 8, 16, 16), wl.NCHW, wl.F32,
                                                              wl.LEAKY_RELU)
    assert (trunk.shape, trunk.layout, trunk.dtype) == ((64, 256, 56, 56), wl.NHWC, wl.BF16)
    assert (seg.shape, seg.layout, seg.x_dist) == ((16, 512, 84, 84), wl.NHWC, "student_t3")
    assert (many.shape, many.layout, many.dtype, many.act) == ((128, 2048, 7, 7), wl.NCHW,
                                                              wl.F16, wl.ELU)
    assert many.gamma_lo == 0.05 and trunk.gamma_lo == 0.5
    sweep = [wl.spec(4, l) for l in range(16)]
    assert [(s.c, s.h) for s in sweep] == wl.SWEEP_SHAPES
    assert all(s.n == 8 and s.layout == wl.NHWC and s.dtype == wl.BF16 for s in sweep)
    assert [s.act for s in sweep] == [wl.LEAKY_RELU, wl.ELU] * 8
    assert len({s.seed for s in sweep}) == 16


def test_draw_is_reproducible_and_seed_dependent():
    sp = wl.spec(0)
    a, b = wl.draw(sp), wl.draw(sp)
    for f in ("x", "dz", "gamma", "beta"):
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))
    c = wl.draw(sp.with_(seed=sp.seed + 1))
    assert not np.array_equal(a.x, c.x)


def test_value_distributions():
    sp = wl.spec(1).with_(n=16, h=14, w=14)
    inp = wl.draw(sp)
    x = wl.logical_view(inp.x64, sp.shape, sp.layout)
    mean_c = x.mean(axis=(0, 2, 3))
    std_c = x.std(axis=(0, 2, 3))
    assert np.all(np.abs(mean_c) < 2.0 + 4 * std_c / np.sqrt(16 * 14 * 14))
    assert np.all((std_c > 0.4) & (std_c < 3.2))
    g = inp.gamma.astype(np.float64)
    assert np.all((np.abs(g) >= 0.5) & (np.abs(g) <= 1.5))
    assert (g < 0).any() and (g > 0).any()                       # random sign
    assert abs(inp.beta.std() - np.sqrt(0.1)) < 0.1               # variance 0.1
    dz = inp.dz64
    assert abs(dz.mean()) < 0.05 and abs(dz.std() - 1.0) < 0.05
    np.testing.assert_array_equal(inp.running_mean, 0.0)
    np.testing.assert_array_equal(inp.running_var, 1.0)
    # heavy tail of the segmentation workload: Student-t (nu = 3) has excess
    # kurtosis far above the normal's 0
    seg = wl.spec(2).with_(n=4, c=16, h=32, w=32)
    xs = wl.logical_view(wl.draw(seg).x64, seg.shape, seg.layout)
    e = (xs - xs.mean(axis=(0, 2, 3), keepdims=True)) / xs.std(axis=(0, 2, 3), keepdims=True)
    assert (e ** 4).mean() > 4.0
    many = wl.draw(wl.spec(3).with_(n=2))
    assert np.abs(many.gamma).min() >= 0.05


@pytest.mark.parametrize("dtype", [wl.F32, wl.BF16, wl.F16])
def test_storage_round_trip_is_exact(dtype):
    rng = np.random.default_rng(7)
    a = rng.standard_normal(4096) * 3
    s = wl.to_storage(a, dtype)
    back = wl.to_f64(s, dtype)
    np.testing.assert_array_equal(wl.to_storage(back, dtype), s)   # idempotent
    # unit roundoff: half an ulp, relative (24, 8 and 11 significand bits)
    ulp = {wl.F32: 2.0 ** -24, wl.BF16: 2.0 ** -8, wl.F16: 2.0 ** -11}[dtype]
    assert np.all(np.abs(back - a) <= np.abs(a) * ulp * 1.0000001 + 1e-300)


def test_layout_views_agree():
    rng = np.random.default_rng(3)
    logical = rng.standard_normal((2, 5, 3, 4))
    for layout in (wl.NCHW, wl.NHWC):
        flat = wl._arrange(logical, layout)
        np.testing.assert_array_equal(wl.logical_view(flat, logical.shape, layout), logical)
    nhwc = wl._arrange(logical, wl.NHWC).reshape(2, 3, 4, 5)
    assert nhwc[1, 2, 3, 4] == logical[1, 4, 2, 3]


def test_sweep_adapter_subsamples_and_cycles_channels():
    prev = wl.spec(4, 0).with_(n=2, c=4, h=8, w=8)
    nxt = wl.spec(4, 1).with_(n=2, c=6, h=4, w=4)
    z = np.arange(2 * 4 * 8 * 8, dtype=np.float64).reshape(2, 4, 8, 8)
    x = wl.sweep_adapter(z, nxt)
    assert x.shape == (2, 6, 4, 4)
    for c in range(6):
        np.testing.assert_array_equal(x[:, c], z[:, c % 4, ::2, ::2])


def _imports(path):
    tree = ast.parse(open(path).read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            names.add(node.module.split(".")[0])
    return names


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "place_batchnorm_activation_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                assert "oracle" not in _imports(os.path.join(dirpath, f)), f
            if f.endswith((".cu", ".cuh", ".h")):
                assert "oracle" not in open(os.path.join(dirpath, f)).read().lower(), f


def test_binding_fails_loudly_without_the_library(monkeypatch):
    import place_batchnorm_activation_b200 as iabn
    monkeypatch.setattr(iabn, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libiabn.so"))
    monkeypatch.setattr(iabn, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        iabn.workspace_size((2, 8, 4, 4), iabn.IABN_NHWC, iabn.IABN_BF16)
