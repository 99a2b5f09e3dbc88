"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element, for every workload at full size and
for edge shapes, under both launch plans.

Forward: z (storage type), batch mean and biased variance.
Backward (stage-separated): both sides start from the oracle's own rounded z
and fp32 variance, so a one-ulp rounding flip in the forward is not blamed on
the backward.  End to end: the GPU forward feeds the GPU backward; the
oracle's chain feeds the oracle.
Bound |got - want| <= abs + rel*|want|, fp32 rel 1e-5 / abs 1e-6; bf16, fp16
rel 2e-2 / abs 1e-2, for the forward.  The stage-separated backward adds the
fp32 rounding noise of the kernel's own summation order (gpu_util); the
end-to-end outputs take the wider relative scale of gpu_util (one-ulp flips
of z).  Every comparison's worst ratio under the plain bound is printed at
the end of the session.
Every device buffer is guarded against writes past its ends (gpu_util).
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_util import PLANS, TOL, GpuLayer, backward_noise, compare, forced_plan, \
    oracle_expect, oracle_sweep_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

_cache = {}


def expect_for(workload):
    if workload not in _cache:
        inp = wl.draw(wl.spec(workload))
        _cache[workload] = (inp, oracle_expect(inp))
    return _cache[workload]


def check_layer(inp, exp, plan, *, running=False, e2e=True):
    sp = inp.spec
    tol = TOL[sp.dtype]
    with forced_plan(plan):
        L = GpuLayer(inp)
        # forward
        L.forward()
        if running:
            L.running()
        torch.cuda.synchronize()
        compare(L.host(L.x), exp["z"], sp.dtype, f"{sp.name} z")
        compare(L.mean.cpu().numpy(), exp["mean"], tol, f"{sp.name} mean")
        compare(L.var.cpu().numpy(), exp["var"], tol, f"{sp.name} var")
        if running:
            compare(L.rmean.cpu().numpy(), exp["running_mean"], tol, f"{sp.name} running_mean")
            compare(L.rvar.cpu().numpy(), exp["running_var"], tol, f"{sp.name} running_var")
        if e2e:
            # end to end: GPU z and GPU variance feed the GPU backward
            L.backward()
            torch.cuda.synchronize()
            compare(L.host(L.dz), exp["dx"], sp.dtype, f"{sp.name} e2e dx", exp["dx_scale"])
            compare(L.dgamma.cpu().numpy(), exp["dgamma"], tol, f"{sp.name} e2e dgamma",
                    exp["dgamma_scale"])
            compare(L.dbeta.cpu().numpy(), exp["dbeta"], tol, f"{sp.name} e2e dbeta",
                    exp["dbeta_scale"])
        # stage-separated backward from the oracle's z and variance
        z = L.load_z(exp["z"])
        L.reset_dz()
        var32 = torch.from_numpy(exp["var32"].astype(np.float32)).cuda()
        L.backward(z=z, var=var32)
        torch.cuda.synchronize()
        nz = backward_noise(exp, sp)
        compare(L.host(L.dz), exp["dx"], sp.dtype, f"{sp.name} dx", noise=nz["dx"])
        compare(L.dgamma.cpu().numpy(), exp["dgamma"], tol, f"{sp.name} dgamma",
                noise=nz["dgamma"])
        compare(L.dbeta.cpu().numpy(), exp["dbeta"], tol, f"{sp.name} dbeta", noise=nz["dbeta"])
        # z is read-only for the backward
        np.testing.assert_array_equal(L.host(L.x), exp["z"])
        assert L.status() == 0


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("workload", [0, 1, 2, 3])
def test_workload_parity(workload, plan):
    inp, exp = expect_for(workload)
    check_layer(inp, exp, plan, running=(workload == 1))


@pytest.mark.parametrize("plan", PLANS)
def test_layer_sweep_parity(plan):
    """All 16 layers of the layer sweep (full size), each from the oracle's
    chained input."""
    for inp, exp in oracle_sweep_inputs():
        check_layer(inp, exp, plan, e2e=False)


# fp32 NHWC layers whose per-channel statistics stress the summation: the
# resident plan's size (64x256x28x28, several tiles per CTA, ragged tile
# ends) with heavy tails (Student-t, 3 degrees of freedom) or with the
# first row of every channel 30 sigma away from the channel mean.
STATS_STRESS = [
    wl.LayerSpec("f32_nhwc_t3", 64, 256, 28, 28, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01,
                 seed=20180611, x_dist="student_t3"),
    wl.LayerSpec("f32_nhwc_outlier_row0", 64, 256, 28, 28, wl.NHWC, wl.F32, wl.LEAKY_RELU,
                 0.01, seed=20180612, first_row_outlier=30.0),
    wl.LayerSpec("f32_nhwc_outlier_row0_neg", 16, 96, 23, 29, wl.NHWC, wl.F32, wl.ELU, 1.0,
                 seed=20180613, first_row_outlier=-30.0),
    wl.LayerSpec("f32_nchw_t3_outlier", 32, 64, 19, 21, wl.NCHW, wl.F32, wl.LEAKY_RELU, 0.01,
                 seed=20180614, x_dist="student_t3", first_row_outlier=30.0),
]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("sp", STATS_STRESS, ids=lambda s: s.name)
def test_statistics_stress(sp, plan):
    inp = wl.draw(sp)
    check_layer(inp, oracle_expect(inp), plan, running=True)


EDGE = [
    # (n, c, h, w, layout, dtype, act, param)
    (3, 1, 5, 7, wl.NCHW, wl.F32, wl.LEAKY_RELU, 0.01),
    (3, 1, 5, 7, wl.NHWC, wl.BF16, wl.ELU, 1.0),
    (2, 3, 4, 5, wl.NHWC, wl.F32, wl.ELU, 0.5),
    (2, 3, 4, 5, wl.NCHW, wl.F16, wl.LEAKY_RELU, 0.2),
    (5, 6, 1, 1, wl.NCHW, wl.F32, wl.IDENTITY, 0.0),
    (5, 6, 1, 1, wl.NHWC, wl.F16, wl.LEAKY_RELU, 0.01),
    (1, 4, 1, 2, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),
    (1, 4, 2, 1, wl.NCHW, wl.BF16, wl.ELU, 1.0),
    (4, 12, 3, 3, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01),
    (4, 12, 3, 3, wl.NCHW, wl.F32, wl.ELU, 1.0),
    (2, 16, 7, 7, wl.NCHW, wl.F16, wl.ELU, 1.0),
    (2, 16, 7, 7, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),
    (7, 40, 9, 11, wl.NHWC, wl.F16, wl.ELU, 1.0),
    (7, 40, 9, 11, wl.NCHW, wl.BF16, wl.LEAKY_RELU, 0.01),
    (2, 300, 5, 5, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),
    (2, 300, 5, 5, wl.NCHW, wl.F16, wl.IDENTITY, 0.0),
    (1, 2, 1000, 37, wl.NCHW, wl.F32, wl.ELU, 1.0),
    (1, 2, 1000, 37, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01),
    (16, 24, 13, 13, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),
    (16, 24, 13, 13, wl.NCHW, wl.F32, wl.ELU, 1.0),
    (3, 8200, 2, 2, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01),
    (32, 64, 31, 29, wl.NHWC, wl.F32, wl.ELU, 1.0),
    (32, 64, 31, 29, wl.NCHW, wl.F32, wl.LEAKY_RELU, 0.01),
    (8, 8192, 3, 3, wl.NHWC, wl.BF16, wl.ELU, 1.0),
    (8, 4096, 3, 3, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),
    (8, 4104, 3, 3, wl.NHWC, wl.F16, wl.LEAKY_RELU, 0.01),
    (2, 1024, 1, 1, wl.NHWC, wl.BF16, wl.IDENTITY, 0.0),
    (64, 40, 3, 3, wl.NCHW, wl.F16, wl.ELU, 1.0),
    # NCHW forwards whose small planes get two or four lanes each (tiles of
    # 240 or 120 planes for the 480 consumer threads), several ragged tiles
    # per CTA, and one whose tile is rounded to whole rounds of planes
    (128, 512, 7, 7, wl.NCHW, wl.F32, wl.ELU, 1.0),
    (512, 128, 8, 8, wl.NCHW, wl.BF16, wl.LEAKY_RELU, 0.01),
    (640, 60, 8, 8, wl.NCHW, wl.F32, wl.IDENTITY, 0.0),
    (768, 96, 6, 6, wl.NCHW, wl.F16, wl.ELU, 1.0),
]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("case", EDGE, ids=lambda c: "x".join(map(str, c[:4])) +
                         f"-{'nhwc' if c[4] else 'nchw'}-{wl.DTYPE_NAMES[c[5]]}-"
                         f"{wl.ACT_NAMES[c[6]]}")
def test_edge_shapes(case, plan):
    n, c, h, w, layout, dtype, act, p = case
    sp = wl.LayerSpec("edge", n, c, h, w, layout, dtype, act, p, seed=777 + n * c + h * w)
    inp = wl.draw(sp)
    check_layer(inp, oracle_expect(inp), plan, running=True)


@pytest.mark.parametrize("plan", PLANS)
def test_deterministic(plan):
    """Bitwise-identical outputs over repeated calls (fixed reduction order)."""
    sp = wl.spec(1).with_(n=8)
    inp = wl.draw(sp)
    outs = []
    with forced_plan(plan):
        for _ in range(3):
            L = GpuLayer(inp)
            L.forward()
            L.backward()
            torch.cuda.synchronize()
            outs.append([wl.torch_to_storage(L.x, sp.dtype), wl.torch_to_storage(L.dz, sp.dtype),
                         L.mean.cpu().numpy(), L.var.cpu().numpy(), L.dgamma.cpu().numpy(),
                         L.dbeta.cpu().numpy()])
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("plan", PLANS)
def test_singular_gamma(plan):
    sp = wl.LayerSpec("singular", 4, 6, 5, 5, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01, seed=99)
    inp = wl.draw(sp)
    inp.gamma[2] = 0.0
    exp = oracle_expect(inp)
    with forced_plan(plan):
        L = GpuLayer(inp)
        L.forward()
        torch.cuda.synchronize()
        compare(L.host(L.x), exp["z"], sp.dtype, "z")
        assert L.status() == 0
        L.backward()
        import place_batchnorm_activation_b200 as iabn
        assert L.status() == iabn.IABN_ERR_SINGULAR_GAMMA
        assert L.status() == 0          # read clears it
        dx = wl.logical_view(L.host(L.dz), sp.shape, sp.layout)
        assert np.isnan(dx[:, 2]).all()
        assert np.isfinite(np.delete(dx, 2, axis=1)).all()
        dg = L.dgamma.cpu().numpy()
        assert np.isnan(dg[2]) and np.isfinite(np.delete(dg, 2)).all()


STASH_CASES = [
    # NHWC shapes whose resident plan keeps rows in Tensor Memory
    (8, 256, 14, 14, wl.BF16, wl.LEAKY_RELU, 0.01),   # 8 row phases, full stash
    (4, 512, 9, 9, wl.BF16, wl.ELU, 1.0),             # 4 row phases
    (3, 128, 10, 10, wl.F32, wl.LEAKY_RELU, 0.2),     # fp32, 8 row phases
    (6, 768, 7, 7, wl.BF16, wl.IDENTITY, 0.0),        # 2 row phases, two idle warps
    (2, 4096, 5, 5, wl.BF16, wl.LEAKY_RELU, 0.01),    # 2 columns per thread
    (8, 4104, 3, 3, wl.F16, wl.ELU, 1.0),             # 4 columns per thread, ragged
    (64, 256, 8, 8, wl.BF16, wl.LEAKY_RELU, 0.01),    # ~28 rows per CTA: partial stash
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", STASH_CASES, ids=lambda c: "x".join(map(str, c[:4])))
def test_tmem_stash_bitwise(case, monkeypatch):
    """Rows kept in Tensor Memory give the same bits as rows streamed back
    through L2 (the stash only changes where phase B reads them from), and
    both match the oracle."""
    n, c, h, w, dtype, act, p = case
    sp = wl.LayerSpec("stash", n, c, h, w, wl.NHWC, dtype, act, p, seed=4242 + c + n)
    inp = wl.draw(sp)
    outs = {}
    for on in ("1", "0"):
        monkeypatch.setenv("IABN_TMEM_STASH", on)
        with forced_plan("resident"):
            L = GpuLayer(inp)
            L.forward()
            L.backward()
            torch.cuda.synchronize()
            assert L.status() == 0
            outs[on] = [wl.torch_to_storage(L.x, sp.dtype), wl.torch_to_storage(L.dz, sp.dtype),
                        L.mean.cpu().numpy(), L.var.cpu().numpy(), L.dgamma.cpu().numpy(),
                        L.dbeta.cpu().numpy()]
    for a, b in zip(outs["1"], outs["0"]):
        np.testing.assert_array_equal(a, b)
    monkeypatch.setenv("IABN_TMEM_STASH", "1")
    check_layer(inp, oracle_expect(inp), "resident", running=False)


FUSED_RUNNING = [
    wl.spec(0),
    wl.LayerSpec("fused_running_nhwc", 8, 64, 28, 28, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01,
                 seed=20180640),
    wl.LayerSpec("fused_running_nchw", 6, 32, 7, 7, wl.NCHW, wl.F16, wl.ELU, 1.0,
                 seed=20180641),
]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("sp", FUSED_RUNNING, ids=lambda s: s.name)
def test_forward_with_running_stats(sp, plan):
    """The forward that updates the running statistics in its own finalize
    gives the bits of iabn_forward followed by iabn_update_running_stats, and
    the oracle's running update."""
    import place_batchnorm_activation_b200 as iabn
    inp = wl.draw(sp)
    exp = oracle_expect(inp)
    with forced_plan(plan):
        a, b = GpuLayer(inp), GpuLayer(inp)
        a.forward()
        a.running()
        iabn.forward_with_running_stats(b.x, b.gamma, b.beta, b.mean, b.var, b.rmean, b.rvar,
                                        b.ws, shape=sp.shape, layout=sp.layout, eps=sp.eps,
                                        act=sp.act, act_param=sp.act_param,
                                        momentum=sp.momentum)
        b.check_guards("forward with running statistics")
    torch.cuda.synchronize()
    for name in ("x", "mean", "var", "rmean", "rvar"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    tol = TOL[sp.dtype]
    compare(b.rmean.cpu().numpy(), exp["running_mean"], tol, f"{sp.name} fused running_mean")
    compare(b.rvar.cpu().numpy(), exp["running_var"], tol, f"{sp.name} fused running_var")
    assert b.status() == 0
