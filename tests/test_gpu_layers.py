"""GPU parity of the two layers InPlace-ABN is measured against, through the
C ABI, against the fp64 oracle on the same seeded inputs:

  * the standard BN+ACT layer, which keeps x and z ("Standard and
    Checkpointed Computation"): iabn_forward_standard (x kept, z to its own
    buffer) and iabn_backward_standard (from x and the saved statistics);
  * the optimized-checkpointing layer, which keeps xhat ("Proposed
    Checkpointing"): iabn_forward_checkpoint (xhat over x, z to its own
    buffer), iabn_checkpoint_recompute (z from xhat) and
    iabn_backward_checkpoint (from xhat).

Forward outputs (z, xhat, mean, var) are held to the plain bound.  The
backward adds the fp32 rounding noise of the kernel's own summation order
(gpu_util), with the term sizes of these layers: dgamma sums dy*xhat, where
the standard layer forms xhat = x*rstd - mean*rstd from x (|dz| (|xhat| +
2|mean| rstd)) and the checkpointing layer reads it (|dz| |xhat|).

Both recompute y and decide the activation's branch on it in fp32; the
oracle decides in fp64.  Where |y| is within the fp32 evaluation error of
zero both branches are correct readings: such elements (a handful per
million) are left out of the dx comparison and their largest possible
effect on dgamma and dbeta is added to those bounds.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_util import KAPPA, PLANS, TOL, U32, Guarded, compare, f32, forced_plan, \
    fp32_chain_length

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import place_batchnorm_activation_b200 as iabn  # noqa: E402

CALL_BWD_STANDARD, CALL_BWD_CHECKPOINT = 3, 5


class Buffers:
    """Guarded device buffers of one layer call sequence."""

    def __init__(self, inp):
        sp = inp.spec
        self.sp = sp
        dev = "cuda"
        sdt = wl.torch_dtype(sp.dtype)
        nan = float("nan")
        f = torch.float32
        self.g = {
            "x": Guarded(sp.numel, sdt, dev, wl.storage_to_torch(inp.x, sp.dtype)),
            "z": Guarded(sp.numel, sdt, dev, torch.zeros(1, dtype=sdt)),
            "dz": Guarded(sp.numel, sdt, dev, wl.storage_to_torch(inp.dz, sp.dtype)),
            "gamma": Guarded(sp.c, f, dev, torch.from_numpy(inp.gamma)),
            "beta": Guarded(sp.c, f, dev, torch.from_numpy(inp.beta)),
            "mean": Guarded(sp.c, f, dev, torch.full((sp.c,), nan)),
            "var": Guarded(sp.c, f, dev, torch.full((sp.c,), nan)),
            "mean_in": Guarded(sp.c, f, dev, torch.full((sp.c,), nan)),
            "var_in": Guarded(sp.c, f, dev, torch.full((sp.c,), nan)),
            "dgamma": Guarded(sp.c, f, dev, torch.full((sp.c,), nan)),
            "dbeta": Guarded(sp.c, f, dev, torch.full((sp.c,), nan)),
            "ws": Guarded(iabn.workspace_size(sp.shape, sp.layout, sp.dtype), torch.uint8, dev,
                          torch.zeros(1, dtype=torch.uint8)),
        }
        for k, v in self.g.items():
            setattr(self, k, v.t)
        self.kw = dict(shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act,
                       act_param=sp.act_param)

    def check(self, what):
        torch.cuda.synchronize()
        bad = [k for k, v in self.g.items() if not v.intact()]
        assert not bad, f"{self.sp.name} {what}: write outside the buffer(s) {bad}"
        assert iabn.get_device_status(self.ws) == 0

    def host(self, t):
        return wl.to_f64(wl.torch_to_storage(t, self.sp.dtype), self.sp.dtype)

    def load(self, t, values64):
        t.copy_(wl.storage_to_torch(wl.to_storage(values64, self.sp.dtype), self.sp.dtype)
                .to(t.device))


def _cb(v):
    return v[None, :, None, None]


def backward_noise(sp, call, dz64, xhat, mean, rstd, g, dgamma, dbeta, ambiguous):
    """fp32 noise allowance of a standard / checkpointing backward (see the
    module docstring and gpu_util): per-channel for dgamma and dbeta,
    per-element for dx; plus the ambiguous elements' largest effect."""
    dzl = np.abs(wl.logical_view(dz64, sp.shape, sp.layout))
    axh = np.abs(wl.logical_view(xhat, sp.shape, sp.layout))
    shift = 2 * np.abs(mean) * rstd if call == CALL_BWD_STANDARD else np.zeros(sp.c)
    root = np.sqrt(fp32_chain_length(sp, call) + 4.0)
    M = sp.per_channel
    amb = wl.logical_view(ambiguous, sp.shape, sp.layout)
    extra_b = (dzl * amb).sum(axis=(0, 2, 3))
    extra_g = (dzl * (axh + _cb(shift)) * amb).sum(axis=(0, 2, 3))
    nb = KAPPA * U32 * root * np.sqrt((dzl ** 2).sum(axis=(0, 2, 3))) + extra_b
    ng = KAPPA * U32 * root * np.sqrt(((dzl * (axh + _cb(shift))) ** 2).sum(axis=(0, 2, 3))) \
        + extra_g
    A = np.abs(g) * rstd
    T = _cb(A) * (dzl + _cb(np.abs(dbeta) / M)) \
        + _cb(A * np.abs(dgamma) / M) * (axh + _cb(shift))
    ndx = KAPPA * U32 * 4.0 * T + _cb(A / M) * (_cb(nb) + (axh + _cb(shift)) * _cb(ng))
    return wl._arrange(ndx, sp.layout), ng, nb


def ambiguous_branch(sp, y64, y_terms):
    """Elements whose activation branch fp32 may decide either way."""
    if sp.act == wl.IDENTITY:
        return np.zeros(y64.shape, bool)
    return np.abs(y64) <= 16 * U32 * y_terms


def check_standard(inp, plan):
    sp = inp.spec
    tol = TOL[sp.dtype]
    g, b = inp.gamma.astype(np.float64), inp.beta.astype(np.float64)
    eps, p = f32(sp.eps), f32(sp.act_param)
    fw = oracle.forward(sp.shape, sp.layout, inp.x64, g, b, eps, sp.act, p, want_xhat_y=True)
    bw = oracle.backward_standard(sp.shape, sp.layout, inp.x64, inp.dz64, g, b, eps, sp.act, p)
    with forced_plan(plan):
        B = Buffers(inp)
        iabn.forward_standard(B.x, B.z, B.gamma, B.beta, B.mean, B.var, B.ws, **B.kw)
        B.check("forward_standard")
        compare(B.host(B.z), oracle.round_to(fw["z"], sp.dtype), sp.dtype, f"{sp.name} std z")
        compare(B.mean.cpu().numpy(), fw["mean"], tol, f"{sp.name} std mean")
        compare(B.var.cpu().numpy(), fw["var"], tol, f"{sp.name} std var")
        np.testing.assert_array_equal(wl.torch_to_storage(B.x, sp.dtype), inp.x)   # x kept
        # backward from x with the forward's own saved statistics
        iabn.backward_standard(B.x, B.dz, B.gamma, B.beta, B.mean, B.var, B.dgamma, B.dbeta,
                               B.ws, **B.kw)
        B.check("backward_standard")
        np.testing.assert_array_equal(wl.torch_to_storage(B.x, sp.dtype), inp.x)
        mean32 = B.mean.cpu().numpy().astype(np.float64)
        rstd = 1.0 / np.sqrt(fw["var"] + eps)
        xl = np.abs(wl.logical_view(inp.x64, sp.shape, sp.layout))
        y_terms = wl._arrange(_cb(np.abs(g) * rstd) * (xl + _cb(np.abs(mean32)))
                              + _cb(np.abs(b)), sp.layout)
        amb = ambiguous_branch(sp, fw["y"], y_terms)
        assert amb.mean() < 1e-4, f"{sp.name}: {int(amb.sum())} elements near y = 0"
        ndx, ng, nb = backward_noise(sp, CALL_BWD_STANDARD, inp.dz64, fw["xhat"], mean32, rstd,
                                     g, bw["dgamma"], bw["dbeta"], amb)
        dx = B.host(B.dz)
        keep = ~amb
        compare(dx[keep], oracle.round_to(bw["dx"], sp.dtype)[keep], sp.dtype,
                f"{sp.name} std dx", noise=ndx[keep])
        compare(B.dgamma.cpu().numpy(), bw["dgamma"], tol, f"{sp.name} std dgamma", noise=ng)
        compare(B.dbeta.cpu().numpy(), bw["dbeta"], tol, f"{sp.name} std dbeta", noise=nb)


def check_checkpoint(inp, plan):
    sp = inp.spec
    tol = TOL[sp.dtype]
    g, b = inp.gamma.astype(np.float64), inp.beta.astype(np.float64)
    eps, p = f32(sp.eps), f32(sp.act_param)
    fw = oracle.forward(sp.shape, sp.layout, inp.x64, g, b, eps, sp.act, p, want_xhat_y=True)
    xhat_s = oracle.round_to(fw["xhat"], sp.dtype)      # what the layer stores
    var32 = oracle.round_to(fw["var"], oracle.F32)
    with forced_plan(plan):
        B = Buffers(inp)
        iabn.forward_checkpoint(B.x, B.z, B.gamma, B.beta, B.mean, B.var, B.ws, **B.kw)
        B.check("forward_checkpoint")
        compare(B.host(B.x), xhat_s, sp.dtype, f"{sp.name} ckpt xhat")
        compare(B.host(B.z), oracle.round_to(fw["z"], sp.dtype), sp.dtype, f"{sp.name} ckpt z")
        compare(B.mean.cpu().numpy(), fw["mean"], tol, f"{sp.name} ckpt mean")
        compare(B.var.cpu().numpy(), fw["var"], tol, f"{sp.name} ckpt var")
        # stage-separated from here on: both sides read the oracle's stored xhat
        B.load(B.x, xhat_s)
        B.z.zero_()
        iabn.checkpoint_recompute(B.x, B.z, B.gamma, B.beta, shape=sp.shape, layout=sp.layout,
                                  act=sp.act, act_param=sp.act_param)
        B.check("checkpoint_recompute")
        zr = oracle.checkpoint_recompute(sp.shape, sp.layout, xhat_s, g, b, sp.act, p)
        compare(B.host(B.z), oracle.round_to(zr, sp.dtype), sp.dtype, f"{sp.name} ckpt recompute z")
        B.var_in.copy_(torch.from_numpy(var32.astype(np.float32)))
        iabn.backward_checkpoint(B.x, B.dz, B.gamma, B.beta, B.var_in, B.dgamma, B.dbeta, B.ws,
                                 **B.kw)
        B.check("backward_checkpoint")
        np.testing.assert_array_equal(B.host(B.x), xhat_s)                 # xhat kept
        bw = oracle.backward_checkpoint(sp.shape, sp.layout, xhat_s, inp.dz64, g, b, var32, eps,
                                        sp.act, p)
        xl = np.abs(wl.logical_view(xhat_s, sp.shape, sp.layout))
        y64 = wl._arrange(_cb(g) * wl.logical_view(xhat_s, sp.shape, sp.layout) + _cb(b),
                          sp.layout)
        y_terms = wl._arrange(_cb(np.abs(g)) * xl + _cb(np.abs(b)), sp.layout)
        amb = ambiguous_branch(sp, y64, y_terms)
        assert amb.mean() < 1e-4, f"{sp.name}: {int(amb.sum())} elements near y = 0"
        rstd = 1.0 / np.sqrt(var32 + eps)
        ndx, ng, nb = backward_noise(sp, CALL_BWD_CHECKPOINT, inp.dz64, xhat_s, np.zeros(sp.c),
                                     rstd, g, bw["dgamma"], bw["dbeta"], amb)
        dx = B.host(B.dz)
        keep = ~amb
        compare(dx[keep], oracle.round_to(bw["dx"], sp.dtype)[keep], sp.dtype,
                f"{sp.name} ckpt dx", noise=ndx[keep])
        compare(B.dgamma.cpu().numpy(), bw["dgamma"], tol, f"{sp.name} ckpt dgamma", noise=ng)
        compare(B.dbeta.cpu().numpy(), bw["dbeta"], tol, f"{sp.name} ckpt dbeta", noise=nb)


_inputs = {}


def inputs_for(workload):
    if workload not in _inputs:
        _inputs[workload] = wl.draw(wl.spec(workload))
    return _inputs[workload]


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("workload", [0, 1, 2, 3])
def test_standard_layer_parity(workload, plan):
    check_standard(inputs_for(workload), plan)


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("workload", [0, 1, 2, 3])
def test_checkpoint_layer_parity(workload, plan):
    check_checkpoint(inputs_for(workload), plan)


EDGE = [
    # (n, c, h, w, layout, dtype, act, param)
    (3, 1, 5, 7, wl.NCHW, wl.F32, wl.LEAKY_RELU, 0.01),
    (2, 3, 4, 5, wl.NHWC, wl.F32, wl.ELU, 0.5),          # ragged C: two-phase
    (5, 6, 1, 1, wl.NHWC, wl.F16, wl.LEAKY_RELU, 0.01),
    (1, 4, 1, 2, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),  # M = 2
    (4, 12, 3, 3, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01),
    (2, 16, 7, 7, wl.NCHW, wl.F16, wl.ELU, 1.0),
    (7, 40, 9, 11, wl.NHWC, wl.F16, wl.ELU, 1.0),
    (2, 300, 5, 5, wl.NCHW, wl.F16, wl.IDENTITY, 0.0),
    (16, 24, 13, 13, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),
    (32, 64, 31, 29, wl.NCHW, wl.F32, wl.ELU, 1.0),
    (8, 2048, 3, 3, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01),   # the widest one-column rows
    (8, 4096, 3, 3, wl.NHWC, wl.BF16, wl.ELU, 1.0),           # two columns: two-phase
    (8, 256, 14, 14, wl.NHWC, wl.BF16, wl.ELU, 1.0),          # Tensor Memory stash
    (64, 40, 3, 3, wl.NCHW, wl.F16, wl.ELU, 1.0),
]


def _edge_id(c):
    return ("x".join(map(str, c[:4])) + f"-{'nhwc' if c[4] else 'nchw'}-"
            f"{wl.DTYPE_NAMES[c[5]]}-{wl.ACT_NAMES[c[6]]}")


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("case", EDGE, ids=_edge_id)
def test_standard_layer_edge_shapes(case, plan):
    n, c, h, w, layout, dtype, act, p = case
    sp = wl.LayerSpec("std_edge", n, c, h, w, layout, dtype, act, p, seed=901 + n * c + h * w)
    check_standard(wl.draw(sp), plan)


@pytest.mark.parametrize("plan", PLANS)
@pytest.mark.parametrize("case", EDGE, ids=_edge_id)
def test_checkpoint_layer_edge_shapes(case, plan):
    n, c, h, w, layout, dtype, act, p = case
    sp = wl.LayerSpec("ckpt_edge", n, c, h, w, layout, dtype, act, p, seed=902 + n * c + h * w)
    check_checkpoint(wl.draw(sp), plan)


@pytest.mark.parametrize("plan", PLANS)
def test_statistics_stress_standard_and_checkpoint(plan):
    """fp32 NHWC with an outlier first row (30 sigma), resident-plan size."""
    sp = wl.LayerSpec("f32_outlier_layers", 32, 128, 28, 28, wl.NHWC, wl.F32, wl.LEAKY_RELU,
                      0.01, seed=20180615, first_row_outlier=30.0)
    inp = wl.draw(sp)
    check_standard(inp, plan)
    check_checkpoint(inp, plan)


def test_checkpoint_backward_with_zero_gamma():
    """Nothing is divided by gamma in the checkpointing backward: a channel
    with gamma = 0 gets finite gradients (dx = 0 there)."""
    sp = wl.LayerSpec("ckpt_zero_gamma", 4, 8, 5, 5, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01,
                      seed=77)
    inp = wl.draw(sp)
    inp.gamma[3] = 0.0
    check_checkpoint(inp, "resident")
    check_checkpoint(inp, "twophase")
