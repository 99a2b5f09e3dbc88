"""Pins for the fp64 oracle: each test checks it against something other than
itself -- hand-derived closed forms, library routines (numpy casts, PyTorch's
own batch_norm / activations / autograd in fp64), brute force, invariants of
batch normalisation, and central finite differences.

Method sources: "In-Place Activated BatchNorm for Memory-Optimized Training of
DNNs" (paperlayer.ai summary), section 3 ("Batch Normalization Review",
"INPLACE-ABN", "INPLACE-ABN II", "Standard and Checkpointed Computation") and
section 4 ("Experimental setup"); the batch-normalisation paper it cites
(Ioffe & Szegedy) for the statistics and the BN backward.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")
ACTS = [(oracle.LEAKY_RELU, 0.01), (oracle.ELU, 1.0), (oracle.IDENTITY, 0.0)]


def _rand_layer(rng, shape, layout, gamma_lo=0.5):
    n, c, h, w = shape
    mu = rng.uniform(-2, 2, c)
    sig = rng.uniform(0.5, 3, c)
    xl = mu[None, :, None, None] + sig[None, :, None, None] * rng.standard_normal(shape)
    g = np.where(rng.random(c) < 0.5, -1.0, 1.0) * rng.uniform(gamma_lo, 1.5, c)
    b = rng.normal(0, math.sqrt(0.1), c)
    dzl = rng.standard_normal(shape)
    return xl, g, b, dzl


def _flat(logical, layout):
    return wl._arrange(logical, layout)


def _torch_reference(xl, g, b, dzl, eps, act, p):
    """PyTorch fp64 autograd of batch_norm (training) followed by the activation."""
    x = torch.tensor(xl, dtype=torch.float64, requires_grad=True)
    gt = torch.tensor(g, dtype=torch.float64, requires_grad=True)
    bt = torch.tensor(b, dtype=torch.float64, requires_grad=True)
    y = torch.nn.functional.batch_norm(x, None, None, gt, bt, training=True, eps=eps)
    if act == oracle.LEAKY_RELU:
        z = torch.nn.functional.leaky_relu(y, p)
    elif act == oracle.ELU:
        z = torch.nn.functional.elu(y, p)
    else:
        z = y
    (z * torch.tensor(dzl, dtype=torch.float64)).sum().backward()
    var, mean = torch.var_mean(x.detach(), dim=(0, 2, 3), unbiased=False)
    return {"z": z.detach().numpy(), "mean": mean.numpy(), "var": var.numpy(),
            "dx": x.grad.numpy(), "dgamma": gt.grad.numpy(), "dbeta": bt.grad.numpy()}


def _close(a, b, rel, abs_=0.0):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape
    err = np.abs(a - b)
    bound = abs_ + rel * np.abs(b)
    bad = err > bound
    assert not bad.any(), f"max err {err.max():.3e}; worst at {np.argmax(err - bound)}"


# ------------------------------------------------------------------ rounding

@pytest.mark.parametrize("dtype,npt", [(oracle.F32, np.float32), (oracle.F16, np.float16)])
def test_round_matches_numpy_cast(dtype, npt):
    """numpy's float64 -> float32 / float16 casts round to nearest even directly."""
    rng = np.random.default_rng(1)
    info = np.finfo(npt)
    vals = [rng.standard_normal(20000) * s for s in (1e-3, 1.0, 1e3)]
    vals.append(rng.uniform(-1, 1, 5000) * float(info.tiny) * 4)       # subnormal range
    base = rng.standard_normal(5000).astype(npt)
    nxt = np.nextafter(base, np.array(np.inf, npt))
    vals.append((base.astype(np.float64) + nxt.astype(np.float64)) / 2)  # exact ties
    vals.append(np.array([float(info.max), float(info.max) * (1 + 2.0 ** -12),
                          -float(info.max) * 1.01, 0.0, -0.0, np.inf, -np.inf]))
    v = np.concatenate(vals)
    with np.errstate(over="ignore"):
        want = v.astype(npt).astype(np.float64)
    got = oracle.round_to(v, dtype)
    np.testing.assert_array_equal(got, want)
    assert np.isnan(oracle.round_to([np.nan], dtype)[0])


def test_round_bf16_brute_force():
    """bf16: nearest of all finite bf16 values (ties to the even significand)."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)                  # positive finite bf16
    table = (bits << np.uint32(16)).view(np.float32).astype(np.float64)
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        (table[1000:3000] + table[1001:3001]) / 2,       # exact ties
                        table[5000:5100]])
    a = np.abs(v)
    hi = np.clip(np.searchsorted(table, a), 1, table.size - 1)
    lo = hi - 1
    d_lo, d_hi = a - table[lo], table[hi] - a
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    want = np.copysign(table[pick], v)
    got = oracle.round_to(v, oracle.BF16)
    np.testing.assert_array_equal(got, want)
    assert oracle.round_to([3.5e38], oracle.BF16)[0] == np.inf


# --------------------------------------------------------------- activation

@pytest.mark.parametrize("act,p", [(oracle.LEAKY_RELU, 0.01), (oracle.LEAKY_RELU, 0.3),
                                   (oracle.ELU, 1.0), (oracle.ELU, 0.7)])
def test_activation_matches_torch_and_inverts(act, p):
    y = np.concatenate([np.linspace(-15, 15, 3001), [0.0, -1e-300, 1e-300]])
    z = np.array([oracle.act(v, act, p) for v in y])
    yt = torch.tensor(y, dtype=torch.float64)
    zt = (torch.nn.functional.leaky_relu(yt, p) if act == oracle.LEAKY_RELU
          else torch.nn.functional.elu(yt, p)).numpy()
    _close(z, zt, rel=1e-15, abs_=1e-300)
    back = np.array([oracle.act_inv(v, act, p) for v in z])
    if act == oracle.ELU:
        # d(phi^-1)/dz = 1/(z + alpha) = e^-y / alpha on the negative branch: one
        # rounding of z costs up to ulp(z) * e^-y / alpha in y.
        cond = np.where(y < 0, np.exp(-y) * np.abs(z) / p, 0.0)
        assert np.all(np.abs(back - y) <= 4 * 2.0 ** -53 * (np.abs(y) + cond) + 1e-300)
    else:
        _close(back, y, rel=4 * 2.0 ** -52, abs_=1e-300)
    # slope taken from z equals the textbook phi'(y)
    dz = np.linspace(-2, 2, y.size)
    a = np.array([oracle.act_dy_from_z(zv, d, act, p) for zv, d in zip(z, dz)])
    b = np.array([d * oracle.act_deriv_from_y(yv, act, p) for yv, d in zip(y, dz)])
    # z + alpha carries the rounding of z (absolute ulp(z) <= 2^-53 * alpha).
    _close(a, b, rel=1e-13, abs_=4 * 2.0 ** -53 * max(p, 1.0) * 2.0)


def test_activation_branch_at_zero_and_torch_slope():
    """Tie: phi'(0) is the negative-branch slope; PyTorch's autograd agrees."""
    for act, p in [(oracle.LEAKY_RELU, 0.01), (oracle.ELU, 1.0)]:
        y = torch.zeros(1, dtype=torch.float64, requires_grad=True)
        f = torch.nn.functional.leaky_relu if act == oracle.LEAKY_RELU else torch.nn.functional.elu
        f(y, p).sum().backward()
        assert oracle.act_deriv_from_y(0.0, act, p) == pytest.approx(float(y.grad[0]))
        assert oracle.act_inv(0.0, act, p) == 0.0


def test_elu_saturation_rule():
    floor = 2.0 ** -24
    assert oracle.act_inv(-1.0, oracle.ELU, 1.0) == math.log(floor)
    assert oracle.act_inv(-1.5, oracle.ELU, 1.5) == math.log(floor)
    assert oracle.act_dy_from_z(-1.0, 3.0, oracle.ELU, 1.0) == 0.0
    # just above the floor the plain inverse applies
    z = -1.0 + 2.0 ** -20
    assert oracle.act_inv(z, oracle.ELU, 1.0) == math.log1p(z)


# ---------------------------------------------------------------- forward

@pytest.mark.parametrize("layout", [oracle.NCHW, oracle.NHWC])
@pytest.mark.parametrize("act,p", ACTS)
def test_forward_matches_torch_batch_norm(layout, act, p):
    rng = np.random.default_rng(10 + layout)
    shape = (3, 5, 4, 6)
    xl, g, b, dzl = _rand_layer(rng, shape, layout)
    ref = _torch_reference(xl, g, b, dzl, 1e-5, act, p)
    out = oracle.forward(shape, layout, _flat(xl, layout), g, b, 1e-5, act, p)
    _close(out["mean"], ref["mean"], rel=1e-13, abs_=1e-15)
    _close(out["var"], ref["var"], rel=1e-13)
    _close(out["z"], _flat(ref["z"], layout), rel=1e-12, abs_=1e-14)


def test_forward_invariants():
    """Per channel: xhat has mean 0 and mean square var/(var+eps); a positive
    affine change of x with eps = 0 leaves z unchanged; channel permutation
    commutes with the layer; NCHW and NHWC agree."""
    rng = np.random.default_rng(11)
    shape = (4, 6, 3, 5)
    n, c, h, w = shape
    xl, g, b, _ = _rand_layer(rng, shape, oracle.NCHW)
    eps = 1e-3
    out = oracle.forward(shape, oracle.NCHW, _flat(xl, 0), g, b, eps, oracle.ELU, 1.0,
                         want_xhat_y=True)
    xh = out["xhat"].reshape(shape)
    np.testing.assert_allclose(xh.mean(axis=(0, 2, 3)), 0, atol=1e-13)
    np.testing.assert_allclose((xh ** 2).mean(axis=(0, 2, 3)),
                               out["var"] / (out["var"] + eps), rtol=1e-12)
    z0 = oracle.forward(shape, 0, _flat(xl, 0), g, b, 0.0, oracle.LEAKY_RELU, 0.01)["z"]
    z1 = oracle.forward(shape, 0, _flat(3.7 * xl - 11.0, 0), g, b, 0.0,
                        oracle.LEAKY_RELU, 0.01)["z"]
    np.testing.assert_allclose(z1, z0, rtol=1e-11, atol=1e-12)
    perm = rng.permutation(c)
    zp = oracle.forward(shape, 0, _flat(xl[:, perm], 0), g[perm], b[perm], eps,
                        oracle.LEAKY_RELU, 0.01)["z"].reshape(shape)
    zr = oracle.forward(shape, 0, _flat(xl, 0), g, b, eps, oracle.LEAKY_RELU, 0.01)["z"]
    np.testing.assert_array_equal(zp, zr.reshape(shape)[:, perm])
    znhwc = oracle.forward(shape, 1, _flat(xl, 1), g, b, eps, oracle.LEAKY_RELU, 0.01)["z"]
    np.testing.assert_array_equal(wl.logical_view(znhwc, shape, 1), zr.reshape(shape))


# -------------------------------------------------------------- inference

def _torch_inference(xl, g, b, rm, rv, eps, act, p):
    """PyTorch fp64 batch_norm in evaluation mode, then the activation."""
    y = torch.nn.functional.batch_norm(torch.tensor(xl), torch.tensor(rm), torch.tensor(rv),
                                       torch.tensor(g), torch.tensor(b), training=False,
                                       eps=eps)
    if act == oracle.LEAKY_RELU:
        return torch.nn.functional.leaky_relu(y, p).numpy()
    if act == oracle.ELU:
        return torch.nn.functional.elu(y, p).numpy()
    return y.numpy()


@pytest.mark.parametrize("layout", [oracle.NCHW, oracle.NHWC])
@pytest.mark.parametrize("act,p", ACTS)
def test_inference_matches_torch_eval_batch_norm(layout, act, p):
    rng = np.random.default_rng(40 + layout)
    shape = (3, 5, 4, 6)
    xl, g, b, _ = _rand_layer(rng, shape, layout)
    rm = rng.uniform(-2, 2, shape[1])
    rv = rng.uniform(0.25, 9, shape[1])
    ref = _torch_inference(xl, g, b, rm, rv, 1e-5, act, p)
    z = oracle.inference(shape, layout, _flat(xl, layout), g, b, rm, rv, 1e-5, act, p)
    _close(z, _flat(ref, layout), rel=1e-12, abs_=1e-14)


def test_inference_with_the_batch_statistics_is_the_training_forward():
    """Fed the batch's own mean and biased variance, evaluation mode gives
    the training-mode z bit for bit (same formula, same precision)."""
    rng = np.random.default_rng(42)
    for layout in (oracle.NCHW, oracle.NHWC):
        shape = (2, 7, 3, 5)
        xl, g, b, _ = _rand_layer(rng, shape, layout)
        for act, p in ACTS:
            fw = oracle.forward(shape, layout, _flat(xl, layout), g, b, 1e-5, act, p)
            z = oracle.inference(shape, layout, _flat(xl, layout), g, b, fw["mean"], fw["var"],
                                 1e-5, act, p)
            np.testing.assert_array_equal(z, fw["z"])


def test_inference_closed_forms():
    """Dyadic statistics make every step exact: with running_var + eps = 4
    the layer is z = phi(gamma*(x - m)/2 + beta) exactly; with m = 0, v = 1,
    eps = 0, gamma = 1 and beta = 0 it is phi itself."""
    rng = np.random.default_rng(43)
    shape = (2, 3, 2, 4)
    xl = rng.integers(-64, 64, shape) / 8.0
    for act, p in ((oracle.LEAKY_RELU, 0.25), (oracle.IDENTITY, 0.0)):
        g = np.array([1.0, -0.5, 2.0])
        b = np.array([0.25, 0.0, -1.0])
        m = np.array([0.5, -1.0, 0.0])
        v = np.array([3.75, 3.75, 3.75])
        z = oracle.inference(shape, oracle.NCHW, _flat(xl, 0), g, b, m, v, 0.25, act, p)
        y = g[None, :, None, None] * (xl - m[None, :, None, None]) / 2 + b[None, :, None, None]
        want = np.where(y > 0, y, p * y) if act == oracle.LEAKY_RELU else y
        np.testing.assert_array_equal(z.reshape(shape), want)
    one = np.ones(3)
    zero = np.zeros(3)
    z = oracle.inference(shape, oracle.NHWC, _flat(xl, 1), one, zero, zero, one, 0.0,
                         oracle.ELU, 1.0)
    np.testing.assert_array_equal(z, np.where(_flat(xl, 1) > 0, _flat(xl, 1),
                                              np.expm1(_flat(xl, 1))))


# --------------------------------------------------------------- backward

@pytest.mark.parametrize("layout", [oracle.NCHW, oracle.NHWC])
@pytest.mark.parametrize("act,p", ACTS)
def test_backward_standard_matches_torch_autograd(layout, act, p):
    rng = np.random.default_rng(20 + layout)
    shape = (3, 4, 5, 3)
    xl, g, b, dzl = _rand_layer(rng, shape, layout)
    ref = _torch_reference(xl, g, b, dzl, 1e-5, act, p)
    out = oracle.backward_standard(shape, layout, _flat(xl, layout), _flat(dzl, layout),
                                   g, b, 1e-5, act, p)
    scale = np.abs(ref["dx"]).max()
    _close(out["dx"], _flat(ref["dx"], layout), rel=1e-10, abs_=1e-12 * scale)
    _close(out["dgamma"], ref["dgamma"], rel=1e-10, abs_=1e-12)
    _close(out["dbeta"], ref["dbeta"], rel=1e-10, abs_=1e-12)


@pytest.mark.parametrize("layout", [oracle.NCHW, oracle.NHWC])
@pytest.mark.parametrize("act,p", ACTS + [(oracle.LEAKY_RELU, 0.2), (oracle.ELU, 0.5)])
def test_inplace_backward_equals_standard(layout, act, p):
    """INPLACE-ABN I and II, from the unrounded z alone, equal the standard
    backward from the stored x (the paper's central claim)."""
    rng = np.random.default_rng(30 + layout)
    shape = (5, 7, 3, 4)
    xl, g, b, dzl = _rand_layer(rng, shape, layout, gamma_lo=0.05)
    x, dz = _flat(xl, layout), _flat(dzl, layout)
    fw = oracle.forward(shape, layout, x, g, b, 1e-5, act, p)
    std = oracle.backward_standard(shape, layout, x, dz, g, b, 1e-5, act, p)
    for form in (1, 2):
        ip = oracle.backward_inplace(shape, layout, fw["z"], dz, g, b, fw["var"], 1e-5,
                                     act, p, form=form)
        scale = np.abs(std["dx"]).max()
        _close(ip["dx"], std["dx"], rel=1e-9, abs_=1e-10 * scale)
        _close(ip["dgamma"], std["dgamma"], rel=1e-9, abs_=1e-10)
        _close(ip["dbeta"], std["dbeta"], rel=1e-9, abs_=1e-10)


def _torch_xhat_var(xl, eps):
    """xhat = (x - mean)/sqrt(var + eps) and the biased variance, from PyTorch."""
    x = torch.tensor(xl, dtype=torch.float64)
    var, mean = torch.var_mean(x, dim=(0, 2, 3), unbiased=False)
    xh = (x - mean[None, :, None, None]) / torch.sqrt(var + eps)[None, :, None, None]
    return xh.numpy(), var.numpy()


@pytest.mark.parametrize("layout", [oracle.NCHW, oracle.NHWC])
@pytest.mark.parametrize("act,p", ACTS + [(oracle.LEAKY_RELU, 0.2)])
def test_checkpoint_backward_matches_torch_autograd(layout, act, p):
    """Optimized checkpointing: the backward from the stored xhat (here taken
    from PyTorch, not from the oracle's forward) gives PyTorch's autograd
    gradients of BN + activation with respect to x, gamma and beta."""
    rng = np.random.default_rng(60 + layout)
    shape = (3, 4, 5, 3)
    xl, g, b, dzl = _rand_layer(rng, shape, layout, gamma_lo=0.05)
    ref = _torch_reference(xl, g, b, dzl, 1e-5, act, p)
    xh, var = _torch_xhat_var(xl, 1e-5)
    out = oracle.backward_checkpoint(shape, layout, _flat(xh, layout), _flat(dzl, layout), g, b,
                                     var, 1e-5, act, p)
    scale = np.abs(ref["dx"]).max()
    _close(out["dx"], _flat(ref["dx"], layout), rel=1e-10, abs_=1e-12 * scale)
    _close(out["dgamma"], ref["dgamma"], rel=1e-10, abs_=1e-12)
    _close(out["dbeta"], ref["dbeta"], rel=1e-10, abs_=1e-12)
    z = oracle.checkpoint_recompute(shape, layout, _flat(xh, layout), g, b, act, p)
    _close(z, _flat(ref["z"], layout), rel=1e-12, abs_=1e-14)


@pytest.mark.parametrize("layout", [oracle.NCHW, oracle.NHWC])
@pytest.mark.parametrize("act,p", ACTS + [(oracle.ELU, 0.5)])
def test_checkpoint_backward_equals_standard(layout, act, p):
    """From the unrounded xhat, the checkpointing backward equals the standard
    backward from x, and the recomputed z is the forward's z bit for bit
    (same scale, shift and activation in the same precision)."""
    rng = np.random.default_rng(70 + layout)
    shape = (5, 7, 3, 4)
    xl, g, b, dzl = _rand_layer(rng, shape, layout, gamma_lo=0.05)
    x, dz = _flat(xl, layout), _flat(dzl, layout)
    fw = oracle.forward(shape, layout, x, g, b, 1e-5, act, p, want_xhat_y=True)
    std = oracle.backward_standard(shape, layout, x, dz, g, b, 1e-5, act, p)
    ck = oracle.backward_checkpoint(shape, layout, fw["xhat"], dz, g, b, fw["var"], 1e-5, act, p)
    scale = np.abs(std["dx"]).max()
    _close(ck["dx"], std["dx"], rel=1e-10, abs_=1e-11 * scale)
    _close(ck["dgamma"], std["dgamma"], rel=1e-10, abs_=1e-11)
    _close(ck["dbeta"], std["dbeta"], rel=1e-10, abs_=1e-11)
    z = oracle.checkpoint_recompute(shape, layout, fw["xhat"], g, b, act, p)
    np.testing.assert_array_equal(z, fw["z"])


def test_checkpoint_backward_needs_no_invertible_gamma():
    """The stored xhat carries what gamma = 0 would erase: the checkpointing
    backward stays finite there and matches PyTorch (dx = 0 for the channel)."""
    rng = np.random.default_rng(80)
    shape = (2, 3, 3, 2)
    xl, g, b, dzl = _rand_layer(rng, shape, oracle.NCHW)
    g[1] = 0.0
    ref = _torch_reference(xl, g, b, dzl, 1e-5, oracle.LEAKY_RELU, 0.01)
    xh, var = _torch_xhat_var(xl, 1e-5)
    out = oracle.backward_checkpoint(shape, 0, _flat(xh, 0), _flat(dzl, 0), g, b, var, 1e-5,
                                     oracle.LEAKY_RELU, 0.01)
    assert np.isfinite(out["dx"]).all() and np.isfinite(out["dgamma"]).all()
    assert np.all(out["dx"].reshape(shape)[:, 1] == 0.0)
    _close(out["dgamma"], ref["dgamma"], rel=1e-10, abs_=1e-12)


def test_bn_backward_invariants():
    """Per channel: sum dx = 0, and sum dx*xhat = gamma*rstd*dgamma*eps/(var+eps)
    (zero for eps = 0: the gradient is orthogonal to the directions that
    normalisation removes; with eps > 0, mean(xhat^2) = var/(var+eps) < 1)."""
    rng = np.random.default_rng(40)
    shape = (6, 5, 4, 4)
    xl, g, b, dzl = _rand_layer(rng, shape, oracle.NCHW)
    x, dz = _flat(xl, 0), _flat(dzl, 0)
    for eps in (0.0, 1e-5, 0.3):
        for act, p in ACTS:
            fw = oracle.forward(shape, 0, x, g, b, eps, act, p, want_xhat_y=True)
            ip = oracle.backward_inplace(shape, 0, fw["z"], dz, g, b, fw["var"], eps, act, p)
            dx = ip["dx"].reshape(shape)
            xh = fw["xhat"].reshape(shape)
            mag = np.abs(dx).sum(axis=(0, 2, 3)) * max(1.0, np.abs(xh).max())
            assert np.all(np.abs(dx.sum(axis=(0, 2, 3))) <= 1e-12 * mag)
            var = fw["var"]
            want = g / np.sqrt(var + eps) * ip["dgamma"] * eps / (var + eps)
            got = (dx * xh).sum(axis=(0, 2, 3))
            assert np.all(np.abs(got - want) <= 1e-12 * mag)


def test_finite_differences_tiny():
    """Central differences of L = sum dz*z on the tiny workload (leaky kink
    avoided) against the in-place backward."""
    sp = wl.spec(0)
    inp = wl.draw(sp)
    shape, lay = sp.shape, sp.layout
    g, b = inp.gamma.astype(np.float64), inp.beta.astype(np.float64)
    x, dz = inp.x64, inp.dz64
    act, p, eps = sp.act, sp.act_param, sp.eps

    def loss(xv, gv, bv):
        return float(np.dot(oracle.forward(shape, lay, xv, gv, bv, eps, act, p)["z"], dz))

    fw = oracle.forward(shape, lay, x, g, b, eps, act, p, want_xhat_y=True)
    ip = oracle.backward_inplace(shape, lay, fw["z"], dz, g, b, fw["var"], eps, act, p)
    rng = np.random.default_rng(41)
    picks = [k for k in rng.permutation(x.size) if abs(fw["y"][k]) > 1e-3][:120]
    for k in picks:
        h = 1e-6
        xp, xm = x.copy(), x.copy()
        xp[k] += h
        xm[k] -= h
        fd = (loss(xp, g, b) - loss(xm, g, b)) / (2 * h)
        assert fd == pytest.approx(ip["dx"][k], rel=1e-5, abs=1e-7)
    for ch in range(sp.c):
        for vec, key in ((g, "dgamma"), (b, "dbeta")):
            vp, vm = vec.copy(), vec.copy()
            vp[ch] += 1e-6
            vm[ch] -= 1e-6
            args_p = (x, vp, b) if key == "dgamma" else (x, g, vp)
            args_m = (x, vm, b) if key == "dgamma" else (x, g, vm)
            fd = (loss(*args_p) - loss(*args_m)) / 2e-6
            assert fd == pytest.approx(ip[key][ch], rel=1e-6, abs=1e-7)


def test_singular_gamma_gives_nan_for_that_channel_only():
    rng = np.random.default_rng(42)
    shape = (2, 3, 2, 2)
    xl, g, b, dzl = _rand_layer(rng, shape, 0)
    g[1] = 0.0
    fw = oracle.forward(shape, 0, _flat(xl, 0), g, b, 1e-5, oracle.LEAKY_RELU, 0.01)
    for form in (1, 2):
        ip = oracle.backward_inplace(shape, 0, fw["z"], _flat(dzl, 0), g, b, fw["var"], 1e-5,
                                     oracle.LEAKY_RELU, 0.01, form=form)
        dx = ip["dx"].reshape(shape)
        assert np.isnan(dx[:, 1]).all() and np.isfinite(dx[:, [0, 2]]).all()
        assert np.isnan(ip["dgamma"][1]) and np.isnan(ip["dbeta"][1])
        assert np.isfinite(ip["dgamma"][[0, 2]]).all()


# ------------------------------------------------------------ running stats

def test_running_update_matches_torch():
    rng = np.random.default_rng(50)
    shape = (4, 6, 3, 3)
    xl, g, b, _ = _rand_layer(rng, shape, 0)
    fw = oracle.forward(shape, 0, _flat(xl, 0), g, b, 1e-5, oracle.IDENTITY, 0.0)
    rm0, rv0 = rng.standard_normal(6), rng.uniform(0.5, 2, 6)
    rm_t, rv_t = torch.tensor(rm0), torch.tensor(rv0)
    torch.nn.functional.batch_norm(torch.tensor(xl), rm_t, rv_t, None, None, training=True,
                                   momentum=0.1, eps=1e-5)
    rm, rv = oracle.running_update(4 * 9, fw["mean"], fw["var"], 0.1, rm0, rv0)
    _close(rm, rm_t.numpy(), rel=1e-13, abs_=1e-15)
    _close(rv, rv_t.numpy(), rel=1e-13)


def test_running_update_closed_forms():
    # constant channel: var 0; two values +-d: biased d^2, unbiased d^2*M/(M-1)
    shape = (2, 2, 1, 2)
    xl = np.zeros(shape)
    xl[:, 0] = 3.25
    d = 1.5
    xl[:, 1, 0, 0], xl[:, 1, 0, 1] = -d, d
    fw = oracle.forward(shape, 0, _flat(xl, 0), np.ones(2), np.zeros(2), 1e-5,
                        oracle.IDENTITY, 0.0)
    assert fw["var"][0] == 0.0 and fw["mean"][0] == 3.25
    assert fw["var"][1] == d * d and fw["mean"][1] == 0.0
    rm, rv = oracle.running_update(4, fw["mean"], fw["var"], 0.25, [1.0, 1.0], [2.0, 2.0])
    assert rm.tolist() == [0.75 + 0.25 * 3.25, 0.75]
    assert rv.tolist() == [1.5, 1.5 + 0.25 * d * d * 4 / 3]


# ---------------------------------------------------------- hand examples

def _ev(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sqrt": math.sqrt, "exp": math.exp}))


def test_hand_derived_examples():
    cases = json.load(open(GOLDEN))["cases"]
    acts = {"leaky_relu": oracle.LEAKY_RELU, "elu": oracle.ELU, "identity": oracle.IDENTITY}
    for case in cases:
        shape = tuple(case["shape"])
        lay = {"NCHW": oracle.NCHW, "NHWC": oracle.NHWC}[case["layout"]]
        act, p, eps = acts[case["act"]], case["act_param"], case["eps"]
        e = {k: np.array([_ev(s) for s in v]) for k, v in case["expect"].items()}
        fw = oracle.forward(shape, lay, case["x"], case["gamma"], case["beta"], eps, act, p)
        for k in ("mean", "var", "z"):
            _close(fw[k], e[k], rel=1e-14, abs_=1e-15)
        std = oracle.backward_standard(shape, lay, case["x"], case["dz"], case["gamma"],
                                       case["beta"], eps, act, p)
        fwx = oracle.forward(shape, lay, case["x"], case["gamma"], case["beta"], eps, act, p,
                             want_xhat_y=True)
        ck = oracle.backward_checkpoint(shape, lay, fwx["xhat"], case["dz"], case["gamma"],
                                        case["beta"], fw["var"], eps, act, p)
        for form in (1, 2):
            ip = oracle.backward_inplace(shape, lay, fw["z"], case["dz"], case["gamma"],
                                         case["beta"], fw["var"], eps, act, p, form=form)
            for res in (std, ip, ck):
                for k in ("dx", "dgamma", "dbeta"):
                    _close(res[k], e[k], rel=1e-13, abs_=1e-14)
        rm, rv = oracle.running_update(shape[0] * shape[2] * shape[3], fw["mean"], fw["var"],
                                       case["momentum"], case["running_mean"], case["running_var"])
        _close(rm, e["running_mean"], rel=1e-14, abs_=1e-15)
        _close(rv, e["running_var"], rel=1e-14)


def test_openmp_build_gives_identical_bits():
    """The multi-core build of the oracle (same source with -fopenmp) splits
    only the loops over channels; every result is bit for bit the plain
    build's."""
    rng = np.random.default_rng(90)
    shape = (3, 9, 4, 5)
    layers = {lay: _rand_layer(rng, shape, lay) for lay in (oracle.NCHW, oracle.NHWC)}
    out = {}
    for omp in (False, True):
        oracle.openmp(omp)
        try:
            res = []
            for layout, (xl, g, b, dzl) in layers.items():
                x, dz = _flat(xl, layout), _flat(dzl, layout)
                fw = oracle.forward(shape, layout, x, g, b, 1e-5, oracle.ELU, 1.0, want_xhat_y=True)
                res += [fw["mean"], fw["var"], fw["z"], fw["xhat"]]
                res += list(oracle.backward_inplace(shape, layout, fw["z"], dz, g, b, fw["var"],
                                                    1e-5, oracle.ELU, 1.0).values())
                res += list(oracle.backward_standard(shape, layout, x, dz, g, b, 1e-5,
                                                     oracle.ELU, 1.0).values())
                res += list(oracle.backward_checkpoint(shape, layout, fw["xhat"], dz, g, b,
                                                       fw["var"], 1e-5, oracle.ELU, 1.0).values())
                res.append(oracle.round_to(fw["z"], oracle.BF16))
            out[omp] = res
        finally:
            oracle.openmp(False)
    assert len(out[False]) == len(out[True]) > 0
    for a, b in zip(out[False], out[True]):
        np.testing.assert_array_equal(a, b)
