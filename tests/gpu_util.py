"""Helpers for the GPU parity tests: run one layer through the C ABI (via the
binding) and through the fp64 oracle on the same seeded inputs, and compare
element by element.

Tolerances (|got - want| <= abs + rel*|want|): fp32 storage rel 1e-5 /
abs 1e-6; bf16 / fp16 storage rel 2e-2 / abs 1e-2.  For dx the relative
part is taken against max(|want|, s) where s = |gamma_c| rstd_c (|dz| +
rms_c(dz)) is the size of the terms dx is the difference of
(dx = gamma rstd (dy - mean dy - xhat mean(dy xhat))): with few values per
channel those terms cancel almost completely (for M = 2, dx is
eps/(var+eps) times them) and no fp32 evaluation can meet a bound relative
to the tiny difference.  Likewise dgamma = sum dy*xhat and dbeta = sum dy
are compared relative to max(|want|, sqrt(sum (dz*xhat)^2)) and
max(|want|, sqrt(sum dz^2)) -- the root-sum-square of their terms (|phi'| <= 1)
-- because a one-ulp difference in each stored z moves a near-cancelling sum
by about that much times the storage rounding.
"""
from __future__ import annotations

import contextlib
import functools
import os

import numpy as np

import oracle
import workloads as wl

TOL = {wl.F32: (1e-5, 1e-6), wl.BF16: (2e-2, 1e-2), wl.F16: (2e-2, 1e-2)}
PLANS = ("twophase", "resident")


@contextlib.contextmanager
def forced_plan(plan: str | None):
    old = os.environ.get("IABN_FORCE_PLAN")
    if plan is None:
        os.environ.pop("IABN_FORCE_PLAN", None)
    else:
        os.environ["IABN_FORCE_PLAN"] = plan
    try:
        yield
    finally:
        if old is None:
            os.environ.pop("IABN_FORCE_PLAN", None)
        else:
            os.environ["IABN_FORCE_PLAN"] = old


def f32(v) -> float:
    """The float32 value the C ABI receives, as an exact double."""
    return float(np.float32(v))


def compare(got, want, dtype_or_tol, what="", scale=None):
    """Element check; returns the worst ratio err / bound (<= 1 passes).
    ``scale`` (optional, same shape) replaces |want| in the relative term
    where it is larger."""
    rel, abs_ = TOL[dtype_or_tol] if isinstance(dtype_or_tol, int) else dtype_or_tol
    got = np.asarray(got, np.float64).reshape(-1)
    want = np.asarray(want, np.float64).reshape(-1)
    assert got.shape == want.shape, what
    nan_g, nan_w = np.isnan(got), np.isnan(want)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    ok = ~nan_w
    err = np.abs(got[ok] - want[ok])
    mag = np.abs(want[ok])
    if scale is not None:
        mag = np.maximum(mag, np.asarray(scale, np.float64).reshape(-1)[ok])
    bound = abs_ + rel * mag
    ratio = err / bound
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        k = int(np.argmax(ratio))
        idx = np.flatnonzero(ok)[k]
        raise AssertionError(f"{what}: {int((ratio > 1).sum())} of {ratio.size} elements out of "
                             f"tolerance; worst at {idx}: got {got[idx]!r} want {want[idx]!r}")
    return worst


@functools.lru_cache(maxsize=4)
def oracle_sweep_inputs():
    """The layer sweep's chained inputs, built from the oracle's own rounded
    z of each layer (never from the GPU)."""
    layers = []
    x_logical = None
    for l in range(len(wl.SWEEP_SHAPES)):
        sp = wl.spec(4, l)
        inp = wl.draw(sp, x_logical=x_logical)
        exp = oracle_expect(inp)
        layers.append((inp, exp))
        z_logical = wl.logical_view(exp["z"], sp.shape, sp.layout)
        if l + 1 < len(wl.SWEEP_SHAPES):
            x_logical = wl.sweep_adapter(z_logical, wl.spec(4, l + 1))
    return layers


def oracle_expect(inp: wl.LayerInputs) -> dict:
    """Oracle results for one layer: the forward on x, and the in-place
    backward on the oracle's own rounded z and fp32 variance."""
    sp = inp.spec
    g = inp.gamma.astype(np.float64)
    b = inp.beta.astype(np.float64)
    eps, p = f32(sp.eps), f32(sp.act_param)
    fw = oracle.forward(sp.shape, sp.layout, inp.x64, g, b, eps, sp.act, p, want_xhat_y=True)
    z = oracle.round_to(fw["z"], sp.dtype)
    var32 = oracle.round_to(fw["var"], oracle.F32)
    bw = oracle.backward_inplace(sp.shape, sp.layout, z, inp.dz64, g, b, var32, eps, sp.act, p)
    rm, rv = oracle.running_update(sp.per_channel, fw["mean"], fw["var"], f32(sp.momentum),
                                   inp.running_mean, inp.running_var)
    # size of the terms of dx (tolerance scale only; see the module docstring)
    dzl = wl.logical_view(np.abs(inp.dz64), sp.shape, sp.layout)
    rms = np.sqrt((dzl ** 2).mean(axis=(0, 2, 3)))
    term = (np.abs(g) / np.sqrt(var32 + eps))[None, :, None, None] * (dzl + rms[None, :, None, None])
    dx_scale = wl._arrange(term, sp.layout)
    xh = wl.logical_view(fw["xhat"], sp.shape, sp.layout)
    dgamma_scale = np.sqrt(((dzl * xh) ** 2).sum(axis=(0, 2, 3)))
    dbeta_scale = np.sqrt((dzl ** 2).sum(axis=(0, 2, 3)))
    return {"mean": fw["mean"], "var": fw["var"], "z": z, "var32": var32,
            "dx": oracle.round_to(bw["dx"], sp.dtype), "dx_scale": dx_scale,
            "dgamma": bw["dgamma"], "dbeta": bw["dbeta"], "dgamma_scale": dgamma_scale,
            "dbeta_scale": dbeta_scale, "running_mean": rm, "running_var": rv}


class GpuLayer:
    """Device buffers of one layer and the calls of the C ABI on them."""

    def __init__(self, inp: wl.LayerInputs, device="cuda"):
        import torch
        import place_batchnorm_activation_b200 as iabn
        self.iabn = iabn
        self.inp = inp
        sp = inp.spec
        self.sp = sp
        self.x = wl.storage_to_torch(inp.x, sp.dtype).to(device)
        self.dz = wl.storage_to_torch(inp.dz, sp.dtype).to(device)
        self.gamma = torch.from_numpy(inp.gamma).to(device)
        self.beta = torch.from_numpy(inp.beta).to(device)
        self.mean = torch.full((sp.c,), float("nan"), device=device)
        self.var = torch.full((sp.c,), float("nan"), device=device)
        self.dgamma = torch.full((sp.c,), float("nan"), device=device)
        self.dbeta = torch.full((sp.c,), float("nan"), device=device)
        self.rmean = torch.from_numpy(inp.running_mean).to(device)
        self.rvar = torch.from_numpy(inp.running_var).to(device)
        self.ws = iabn.new_workspace(sp.shape, sp.layout, sp.dtype, device=device)

    def forward(self):
        sp = self.sp
        self.iabn.forward(self.x, self.gamma, self.beta, self.mean, self.var, self.ws,
                          shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act,
                          act_param=sp.act_param)

    def backward(self, z=None, var=None):
        sp = self.sp
        self.iabn.backward(self.x if z is None else z, self.dz, self.gamma, self.beta,
                           self.var if var is None else var, self.dgamma, self.dbeta, self.ws,
                           shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act,
                           act_param=sp.act_param)

    def running(self):
        self.iabn.update_running_stats(self.mean, self.var, self.rmean, self.rvar,
                                       count=self.sp.per_channel, momentum=self.sp.momentum)

    def status(self) -> int:
        return self.iabn.get_device_status(self.ws)

    def host(self, t) -> np.ndarray:
        """Device storage tensor -> exact fp64 numpy."""
        return wl.to_f64(wl.torch_to_storage(t, self.sp.dtype), self.sp.dtype)

    def load_z(self, z64: np.ndarray):
        """Replace the activation buffer with given (storage-exact) values."""
        import torch
        store = wl.to_storage(z64, self.sp.dtype)
        self.x.copy_(wl.storage_to_torch(store, self.sp.dtype).to(self.x.device))
        self.x_store = store
        return self.x

    def reset_dz(self):
        self.dz.copy_(wl.storage_to_torch(self.inp.dz, self.sp.dtype).to(self.dz.device))
