"""Helpers for the GPU parity tests: run one layer through the C ABI (via the
binding) and through the fp64 oracle on the same seeded inputs, and compare
element by element.

Bound (|got - want| <= abs + rel*|want|): fp32 storage rel 1e-5 / abs 1e-6;
bf16 / fp16 storage rel 2e-2 / abs 1e-2.  This plain bound applies to every
forward output (z, mean, var, running statistics) and to the stage-separated
backward, where the GPU and the oracle read the same stored z bits.

The stage-separated backward adds to it the fp32 rounding noise of the
kernel's own arithmetic (``noise``), where the plain bound alone would ask
for more than fp32 can give: a per-channel sum of M terms that nearly
cancel, or a dx that is a small difference of large terms.  The model
(rounding errors of at most u = 2^-24 relative, independent from one
operation to the next):
  - dbeta = sum dy and dgamma = sum dy*xhat: every term is formed with a few
    fp32 roundings and then passes through a chain of at most L fp32
    additions before it is widened to fp64 (L from the launch plan, see
    fp32_chain_length), so the error is about u sqrt(L + 4) sqrt(sum w_i^2)
    with w_i the size of term i: |dz_i| for dbeta and
    |dz_i| (|xhat_i| + 2|beta_c|/|gamma_c|) for dgamma (the in-place
    kernels form dgamma = (sum dy*y - beta sum dy)/gamma, whose terms are
    dy*y = dy (gamma xhat + beta));
  - dx = A dy + B v + C (v = y or xhat): its three coefficients are rounded
    to fp32 and combined with two fused multiply-adds, so its error is about
    4u times the size of its terms, |gamma_c| rstd_c (|dz| + |dbeta_c|/M) +
    rstd_c |dgamma_c|/M (|gamma_c xhat| + 2|beta_c|), plus the noise of
    dbeta and dgamma carried through 1/M.
The noise allowed is KAPPA = 6 times that estimate.

Only the end-to-end chain (the GPU's own z feeds the GPU backward, the
oracle's z feeds the oracle backward) takes a wider relative scale, passed as
``scale``: there the two z may differ by one storage ulp wherever the
rounding of z was a near tie, and every such flip moves dx, dgamma and
dbeta.  For dx the scale is |gamma_c| rstd_c (|dz| + rms_c(dz)), the size of
the terms dx is the difference of; for dgamma = sum dy*xhat and dbeta =
sum dy it is the root-sum-square of their terms, sqrt(sum (dz*xhat)^2) and
sqrt(sum dz^2).

Every comparison records its worst ratio against the plain bound (and, when
a scale is given, against the bound it was held to); the test session
prints the closest ones at the end (see conftest.py), so a near miss is
visible in the log.

Guard bands: every device buffer of a GpuLayer sits between two 4 KiB bands
of a fixed byte pattern; the layer checks them after every call, so a write
past either end of an output, an input or the workspace fails the test.
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


U32 = 2.0 ** -24
KAPPA = 6.0

# (what, worst ratio under the plain bound, worst ratio under the bound applied,
#  kind: "plain", "noise" (stage-separated fp32 noise added) or "scale" (end to end))
RATIOS: list[tuple[str, float, float, str]] = []


def compare(got, want, dtype_or_tol, what="", scale=None, noise=None):
    """Element check; returns the worst ratio err / bound (<= 1 passes).
    ``scale`` (end-to-end comparisons only; same shape) replaces |want| in
    the relative term where it is larger; ``noise`` (stage-separated
    backward; same shape) is added to the bound."""
    rel, abs_ = TOL[dtype_or_tol] if isinstance(dtype_or_tol, int) else dtype_or_tol
    got = np.asarray(got, np.float64).reshape(-1)
    want = np.asarray(want, np.float64).reshape(-1)
    assert got.shape == want.shape, what
    nan_g, nan_w = np.isnan(got), np.isnan(want)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    ok = ~nan_w
    err = np.abs(got[ok] - want[ok])
    mag = np.abs(want[ok])
    plain = err / (abs_ + rel * mag)
    worst_plain = float(plain.max()) if plain.size else 0.0
    ratio = plain
    if scale is not None or noise is not None:
        if scale is not None:
            mag = np.maximum(mag, np.asarray(scale, np.float64).reshape(-1)[ok])
        extra = 0.0 if noise is None else np.asarray(noise, np.float64).reshape(-1)[ok]
        ratio = err / (abs_ + rel * mag + extra)
    worst = float(ratio.max()) if ratio.size else 0.0
    kind = "scale" if scale is not None else ("noise" if noise is not None else "plain")
    RATIOS.append((what, worst_plain, worst, kind))
    if worst > 1.0:
        k = int(np.argmax(ratio))
        idx = np.flatnonzero(ok)[k]
        raise AssertionError(f"{what}: {int((ratio > 1).sum())} of {ratio.size} elements out of "
                             f"tolerance; worst at {idx}: got {got[idx]!r} want {want[idx]!r}")
    return worst


GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """A device tensor of ``numel`` elements of ``dtype`` between two bands of
    GUARD_BYTE (4 KiB each, plus the padding up to a 16-byte multiple).  The
    tensor starts GUARD_BYTES into a fresh allocation, so it keeps the
    allocation's alignment."""

    def __init__(self, numel, dtype, device, fill=None):
        import torch
        item = torch.empty((), dtype=dtype).element_size()
        self.nbytes = numel * item
        body = (self.nbytes + 15) // 16 * 16
        self.raw = torch.full((GUARD_BYTES + body + GUARD_BYTES,), GUARD_BYTE,
                              dtype=torch.uint8, device=device)
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self) -> bool:
        head = self.raw[:GUARD_BYTES]
        tail = self.raw[GUARD_BYTES + self.nbytes:]
        return bool((head == GUARD_BYTE).all()) and bool((tail == GUARD_BYTE).all())


def fp32_chain_length(sp: wl.LayerSpec, call: int = 1) -> int:
    """The longest chain of fp32 additions a per-channel partial sum of the
    backward passes through before it is widened to fp64, as the plan the
    backward call takes partitions the work (its launch shape comes from
    iabn_describe_plan; the two-phase partition is the one its kernels
    document: NHWC rows of whole 16-byte vectors in blocks of 512 threads
    with fixed vector columns; other NHWC rows in blocks of 512 threads over
    256 columns and at most 256 row blocks, merged in a tree; NCHW planes of
    up to 1 KiB per 16-byte aligned group one thread per plane, larger ones
    one warp per plane)."""
    import math
    import place_batchnorm_activation_b200 as iabn
    n, c, h, w = sp.shape
    hw, rows = h * w, n * h * w
    plan = iabn.describe_plan(sp.shape, sp.layout, sp.dtype, call)
    if plan["plan"] == "resident":
        if sp.layout == wl.NHWC:
            rp = plan["row_phases"]
            return -(-(-(-rows // plan["grid"])) // rp) + rp
        lanes = 1
        if hw > 64:
            while lanes < 32 and lanes * 8 < hw:
                lanes *= 2
        return -(-hw // lanes) + int(math.log2(lanes))
    if sp.layout == wl.NHWC and (c * sp.itemsize) % 16 == 0:
        # 16-byte vector columns: 512 threads, W = min(VC, 512) columns, row
        # blocks a multiple of the SM count (at most 256) and at most the rows
        # over the row phases; the phases are added in fp32 one by one
        import torch
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        vc = c * sp.itemsize // 16
        rp = 512 // min(vc, 512)
        rb = min((256 // sms) * sms or 256, -(-rows // rp))
        return -(-(-(-rows // rb)) // rp) + rp
    if sp.layout == wl.NHWC:
        rb = min(rows, 256)
        rp = 512 // min(c, 256)
        return -(-(-(-rows // rb)) // rp) + int(math.ceil(math.log2(rp)))
    g = 16 // math.gcd(16, hw * sp.itemsize)
    if (n * c) % g == 0 and g * hw * sp.itemsize <= 1024:
        return hw + 1       # small planes: one thread sums a whole plane
    return -(-hw // 32) + 5


def backward_noise(exp: dict, sp: wl.LayerSpec) -> dict:
    """The fp32 noise allowance of the stage-separated backward (module
    docstring) for this layer under the plan its backward call takes."""
    root = np.sqrt(fp32_chain_length(sp) + 4.0)
    nb = KAPPA * U32 * root * exp["dbeta_mag"]
    ng = KAPPA * U32 * root * exp["dgamma_mag"]
    cb = lambda v: v[None, :, None, None]
    axh = np.abs(wl.logical_view(exp["xhat"], sp.shape, sp.layout))
    carried = wl._arrange(cb(exp["g_rstd_over_m"]) * (cb(nb) + axh * cb(ng)), sp.layout)
    return {"dx": KAPPA * U32 * 4.0 * exp["dx_mag"] + carried, "dgamma": ng, "dbeta": nb}


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
    # term sizes of the fp32 noise model (module docstring); |dy| <= |dz|
    # (every slope used is at most 1)
    M = sp.per_channel
    ag, ab = np.abs(g), np.abs(b)
    rstd = 1.0 / np.sqrt(var32 + eps)
    with np.errstate(divide="ignore", invalid="ignore"):
        bg = np.where(ag > 0, 2 * ab / ag, 0.0)
    dgamma_mag = np.sqrt(((dzl * (np.abs(xh) + bg[None, :, None, None])) ** 2).sum(axis=(0, 2, 3)))
    db_abs = np.abs(bw["dbeta"]) if np.isfinite(bw["dbeta"]).all() else np.nan_to_num(
        np.abs(bw["dbeta"]))
    dg_abs = np.nan_to_num(np.abs(bw["dgamma"]))
    cb = lambda v: v[None, :, None, None]
    dx_mag = wl._arrange(cb(ag * rstd) * (dzl + cb(db_abs / M))
                         + cb(rstd * dg_abs / M) * (cb(ag) * np.abs(xh) + cb(2 * ab)), sp.layout)
    return {"mean": fw["mean"], "var": fw["var"], "z": z, "var32": var32,
            "dx": oracle.round_to(bw["dx"], sp.dtype), "dx_scale": dx_scale,
            "dgamma": bw["dgamma"], "dbeta": bw["dbeta"], "dgamma_scale": dgamma_scale,
            "dbeta_scale": dbeta_scale, "running_mean": rm, "running_var": rv,
            "dgamma_mag": dgamma_mag, "dbeta_mag": dbeta_scale, "dx_mag": dx_mag,
            "g_rstd_over_m": ag * rstd / M, "xhat": fw["xhat"]}


class GpuLayer:
    """Device buffers of one layer and the calls of the C ABI on them.  Every
    buffer is guarded (see Guarded); each call checks all guards after it."""

    def __init__(self, inp: wl.LayerInputs, device="cuda"):
        import torch
        import place_batchnorm_activation_b200 as iabn
        self.iabn = iabn
        self.inp = inp
        sp = inp.spec
        self.sp = sp
        sdt = wl.torch_dtype(sp.dtype)
        nan = float("nan")
        self._g = {
            "x": Guarded(sp.numel, sdt, device, wl.storage_to_torch(inp.x, sp.dtype)),
            "dz": Guarded(sp.numel, sdt, device, wl.storage_to_torch(inp.dz, sp.dtype)),
            "gamma": Guarded(sp.c, torch.float32, device, torch.from_numpy(inp.gamma)),
            "beta": Guarded(sp.c, torch.float32, device, torch.from_numpy(inp.beta)),
            "mean": Guarded(sp.c, torch.float32, device, torch.full((sp.c,), nan)),
            "var": Guarded(sp.c, torch.float32, device, torch.full((sp.c,), nan)),
            "var_in": Guarded(sp.c, torch.float32, device, torch.full((sp.c,), nan)),
            "dgamma": Guarded(sp.c, torch.float32, device, torch.full((sp.c,), nan)),
            "dbeta": Guarded(sp.c, torch.float32, device, torch.full((sp.c,), nan)),
            "rmean": Guarded(sp.c, torch.float32, device, torch.from_numpy(inp.running_mean)),
            "rvar": Guarded(sp.c, torch.float32, device, torch.from_numpy(inp.running_var)),
            "ws": Guarded(iabn.workspace_size(sp.shape, sp.layout, sp.dtype), torch.uint8,
                          device, torch.zeros(1, dtype=torch.uint8)),
        }
        for k, g in self._g.items():
            setattr(self, k, g.t)

    def check_guards(self, what: str):
        import torch
        torch.cuda.synchronize()
        bad = [k for k, g in self._g.items() if not g.intact()]
        assert not bad, f"{self.sp.name} {what}: write outside the buffer(s) {bad}"

    def forward(self):
        sp = self.sp
        self.iabn.forward(self.x, self.gamma, self.beta, self.mean, self.var, self.ws,
                          shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act,
                          act_param=sp.act_param)
        self.check_guards("forward")

    def backward(self, z=None, var=None):
        """Backward from the activation buffer (z, or a given z tensor) and the
        layer's forward variance, or ``var`` (copied into a guarded buffer)."""
        sp = self.sp
        if var is not None:
            self.var_in.copy_(var)
            var = self.var_in
        self.iabn.backward(self.x if z is None else z, self.dz, self.gamma, self.beta,
                           self.var if var is None else var, self.dgamma, self.dbeta, self.ws,
                           shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act,
                           act_param=sp.act_param)
        self.check_guards("backward")

    def running(self):
        self.iabn.update_running_stats(self.mean, self.var, self.rmean, self.rvar,
                                       count=self.sp.per_channel, momentum=self.sp.momentum)
        self.check_guards("running statistics")

    def status(self) -> int:
        return self.iabn.get_device_status(self.ws)

    def host(self, t) -> np.ndarray:
        """Device storage tensor -> exact fp64 numpy."""
        return wl.to_f64(wl.torch_to_storage(t, self.sp.dtype), self.sp.dtype)

    def load_z(self, z64: np.ndarray):
        """Replace the activation buffer with given (storage-exact) values."""
        store = wl.to_storage(z64, self.sp.dtype)
        self.x.copy_(wl.storage_to_torch(store, self.sp.dtype).to(self.x.device))
        self.x_store = store
        return self.x

    def reset_dz(self):
        self.dz.copy_(wl.storage_to_torch(self.inp.dz, self.sp.dtype).to(self.dz.device))
