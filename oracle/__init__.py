"""Plain fp64 CPU oracle for In-Place Activated BatchNorm (ctypes wrapper).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and
the CPU-baseline leg of the benchmark may import this package.  It shares no
code with the CUDA library and never imports it.

The arithmetic lives in ``iabn_oracle.c`` (plain C, fp64); this module only
compiles it with gcc, loads it and marshals numpy arrays.  Sources and the
readings taken where the pages are silent are listed in ``iabn_oracle.h``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "iabn_oracle.c")
_HDR = os.path.join(_HERE, "iabn_oracle.h")
_LIB = os.path.join(_HERE, "libiabn_oracle.so")
# the same source built with -fopenmp: its channel loops run on all host cores
# (identical results; used only for the multi-core CPU baseline)
_LIB_OMP = os.path.join(_HERE, "libiabn_oracle_omp.so")

NCHW, NHWC = 0, 1
F32, BF16, F16 = 0, 1, 2
LEAKY_RELU, ELU, IDENTITY = 0, 1, 2

_lock = threading.Lock()
_libs = {}
_use_omp = False


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile the oracle into ``libiabn_oracle.so`` (gcc, -O2, strict IEEE),
    or with ``openmp`` into ``libiabn_oracle_omp.so`` (also -fopenmp)."""
    lib = _LIB_OMP if openmp else _LIB
    stale = (not os.path.exists(lib)) or any(
        os.path.getmtime(p) > os.path.getmtime(lib) for p in (_SRC, _HDR))
    if force or stale:
        tmp = lib + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", *(["-fopenmp"] if openmp else []), "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


def openmp(enabled: bool) -> None:
    """Route the calls below to the -fopenmp build (True) or the plain one."""
    global _use_omp
    _use_omp = bool(enabled)


def _load():
    with _lock:
        key = _use_omp
        if key not in _libs:
            lib = ctypes.CDLL(build(openmp=key))
            d, i64, i32 = ctypes.c_double, ctypes.c_int64, ctypes.c_int
            pd = ctypes.POINTER(ctypes.c_double)
            for name in ("orc_act", "orc_act_inv", "orc_act_deriv_from_y"):
                f = getattr(lib, name)
                f.argtypes = [d, i32, d]
                f.restype = d
            lib.orc_act_dy_from_z.argtypes = [d, d, i32, d]
            lib.orc_act_dy_from_z.restype = d
            lib.orc_round.argtypes = [pd, pd, i64, i32]
            lib.orc_round.restype = i32
            geom = [i64, i64, i64, i64, i32]
            lib.orc_forward.argtypes = geom + [pd, pd, pd, d, i32, d, pd, pd, pd, pd, pd]
            lib.orc_forward.restype = i32
            lib.orc_backward_standard.argtypes = geom + [pd, pd, pd, pd, d, i32, d, pd, pd, pd]
            lib.orc_backward_standard.restype = i32
            for name in ("orc_backward_inplace_1", "orc_backward_inplace_2"):
                f = getattr(lib, name)
                f.argtypes = geom + [pd, pd, pd, pd, pd, d, i32, d, pd, pd, pd]
                f.restype = i32
            lib.orc_backward_checkpoint.argtypes = geom + [pd, pd, pd, pd, pd, d, i32, d, pd,
                                                           pd, pd]
            lib.orc_backward_checkpoint.restype = i32
            lib.orc_checkpoint_recompute.argtypes = geom + [pd, pd, pd, i32, d, pd]
            lib.orc_checkpoint_recompute.restype = i32
            lib.orc_inference.argtypes = geom + [pd, pd, pd, pd, pd, d, i32, d, pd]
            lib.orc_inference.restype = i32
            lib.orc_running_update.argtypes = [i64, i64, pd, pd, d, pd, pd]
            lib.orc_running_update.restype = i32
            _libs[key] = lib
        return _libs[key]


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments")


# ------------------------------------------------------------------ scalars

def act(y: float, kind: int, p: float) -> float:
    return _load().orc_act(float(y), int(kind), float(p))


def act_inv(z: float, kind: int, p: float) -> float:
    return _load().orc_act_inv(float(z), int(kind), float(p))


def act_dy_from_z(z: float, dz: float, kind: int, p: float) -> float:
    return _load().orc_act_dy_from_z(float(z), float(dz), int(kind), float(p))


def act_deriv_from_y(y: float, kind: int, p: float) -> float:
    return _load().orc_act_deriv_from_y(float(y), int(kind), float(p))


def round_to(values, dtype: int) -> np.ndarray:
    """Round fp64 values to the storage type (RNE); exact doubles back."""
    src = _f64(values)
    out = np.empty_like(src)
    _check(_load().orc_round(_p(src), _p(out), src.size, int(dtype)), "round")
    return out


# ------------------------------------------------------------------ tensors

def forward(shape, layout, x, gamma, beta, eps, kind, p, *, want_xhat_y=False):
    """Returns dict(mean, var, z[, xhat, y]) in fp64; x in the given layout."""
    n, c, h, w = (int(v) for v in shape)
    x = _f64(x)
    g, b = _f64(gamma), _f64(beta)
    mean = np.empty(c)
    var = np.empty(c)
    z = np.empty_like(x)
    xhat = np.empty_like(x) if want_xhat_y else None
    y = np.empty_like(x) if want_xhat_y else None
    _check(_load().orc_forward(n, c, h, w, int(layout), _p(x), _p(g), _p(b), float(eps),
                               int(kind), float(p), _p(mean), _p(var), _p(xhat), _p(y), _p(z)),
           "forward")
    out = {"mean": mean, "var": var, "z": z}
    if want_xhat_y:
        out["xhat"], out["y"] = xhat, y
    return out


def backward_standard(shape, layout, x, dz, gamma, beta, eps, kind, p):
    n, c, h, w = (int(v) for v in shape)
    x, dz, g, b = _f64(x), _f64(dz), _f64(gamma), _f64(beta)
    dx = np.empty_like(x)
    dg = np.empty(c)
    db = np.empty(c)
    _check(_load().orc_backward_standard(n, c, h, w, int(layout), _p(x), _p(dz), _p(g), _p(b),
                                         float(eps), int(kind), float(p), _p(dx), _p(dg), _p(db)),
           "backward_standard")
    return {"dx": dx, "dgamma": dg, "dbeta": db}


def backward_inplace(shape, layout, z, dz, gamma, beta, var, eps, kind, p, form: int = 1):
    """INPLACE-ABN backward from z: ``form`` 1 (via xhat) or 2 (via y)."""
    n, c, h, w = (int(v) for v in shape)
    z, dz, g, b, v = _f64(z), _f64(dz), _f64(gamma), _f64(beta), _f64(var)
    dx = np.empty_like(z)
    dg = np.empty(c)
    db = np.empty(c)
    fn = {1: _load().orc_backward_inplace_1, 2: _load().orc_backward_inplace_2}[form]
    _check(fn(n, c, h, w, int(layout), _p(z), _p(dz), _p(g), _p(b), _p(v), float(eps),
              int(kind), float(p), _p(dx), _p(dg), _p(db)), f"backward_inplace_{form}")
    return {"dx": dx, "dgamma": dg, "dbeta": db}


def backward_checkpoint(shape, layout, xhat, dz, gamma, beta, var, eps, kind, p):
    """Optimized-checkpointing backward from the stored xhat (and dz)."""
    n, c, h, w = (int(v) for v in shape)
    xh, dz, g, b, v = _f64(xhat), _f64(dz), _f64(gamma), _f64(beta), _f64(var)
    dx = np.empty_like(xh)
    dg = np.empty(c)
    db = np.empty(c)
    _check(_load().orc_backward_checkpoint(n, c, h, w, int(layout), _p(xh), _p(dz), _p(g),
                                           _p(b), _p(v), float(eps), int(kind), float(p),
                                           _p(dx), _p(dg), _p(db)), "backward_checkpoint")
    return {"dx": dx, "dgamma": dg, "dbeta": db}


def checkpoint_recompute(shape, layout, xhat, gamma, beta, kind, p):
    """z = phi(gamma*xhat + beta) from the stored xhat (fp64)."""
    n, c, h, w = (int(v) for v in shape)
    xh, g, b = _f64(xhat), _f64(gamma), _f64(beta)
    z = np.empty_like(xh)
    _check(_load().orc_checkpoint_recompute(n, c, h, w, int(layout), _p(xh), _p(g), _p(b),
                                            int(kind), float(p), _p(z)), "checkpoint_recompute")
    return z


def inference(shape, layout, x, gamma, beta, running_mean, running_var, eps, kind, p):
    """Evaluation-mode z (fp64) from fixed statistics; x in the given layout."""
    n, c, h, w = (int(v) for v in shape)
    x, g, b = _f64(x), _f64(gamma), _f64(beta)
    rm, rv = _f64(running_mean), _f64(running_var)
    z = np.empty_like(x)
    _check(_load().orc_inference(n, c, h, w, int(layout), _p(x), _p(g), _p(b), _p(rm), _p(rv),
                                 float(eps), int(kind), float(p), _p(z)), "inference")
    return z


def running_update(count, mean, var, momentum, running_mean, running_var):
    """Returns updated (running_mean, running_var) copies."""
    mean, var = _f64(mean), _f64(var)
    rm, rv = _f64(running_mean).copy(), _f64(running_var).copy()
    _check(_load().orc_running_update(mean.size, int(count), _p(mean), _p(var), float(momentum),
                                      _p(rm), _p(rv)), "running_update")
    return rm, rv
