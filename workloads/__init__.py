"""Seeded synthetic inputs for the InPlace-ABN layer (shared by tests and bench).

This module only draws random numbers and stores them in the storage type; it
holds none of the layer's arithmetic.  Neither the oracle nor the CUDA library
imports it; tests and the benchmark hand its arrays to both.

Workloads (all synthetic; the datasets the paper trains on are not used):

  0 tiny          NCHW fp32  N=2   C=8    H=W=16   leaky-ReLU 0.01
  1 resnet_trunk  NHWC bf16  N=64  C=256  H=W=56   leaky-ReLU 0.01 (+ running stats)
  2 segmentation  NHWC bf16  N=16  C=512  H=W=84   leaky-ReLU 0.01, Student-t(3) input
  3 many_channel  NCHW fp16  N=128 C=2048 H=W=7    ELU 1.0, |gamma| in [0.05, 1.5]
  4 layer_sweep   NHWC bf16  N=8, 16 layers of a WideResNet-38-like shape list,
                  even layers leaky-ReLU 0.01, odd layers ELU 1.0

Per channel c: mu_c ~ U(-2, 2), sigma_c ~ U(0.5, 3), x = mu_c + sigma_c * e with
e ~ N(0, 1) (Student-t with 3 degrees of freedom for workload 2);
gamma_c = s_c * U(0.5, 1.5) (U(0.05, 1.5) for workload 3) with s_c = +-1 at
probability 1/2; beta_c ~ N(0, variance 0.1); dz ~ N(0, 1); eps = 1e-5;
momentum = 0.1.  Generator: numpy PCG64 with seed 20180600 + workload id
(+ 100 * layer for the layer sweep).  A spec may replace the first element
of every channel, x[0, c, 0, 0], by mu_c + k*sigma_c (an outlier first row, used to
stress the statistics' summation).  Values are drawn in fp64 in logical
(n, c, h, w) order, arranged in the workload's layout and rounded to the
storage type (round to nearest even).
"""
from __future__ import annotations

import dataclasses

import numpy as np

NCHW, NHWC = 0, 1
F32, BF16, F16 = 0, 1, 2
LEAKY_RELU, ELU, IDENTITY = 0, 1, 2

DTYPE_NAMES = {F32: "f32", BF16: "bf16", F16: "f16"}
ACT_NAMES = {LEAKY_RELU: "leaky_relu", ELU: "elu", IDENTITY: "identity"}
ITEMSIZE = {F32: 4, BF16: 2, F16: 2}

EPS = 1e-5
MOMENTUM = 0.1
SEED_BASE = 20180600

# Layer sweep: (C, H=W) per layer at N=8, a WideResNet-38-like stand-in.
SWEEP_SHAPES = [(64, 224), (128, 112), (128, 112), (256, 56), (256, 56), (256, 56),
                (512, 28), (512, 28), (512, 28), (1024, 28), (1024, 28), (1024, 28),
                (2048, 28), (2048, 28), (4096, 28), (4096, 28)]
SWEEP_N = 8


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    n: int
    c: int
    h: int
    w: int
    layout: int
    dtype: int
    act: int
    act_param: float
    seed: int
    x_dist: str = "normal"          # "normal" or "student_t3"
    first_row_outlier: float = 0.0  # if nonzero: x[0, c, 0, 0] = mu_c + this * sigma_c
    gamma_lo: float = 0.5
    eps: float = EPS
    momentum: float = MOMENTUM

    @property
    def shape(self):
        return (self.n, self.c, self.h, self.w)

    @property
    def numel(self) -> int:
        return self.n * self.c * self.h * self.w

    @property
    def per_channel(self) -> int:
        return self.n * self.h * self.w

    @property
    def itemsize(self) -> int:
        return ITEMSIZE[self.dtype]

    def with_(self, **kw) -> "LayerSpec":
        return dataclasses.replace(self, **kw)


def spec(workload: int, layer: int = 0) -> LayerSpec:
    """The layer spec of a workload (layer index only for the layer sweep)."""
    s = SEED_BASE + workload
    if workload == 0:
        return LayerSpec("tiny", 2, 8, 16, 16, NCHW, F32, LEAKY_RELU, 0.01, s)
    if workload == 1:
        return LayerSpec("resnet_trunk", 64, 256, 56, 56, NHWC, BF16, LEAKY_RELU, 0.01, s)
    if workload == 2:
        return LayerSpec("segmentation", 16, 512, 84, 84, NHWC, BF16, LEAKY_RELU, 0.01, s,
                         x_dist="student_t3")
    if workload == 3:
        return LayerSpec("many_channel", 128, 2048, 7, 7, NCHW, F16, ELU, 1.0, s,
                         gamma_lo=0.05)
    if workload == 4:
        c, hw = SWEEP_SHAPES[layer]
        act, p = (LEAKY_RELU, 0.01) if layer % 2 == 0 else (ELU, 1.0)
        return LayerSpec(f"layer_sweep_l{layer}", SWEEP_N, c, hw, hw, NHWC, BF16, act, p,
                         s + 100 * layer)
    raise ValueError(f"unknown workload {workload}")


# ------------------------------------------------------------ storage types

def to_storage(a64: np.ndarray, dtype: int) -> np.ndarray:
    """fp64 -> storage array (float32, float16, or uint16 holding bf16 bits)."""
    if dtype == F32:
        return np.ascontiguousarray(a64, dtype=np.float32)
    if dtype == F16:
        return np.ascontiguousarray(a64, dtype=np.float16)
    if dtype == BF16:
        f = np.ascontiguousarray(a64, dtype=np.float32).view(np.uint32)
        rounding = np.uint32(0x7FFF) + ((f >> np.uint32(16)) & np.uint32(1))
        out = ((f + rounding) >> np.uint32(16)).astype(np.uint16)
        nan = np.isnan(a64)
        if nan.any():
            out[nan.reshape(out.shape)] = np.uint16(0x7FC0)
        return out
    raise ValueError(f"unknown dtype {dtype}")


def to_f64(store: np.ndarray, dtype: int) -> np.ndarray:
    """Storage array -> exact fp64 values."""
    if dtype in (F32, F16):
        return store.astype(np.float64)
    if dtype == BF16:
        return (store.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype}")


def torch_dtype(dtype: int):
    import torch
    return {F32: torch.float32, BF16: torch.bfloat16, F16: torch.float16}[dtype]


def storage_to_torch(store: np.ndarray, dtype: int):
    """Storage array -> CPU torch tensor of the storage type (same bits)."""
    import torch
    if dtype == BF16:
        return torch.from_numpy(store.view(np.int16).copy()).view(torch.bfloat16)
    return torch.from_numpy(store.copy())


def torch_to_storage(t, dtype: int) -> np.ndarray:
    """CPU torch tensor of the storage type -> storage array (same bits)."""
    import torch
    t = t.detach().cpu().contiguous()
    if dtype == BF16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


# ---------------------------------------------------------------- drawing

def _arrange(logical: np.ndarray, layout: int) -> np.ndarray:
    """(n, c, h, w) logical array -> flat array in the given layout."""
    if layout == NCHW:
        return np.ascontiguousarray(logical).reshape(-1)
    return np.ascontiguousarray(logical.transpose(0, 2, 3, 1)).reshape(-1)


def logical_view(flat: np.ndarray, shape, layout: int) -> np.ndarray:
    """Flat array in ``layout`` -> (n, c, h, w) view/copy."""
    n, c, h, w = shape
    if layout == NCHW:
        return flat.reshape(n, c, h, w)
    return flat.reshape(n, h, w, c).transpose(0, 3, 1, 2)


@dataclasses.dataclass
class LayerInputs:
    spec: LayerSpec
    x: np.ndarray        # storage array, flat, in spec.layout
    x64: np.ndarray      # exact fp64 of x
    dz: np.ndarray       # storage array
    dz64: np.ndarray
    gamma: np.ndarray    # float32 [C]
    beta: np.ndarray     # float32 [C]
    running_mean: np.ndarray  # float32 [C], starts at 0
    running_var: np.ndarray   # float32 [C], starts at 1


def draw(sp: LayerSpec, *, x_logical: np.ndarray | None = None) -> LayerInputs:
    """Seeded inputs of one layer.  ``x_logical`` (fp64, (n, c, h, w)) replaces
    the drawn x, e.g. for the chained layers of the layer sweep."""
    rng = np.random.Generator(np.random.PCG64(sp.seed))
    n, c, h, w = sp.shape
    mu = rng.uniform(-2.0, 2.0, c)
    sigma = rng.uniform(0.5, 3.0, c)
    sign = np.where(rng.random(c) < 0.5, -1.0, 1.0)
    gamma = sign * rng.uniform(sp.gamma_lo, 1.5, c)
    beta = rng.normal(0.0, np.sqrt(0.1), c)
    if x_logical is None:
        if sp.x_dist == "normal":
            e = rng.standard_normal((n, c, h, w))
        elif sp.x_dist == "student_t3":
            e = rng.standard_t(3.0, (n, c, h, w))
        else:
            raise ValueError(sp.x_dist)
        x_logical = mu[None, :, None, None] + sigma[None, :, None, None] * e
        del e
        if sp.first_row_outlier:
            x_logical[0, :, 0, 0] = mu + sp.first_row_outlier * sigma
    else:
        rng.standard_normal((n, c, h, w))   # keep the dz stream independent of x's source
    dz_logical = rng.standard_normal((n, c, h, w))
    x = to_storage(_arrange(x_logical, sp.layout), sp.dtype)
    dz = to_storage(_arrange(dz_logical, sp.layout), sp.dtype)
    return LayerInputs(
        spec=sp, x=x, x64=to_f64(x, sp.dtype), dz=dz, dz64=to_f64(dz, sp.dtype),
        gamma=gamma.astype(np.float32), beta=beta.astype(np.float32),
        running_mean=np.zeros(c, np.float32), running_var=np.ones(c, np.float32))


def sweep_adapter(z_prev_logical: np.ndarray, next_spec: LayerSpec) -> np.ndarray:
    """Stand-in for the convolution between two layers of the layer sweep:
    spatial subsampling plus channel cycling,
    x_next[n, c, h, w] = z_prev[n, c mod C_prev, h*r, w*r], r = H_prev / H_next."""
    n, c_prev, h_prev, _ = z_prev_logical.shape
    r = h_prev // next_spec.h
    sub = z_prev_logical[:, :, ::r, ::r]
    idx = np.arange(next_spec.c) % c_prev
    return np.ascontiguousarray(sub[:, idx, :, :])
