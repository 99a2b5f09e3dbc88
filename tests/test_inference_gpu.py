"""GPU parity of evaluation mode (iabn_inference) against the oracle's
inference on the same seeded inputs.

The running statistics are drawn near the batch's own, as a trained layer's
would be: mean + 0.1*sigma*N(0,1) and variance * U(0.8, 1.25), rounded to
fp32 (the values the C ABI receives; the oracle gets the same values).
Tolerance: the storage type's (fp32 rel 1e-5 / abs 1e-6; bf16, fp16 rel
2e-2 / abs 1e-2), with the relative part taken against the size of the terms
y is the sum of, |gamma*xhat| + |beta|, where that is larger than |z|: fp32
evaluation error scales with the terms, and the activation's slope is at
most 1, so it carries over to z.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_util import compare, f32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import place_batchnorm_activation_b200 as iabn  # noqa: E402


def running_stats_near(inp):
    sp = inp.spec
    rng = np.random.default_rng(sp.seed + 7)
    x = wl.logical_view(inp.x64, sp.shape, sp.layout)
    mean = x.mean(axis=(0, 2, 3))
    var = x.var(axis=(0, 2, 3))
    rm = (mean + 0.1 * np.sqrt(var) * rng.standard_normal(sp.c)).astype(np.float32)
    rv = (var * rng.uniform(0.8, 1.25, sp.c)).astype(np.float32)
    return rm, rv


def check_inference(inp):
    sp = inp.spec
    rm, rv = running_stats_near(inp)
    g, b = inp.gamma.astype(np.float64), inp.beta.astype(np.float64)
    eps, p = f32(sp.eps), f32(sp.act_param)
    rm64, rv64 = rm.astype(np.float64), rv.astype(np.float64)
    want = oracle.round_to(oracle.inference(sp.shape, sp.layout, inp.x64, g, b, rm64, rv64, eps,
                                            sp.act, p), sp.dtype)
    xl = wl.logical_view(inp.x64, sp.shape, sp.layout)
    term = (np.abs(g)[None, :, None, None] * np.abs(xl - rm64[None, :, None, None])
            / np.sqrt(rv64 + eps)[None, :, None, None] + np.abs(b)[None, :, None, None])
    dev = "cuda"
    x = wl.storage_to_torch(inp.x, sp.dtype).to(dev)
    tg, tb = torch.from_numpy(inp.gamma).to(dev), torch.from_numpy(inp.beta).to(dev)
    trm, trv = torch.from_numpy(rm).to(dev), torch.from_numpy(rv).to(dev)
    ws = iabn.new_workspace(sp.shape, sp.layout, sp.dtype, device=dev)
    torch.cuda.synchronize()
    k0 = iabn.iabn_kernel_launches()
    iabn.inference(x, tg, tb, trm, trv, ws, shape=sp.shape, layout=sp.layout, eps=sp.eps,
                   act=sp.act, act_param=sp.act_param)
    k1 = iabn.iabn_kernel_launches()
    torch.cuda.synchronize()
    assert k1 - k0 == 1          # one launch: coefficients and the pass together
    got = wl.to_f64(wl.torch_to_storage(x, sp.dtype), sp.dtype)
    compare(got, want, sp.dtype, f"{sp.name} inference z", wl._arrange(term, sp.layout))
    assert iabn.get_device_status(ws) == 0
    # the statistics and parameters are read only
    np.testing.assert_array_equal(trm.cpu().numpy(), rm)
    np.testing.assert_array_equal(trv.cpu().numpy(), rv)


@pytest.mark.parametrize("workload", [0, 1, 2, 3])
def test_inference_parity_workloads(workload):
    check_inference(wl.draw(wl.spec(workload)))


EDGE = [
    # (n, c, h, w, layout, dtype, act, param)
    (1, 5, 1, 1, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01),      # one value per channel
    (1, 3, 1, 1, wl.NCHW, wl.BF16, wl.ELU, 1.0),             # fewer elements than a vector
    (3, 1, 5, 7, wl.NCHW, wl.F32, wl.ELU, 0.5),
    (2, 3, 4, 5, wl.NHWC, wl.F16, wl.LEAKY_RELU, 0.2),       # ragged C, tail
    (7, 40, 9, 11, wl.NCHW, wl.BF16, wl.IDENTITY, 0.0),
    (2, 300, 5, 5, wl.NHWC, wl.F32, wl.ELU, 1.0),
    (8, 264, 7, 7, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01),
    (64, 40, 3, 3, wl.NCHW, wl.F16, wl.ELU, 1.0),
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "x".join(map(str, c[:4])) +
                         f"-{'nhwc' if c[4] else 'nchw'}-{wl.DTYPE_NAMES[c[5]]}-"
                         f"{wl.ACT_NAMES[c[6]]}")
def test_inference_parity_edge_shapes(case):
    n, c, h, w, layout, dtype, act, p = case
    sp = wl.LayerSpec("eval_edge", n, c, h, w, layout, dtype, act, p, seed=555 + n * c + h * w)
    check_inference(wl.draw(sp))
