"""GPU parity of INPLACE-ABNsync (the pages' segmentation setting, section 4
"Semantic segmentation": statistics synchronised across GPUs) through the C
ABI, against the fp64 oracle of the whole batch.

The batch is split along N into `world` shards of possibly different sizes.
Each shard lives in its own device buffers (as it would on its own GPU); the
records of the shards are stacked in rank order (what the all-gather between
the two calls of each direction delivers) and every shard is then applied
with the same gathered array.  One GPU runs all ranks one after the other:
the exchange is plain data between the calls, so no call waits on another.

Expected values: the oracle's forward and in-place backward of the whole
batch (the definition of synchronised statistics).  Forward outputs are held
to the plain bound; the backward, fed the oracle's own z and fp32 variance,
adds the fp32 noise allowance of the two-phase kernels' summation order
(their chains on a shard are no longer than on the whole batch).  Every rank
must produce bitwise the same statistics and parameter gradients.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_util import TOL, Guarded, backward_noise, compare, forced_plan, oracle_expect

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import place_batchnorm_activation_b200 as iabn  # noqa: E402

CASES = [
    # (n, c, h, w, layout, dtype, act, param), shard sizes along N
    ((4, 8, 16, 16, wl.NCHW, wl.F32, wl.LEAKY_RELU, 0.01), (2, 2)),
    ((5, 40, 9, 11, wl.NHWC, wl.F32, wl.ELU, 1.0), (2, 2, 1)),
    ((8, 64, 28, 28, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01), (3, 1, 4)),
    ((6, 32, 7, 7, wl.NCHW, wl.F16, wl.ELU, 1.0), (1, 2, 3)),
    ((7, 24, 5, 5, wl.NHWC, wl.F16, wl.IDENTITY, 0.0), (7,)),
    ((3, 300, 6, 5, wl.NCHW, wl.BF16, wl.LEAKY_RELU, 0.2), (1, 1, 1)),
    ((16, 256, 14, 14, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01), (4, 4, 4, 4)),
]


def _spec(case):
    (n, c, h, w, layout, dtype, act, param), _ = case
    return wl.LayerSpec(f"sync_{n}x{c}x{h}x{w}_{layout}_{dtype}", n, c, h, w, layout, dtype, act,
                        param, seed=20180620 + n * 131 + c)


def _shards(sp, sizes, flat):
    """Per-shard copies (own allocations) of a flat storage tensor."""
    per_n = sp.numel // sp.n
    out, n0 = [], 0
    for k in sizes:
        out.append(flat[n0 * per_n:(n0 + k) * per_n].clone())
        n0 += k
    return out


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{_spec(c).name}_w{len(c[1])}")
def test_sync_layer(case):
    sp = _spec(case)
    sizes = case[1]
    assert sum(sizes) == sp.n
    world = len(sizes)
    inp = wl.draw(sp)
    exp = oracle_expect(inp)
    tol = TOL[sp.dtype]
    dev = "cuda"
    f = torch.float32
    sdt = wl.torch_dtype(sp.dtype)
    gamma = torch.from_numpy(inp.gamma).to(dev)
    beta = torch.from_numpy(inp.beta).to(dev)
    shapes = [(k, sp.c, sp.h, sp.w) for k in sizes]
    xs = _shards(sp, sizes, wl.storage_to_torch(inp.x, sp.dtype).to(dev))
    ws = [Guarded(iabn.workspace_size(s, sp.layout, sp.dtype), torch.uint8, dev,
                  torch.zeros(1, dtype=torch.uint8)) for s in shapes]
    recs = [Guarded(sp.c * 3, torch.float64, dev, torch.full((sp.c * 3,), float("nan")))
            for _ in sizes]
    kw = dict(layout=sp.layout, eps=sp.eps, act=sp.act, act_param=sp.act_param)

    # forward: records, gather, apply
    for r in range(world):
        iabn.sync_forward_stats(xs[r], recs[r].t, ws[r].t, shape=shapes[r], layout=sp.layout)
    gathered = torch.stack([r.t for r in recs]).contiguous()
    torch.cuda.synchronize()
    # each record against the oracle's statistics of its own shard
    per_n = sp.numel // sp.n
    n0 = 0
    for r, k in enumerate(sizes):
        sub = wl.LayerSpec(sp.name, k, sp.c, sp.h, sp.w, sp.layout, sp.dtype, sp.act,
                           sp.act_param, sp.seed)
        fw = oracle.forward(sub.shape, sp.layout, inp.x64[n0 * per_n:(n0 + k) * per_n],
                            inp.gamma.astype(np.float64), inp.beta.astype(np.float64),
                            float(np.float32(sp.eps)), sp.act,
                            float(np.float32(sp.act_param)))
        rec = gathered[r].view(sp.c, 3).cpu().numpy()
        np.testing.assert_array_equal(rec[:, 0], np.full(sp.c, float(sub.per_channel)))
        # the record sums the exact storage values in fp32 per thread
        compare(rec[:, 1], fw["mean"], wl.F32, f"{sp.name} record {r} mean")
        compare(rec[:, 2] / sub.per_channel, fw["var"], wl.F32, f"{sp.name} record {r} M2/n")
        n0 += k
    means = [Guarded(sp.c, f, dev, torch.full((sp.c,), float("nan"))) for _ in sizes]
    vars_ = [Guarded(sp.c, f, dev, torch.full((sp.c,), float("nan"))) for _ in sizes]
    for r in range(world):
        iabn.sync_forward_apply(xs[r], gathered, gamma, beta, means[r].t, vars_[r].t, ws[r].t,
                                shape=shapes[r], **kw)
    torch.cuda.synchronize()
    z = torch.cat(xs)
    compare(wl.to_f64(wl.torch_to_storage(z, sp.dtype), sp.dtype), exp["z"], sp.dtype,
            f"{sp.name} sync z")
    compare(means[0].t.cpu().numpy(), exp["mean"], tol, f"{sp.name} sync mean")
    compare(vars_[0].t.cpu().numpy(), exp["var"], tol, f"{sp.name} sync var")
    for r in range(1, world):
        assert torch.equal(means[r].t, means[0].t) and torch.equal(vars_[r].t, vars_[0].t)

    # backward from the oracle's z and fp32 variance (stage-separated)
    zo = _shards(sp, sizes, wl.storage_to_torch(wl.to_storage(exp["z"], sp.dtype),
                                                sp.dtype).to(dev))
    dzs = _shards(sp, sizes, wl.storage_to_torch(inp.dz, sp.dtype).to(dev))
    var32 = torch.from_numpy(exp["var32"].astype(np.float32)).to(dev)
    for r in range(world):
        iabn.sync_backward_stats(zo[r], dzs[r], gamma, beta, recs[r].t, ws[r].t,
                                 shape=shapes[r], layout=sp.layout, act=sp.act,
                                 act_param=sp.act_param)
    gathered_b = torch.stack([r.t for r in recs]).contiguous()
    dgs = [Guarded(sp.c, f, dev, torch.full((sp.c,), float("nan"))) for _ in sizes]
    dbs = [Guarded(sp.c, f, dev, torch.full((sp.c,), float("nan"))) for _ in sizes]
    for r in range(world):
        iabn.sync_backward_apply(zo[r], dzs[r], gathered_b, gamma, beta, var32, dgs[r].t,
                                 dbs[r].t, ws[r].t, shape=shapes[r], **kw)
    torch.cuda.synchronize()
    with forced_plan("twophase"):
        nz = backward_noise(exp, sp)
    dx = torch.cat(dzs)
    compare(wl.to_f64(wl.torch_to_storage(dx, sp.dtype), sp.dtype), exp["dx"], sp.dtype,
            f"{sp.name} sync dx", noise=nz["dx"])
    compare(dgs[0].t.cpu().numpy(), exp["dgamma"], tol, f"{sp.name} sync dgamma",
            noise=nz["dgamma"])
    compare(dbs[0].t.cpu().numpy(), exp["dbeta"], tol, f"{sp.name} sync dbeta",
            noise=nz["dbeta"])
    for r in range(1, world):
        assert torch.equal(dgs[r].t, dgs[0].t) and torch.equal(dbs[r].t, dbs[0].t)
    # guards and device status of every rank
    for g in ws + recs + means + vars_ + dgs + dbs:
        assert g.intact()
    for w in ws:
        assert iabn.get_device_status(w.t) == 0


def test_sync_world_one_is_the_layer():
    """One rank: the sync calls give the plain layer's results (the same
    definition; the summation orders differ only in rounding)."""
    sp = wl.LayerSpec("sync_w1", 4, 64, 12, 12, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.01, 20180630)
    inp = wl.draw(sp)
    dev = "cuda"
    x = wl.storage_to_torch(inp.x, sp.dtype).to(dev)
    x2 = x.clone()
    g = torch.from_numpy(inp.gamma).to(dev)
    b = torch.from_numpy(inp.beta).to(dev)
    kw = dict(shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act, act_param=sp.act_param)
    m1, v1, m2, v2 = (torch.empty(sp.c, device=dev) for _ in range(4))
    ws1 = iabn.new_workspace(sp.shape, sp.layout, sp.dtype, device=dev)
    ws2 = iabn.new_workspace(sp.shape, sp.layout, sp.dtype, device=dev)
    rec = torch.empty(sp.c * 3, dtype=torch.float64, device=dev)
    iabn.forward(x, g, b, m1, v1, ws1, **kw)
    gathered = iabn.forward_sync(x2, g, b, m2, v2, rec, ws2, **kw)
    torch.cuda.synchronize()
    assert gathered.shape == (1, sp.c * 3)
    compare(m2.cpu().numpy(), m1.cpu().numpy().astype(np.float64), (1e-6, 1e-7), "w1 mean")
    compare(v2.cpu().numpy(), v1.cpu().numpy().astype(np.float64), (1e-6, 1e-7), "w1 var")
    compare(x2.cpu().numpy().astype(np.float64), x.cpu().numpy().astype(np.float64),
            (1e-5, 1e-6), "w1 z")
