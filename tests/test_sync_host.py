"""INPLACE-ABNsync without a GPU:

* the exchange between the two calls of each direction
  (``gather_records``): an all-gather over a torch.distributed group, here
  world size 2 over gloo on CPU tensors, delivers every rank the records of
  all ranks in rank order; without a process group it is the rank's own;
* the decomposition the sync layer relies on, pinned with the oracle: the
  whole batch's mean and biased variance equal the rank-order combination of
  the shards' (n, mean, M2) records (one pass around the first shard's mean,
  as the CUDA finalize does), and the backward sums of the whole batch are
  the sums of the shards' (sum dy, sum dy*xhat) records -- for shards of
  unequal sizes, in both layouts.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads as wl
import place_batchnorm_activation_b200 as iabn


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rec = torch.arange(12, dtype=torch.float64) + 100.0 * rank
        g = iabn.gather_records(rec)
        out[rank] = g.numpy().tolist()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gather_records_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    want = [list(np.arange(12.0)), list(np.arange(12.0) + 100.0)]
    assert res[0] == want and res[1] == want


def test_gather_records_without_a_group_is_the_own_record():
    rec = torch.arange(6, dtype=torch.float64)
    g = iabn.gather_records(rec)
    assert g.shape == (1, 6) and torch.equal(g[0], rec)


def _combine_forward(recs):
    """Rank-order combination of (n, mean, M2) records around the first
    record's mean (the arithmetic of the sync finalize)."""
    r = recs[0][:, 1]
    n = np.zeros_like(r)
    s1 = np.zeros_like(r)
    s2 = np.zeros_like(r)
    for q in recs:
        d = q[:, 1] - r
        n += q[:, 0]
        s1 += q[:, 0] * d
        s2 += q[:, 2] + q[:, 0] * d * d
    return r + s1 / n, (s2 - s1 * (s1 / n)) / n


@pytest.mark.parametrize("layout", [wl.NCHW, wl.NHWC])
def test_sharded_statistics_combine_to_the_whole_batch(layout):
    sp = wl.LayerSpec("sync_split", 7, 5, 3, 4, layout, wl.F32, wl.LEAKY_RELU, 0.01, 20180701)
    inp = wl.draw(sp)
    g = inp.gamma.astype(np.float64)
    b = inp.beta.astype(np.float64)
    eps, p = float(np.float32(sp.eps)), float(np.float32(sp.act_param))
    whole = oracle.forward(sp.shape, layout, inp.x64, g, b, eps, sp.act, p)
    per_n = sp.numel // sp.n
    recs, n0 = [], 0
    for k in (3, 1, 3):
        fw = oracle.forward((k, sp.c, sp.h, sp.w), layout, inp.x64[n0 * per_n:(n0 + k) * per_n],
                            g, b, eps, sp.act, p)
        m = k * sp.h * sp.w
        recs.append(np.stack([np.full(sp.c, float(m)), fw["mean"], fw["var"] * m], axis=1))
        n0 += k
    mean, var = _combine_forward(recs)
    np.testing.assert_allclose(mean, whole["mean"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(var, whole["var"], rtol=1e-12, atol=1e-15)

    # backward: the whole batch's dbeta = sum dy and dgamma = sum dy*xhat are
    # the sums of the shards' (the shards' own backward sums, with the
    # whole batch's z and statistics)
    z = oracle.round_to(whole["z"], sp.dtype)
    var32 = oracle.round_to(whole["var"], oracle.F32)
    bw = oracle.backward_inplace(sp.shape, layout, z, inp.dz64, g, b, var32, eps, sp.act, p)
    db = np.zeros(sp.c)
    dg = np.zeros(sp.c)
    n0 = 0
    for k in (3, 1, 3):
        sl = slice(n0 * per_n, (n0 + k) * per_n)
        part = oracle.backward_inplace((k, sp.c, sp.h, sp.w), layout, z[sl], inp.dz64[sl], g, b,
                                       var32, eps, sp.act, p)
        db += part["dbeta"]
        dg += part["dgamma"]
        n0 += k
    np.testing.assert_allclose(db, bw["dbeta"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dg, bw["dgamma"], rtol=1e-12, atol=1e-12)
