"""Failure detection on the GPU without a GPU fault: a bounded wait is made to
run out on purpose and the status word must say so.

One CTA of the resident kernel waits, before the first grid barrier, on a
control-block word that nothing sets; that wait gives up after twice the time
budget.  The other CTAs' barrier waits (budget 20 ms) therefore run out: they
set IABN_ERR_TIMEOUT, skip the rest of their work and finish.  The next call
on the same workspace must be correct -- every CTA still arrives at every
barrier, so the barrier counter stays balanced -- and the status stays
sticky until it is read.
"""
import pytest

import workloads as wl
from gpu_util import GpuLayer, compare, forced_plan, oracle_expect, TOL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

IABN_OK, IABN_ERR_TIMEOUT = 0, 6


def test_barrier_wait_timeout_sets_status(monkeypatch):
    sp = wl.LayerSpec("timeout", 8, 256, 14, 14, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01,
                      seed=9191)
    inp = wl.draw(sp)
    exp = oracle_expect(inp)
    with forced_plan("resident"):
        L = GpuLayer(inp)
        monkeypatch.setenv("IABN_BARRIER_BUDGET_NS", str(20_000_000))
        monkeypatch.setenv("IABN_TEST_STALL_CTA", "3")
        L.forward()
        torch.cuda.synchronize()
        monkeypatch.delenv("IABN_TEST_STALL_CTA")
        monkeypatch.delenv("IABN_BARRIER_BUDGET_NS")

        # a normal call on the same workspace, before the status is read
        L.load_z(inp.x64)
        L.forward()
        torch.cuda.synchronize()
        z = L.host(L.x)
        mean, var = L.mean.cpu().numpy(), L.var.cpu().numpy()
        assert L.status() == IABN_ERR_TIMEOUT          # sticky until read
        tol = TOL[sp.dtype]
        compare(z, exp["z"], sp.dtype, "z after a timed-out call")
        compare(mean, exp["mean"], tol, "mean after a timed-out call")
        compare(var, exp["var"], tol, "var after a timed-out call")

        # the read cleared it
        L.load_z(inp.x64)
        L.forward()
        assert L.status() == IABN_OK
