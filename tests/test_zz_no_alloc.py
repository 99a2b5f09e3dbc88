"""iabn_forward_static_ws: the forward entry point for callers that cannot
allocate device memory (a plugin whose host framework owns the GPU's memory,
a real-time loop that forbids allocation after start-up).  It takes no
workspace; its scratch is an 8 MiB array the library reserves on each GPU.

Checked through the C ABI against the existing entry point iabn_forward (with
a caller-allocated workspace) on the same inputs, on two calls in a row, with
the tolerance of the other parity tests.  This file is collected last so
that a failure here stops a ``-x`` run only after every other test ran; it
also passes on its own in a fresh process.
"""
import numpy as np
import pytest

import workloads as wl
from gpu_util import TOL, compare

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import place_batchnorm_activation_b200 as iabn  # noqa: E402

LIMIT = 8 << 20

CASES = [
    # NHWC bf16, a slice of the ResNet-trunk layer (resident plan)
    wl.LayerSpec("nhwc_bf16", 8, 256, 56, 56, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01, seed=31),
    # NCHW fp16 with 49-value planes and ELU
    wl.LayerSpec("nchw_f16", 16, 512, 7, 7, wl.NCHW, wl.F16, wl.ELU, 1.0, seed=32),
    # odd shape (two-phase plan)
    wl.LayerSpec("odd_f32", 3, 5, 7, 9, wl.NHWC, wl.F32, wl.LEAKY_RELU, 0.2, seed=33),
]


def _run(sp, inp, static: bool):
    dev = torch.device("cuda")
    x = wl.storage_to_torch(inp.x, sp.dtype).to(dev)
    g = torch.from_numpy(inp.gamma).to(dev)
    b = torch.from_numpy(inp.beta).to(dev)
    mean = torch.full((sp.c,), float("nan"), device=dev)
    var = torch.full((sp.c,), float("nan"), device=dev)
    desc = iabn.make_desc(sp.shape, sp.layout, sp.dtype)
    stream = torch.cuda.current_stream().cuda_stream
    if static:
        st = iabn.iabn_forward_static_ws(desc, x.data_ptr(), g.data_ptr(), b.data_ptr(),
                                         sp.eps, sp.act, sp.act_param, mean.data_ptr(),
                                         var.data_ptr(), stream)
    else:
        ws = iabn.new_workspace(sp.shape, sp.layout, sp.dtype, device=dev)
        st = iabn.iabn_forward(desc, x.data_ptr(), g.data_ptr(), b.data_ptr(), sp.eps, sp.act,
                               sp.act_param, mean.data_ptr(), var.data_ptr(), ws.data_ptr(),
                               ws.numel(), stream)
    assert st == iabn.IABN_OK, iabn.STATUS_NAMES.get(st, st)
    torch.cuda.synchronize()
    z = wl.to_f64(wl.torch_to_storage(x, sp.dtype), sp.dtype)
    return z, mean.cpu().numpy().astype(np.float64), var.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("sp", CASES, ids=lambda s: s.name)
def test_static_workspace_forward_matches_iabn_forward(sp):
    assert iabn.workspace_size(sp.shape, sp.layout, sp.dtype) <= LIMIT
    inp = wl.draw(sp)
    z_ref, m_ref, v_ref = _run(sp, inp, static=False)
    tol = TOL[sp.dtype]
    for _ in range(2):   # two calls in a row share (and reuse) the static scratch
        z, m, v = _run(sp, inp, static=True)
        compare(z, z_ref, sp.dtype, f"{sp.name} z")
        compare(m, m_ref, tol, f"{sp.name} mean")
        compare(v, v_ref, tol, f"{sp.name} var")


def test_static_workspace_rejects_oversized_descriptor():
    # NCHW partial summaries: N*C*16 bytes > 8 MiB
    sp = wl.LayerSpec("big", 256, 4096, 2, 2, wl.NCHW, wl.BF16, wl.LEAKY_RELU, 0.01, seed=1)
    assert iabn.workspace_size(sp.shape, sp.layout, sp.dtype) > LIMIT
    dev = torch.device("cuda")
    x = torch.zeros(sp.numel, dtype=torch.bfloat16, device=dev)
    g = torch.ones(sp.c, device=dev)
    before = x.clone()
    desc = iabn.make_desc(sp.shape, sp.layout, sp.dtype)
    st = iabn.iabn_forward_static_ws(desc, x.data_ptr(), g.data_ptr(), g.data_ptr(), 1e-5, 0,
                                     0.01, g.data_ptr(), g.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    assert st == iabn.IABN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(x, before)
    # other argument errors are reported as by iabn_forward
    st = iabn.iabn_forward_static_ws(iabn.make_desc((1, 4, 1, 1), 0, 0), x.data_ptr(),
                                     g.data_ptr(), g.data_ptr(), 1e-5, 0, 0.01, g.data_ptr(),
                                     g.data_ptr(), None)
    assert st == iabn.IABN_ERR_INVALID_ARG


def test_static_ws_status_reports_a_timed_out_wait(monkeypatch):
    """A bounded wait of the resident kernel made to run out (one CTA waits
    on a word nothing sets; the others' barrier budget is 20 ms) inside
    iabn_forward_static_ws: the call returns IABN_OK (the condition is found
    on the device), iabn_get_static_ws_status reports IABN_ERR_TIMEOUT once
    and clears it, and the next call is correct."""
    sp = wl.LayerSpec("static_timeout", 8, 256, 14, 14, wl.NHWC, wl.BF16, wl.LEAKY_RELU, 0.01,
                      seed=34)
    inp = wl.draw(sp)
    monkeypatch.setenv("IABN_FORCE_PLAN", "resident")
    assert iabn.get_static_ws_status() == 0
    monkeypatch.setenv("IABN_BARRIER_BUDGET_NS", str(20_000_000))
    monkeypatch.setenv("IABN_TEST_STALL_CTA", "3")
    _run(sp, inp, True)
    monkeypatch.delenv("IABN_TEST_STALL_CTA")
    monkeypatch.delenv("IABN_BARRIER_BUDGET_NS")
    assert iabn.get_static_ws_status() == 6      # IABN_ERR_TIMEOUT
    assert iabn.get_static_ws_status() == 0      # the read cleared it
    z1, m1, v1 = _run(sp, inp, True)
    z2, m2, v2 = _run(sp, inp, False)
    assert iabn.get_static_ws_status() == 0
    tol = TOL[sp.dtype]
    compare(z1, z2, sp.dtype, "static z after a timed-out call")
    compare(m1, m2, tol, "static mean after a timed-out call")
    compare(v1, v2, tol, "static var after a timed-out call")
