"""The C ABI without a GPU: libiabn.so loads, exports every entry point that
include/iabn.h declares, and rejects bad arguments synchronously on the host
(before any CUDA call).

The rejection tests pass fake device addresses; every case carries a defect
the host checks catch first.  They are skipped when a GPU is present so a
fake address can never reach a kernel.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import place_batchnorm_activation_b200 as iabn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "iabn.h")
PROBE_HEADER = os.path.join(ROOT, "include", "iabn_probe.h")

no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="fake device addresses are only passed without a GPU")


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(iabn_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(iabn.EXPORTS)
    assert declared_functions(PROBE_HEADER) == sorted(iabn.PROBE_EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = iabn.lib()
    declared = declared_functions() + declared_functions(PROBE_HEADER)
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", iabn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (iabn_\w+)", out))
    assert set(declared) <= exported


def test_workspace_size():
    d = iabn.make_desc((64, 256, 56, 56), iabn.IABN_NHWC, iabn.IABN_BF16)
    n = iabn.iabn_workspace_size(d)
    assert n > 0 and n % 256 == 0
    # partial summaries (16 B) for up to 256 blocks per channel + coefficients
    assert n >= 256 + 256 * 256 * 16 + 256 * 16
    d2 = iabn.make_desc((128, 2048, 7, 7), iabn.IABN_NCHW, iabn.IABN_F16)
    assert iabn.iabn_workspace_size(d2) >= 256 + 128 * 2048 * 16 + 2048 * 16
    for bad in [(0, 1, 1, 2), (1, 0, 2, 2), (-1, 2, 2, 2)]:
        assert iabn.iabn_workspace_size(iabn.make_desc(bad, 0, 0)) == 0
    # one value per channel is a valid descriptor for inference
    assert iabn.iabn_workspace_size(iabn.make_desc((1, 1, 1, 1), 0, 0)) > 0
    assert iabn.iabn_workspace_size(iabn.make_desc((2, 2, 2, 2), 2, 0)) == 0
    assert iabn.iabn_workspace_size(iabn.make_desc((2, 2, 2, 2), 0, 3)) == 0


FAKE = 0x10000000  # 16-byte aligned fake device address (never dereferenced)


def _fwd(desc=None, x=FAKE, eps=1e-5, act=0, p=0.01, ws=FAKE, ws_bytes=None, g=FAKE,
         mean=FAKE):
    desc = desc or iabn.make_desc((2, 4, 3, 3), iabn.IABN_NCHW, iabn.IABN_F32)
    if ws_bytes is None:
        ws_bytes = iabn.iabn_workspace_size(desc)
    return iabn.iabn_forward(desc, x, g, FAKE, eps, act, p, mean, FAKE, ws, ws_bytes, None)


def _bwd(desc=None, z=FAKE, dz=FAKE + 4096, eps=1e-5, act=0, p=0.01, ws=FAKE + 8192,
         ws_bytes=None, dg=FAKE):
    desc = desc or iabn.make_desc((2, 4, 3, 3), iabn.IABN_NHWC, iabn.IABN_BF16)
    if ws_bytes is None:
        ws_bytes = iabn.iabn_workspace_size(desc)
    return iabn.iabn_backward(desc, z, dz, FAKE, FAKE, FAKE, eps, act, p, dg, FAKE, ws,
                              ws_bytes, None)


@no_gpu_only
def test_forward_rejects_bad_arguments():
    E = iabn
    assert _fwd(desc=iabn.make_desc((1, 4, 1, 1), 0, 0)) == E.IABN_ERR_INVALID_ARG  # M = 1
    assert _fwd(desc=iabn.make_desc((2, 0, 3, 3), 0, 0)) == E.IABN_ERR_INVALID_ARG
    assert _fwd(desc=iabn.make_desc((2, 4, 3, 3), 5, 0)) == E.IABN_ERR_INVALID_ARG
    assert _fwd(desc=iabn.make_desc((2, 4, 3, 3), 0, 9)) == E.IABN_ERR_INVALID_ARG
    assert _fwd(desc=iabn.make_desc((1 << 41, 4, 3, 3), 0, 0)) == E.IABN_ERR_UNSUPPORTED
    assert _fwd(x=None) == E.IABN_ERR_INVALID_ARG
    assert _fwd(g=None) == E.IABN_ERR_INVALID_ARG
    assert _fwd(mean=None) == E.IABN_ERR_INVALID_ARG
    assert _fwd(eps=-1e-5) == E.IABN_ERR_INVALID_ARG
    assert _fwd(eps=float("nan")) == E.IABN_ERR_INVALID_ARG
    assert _fwd(act=7) == E.IABN_ERR_INVALID_ARG
    assert _fwd(act=E.IABN_ACT_LEAKY_RELU, p=0.0) == E.IABN_ERR_INVALID_ARG
    assert _fwd(act=E.IABN_ACT_LEAKY_RELU, p=-0.1) == E.IABN_ERR_INVALID_ARG
    assert _fwd(act=E.IABN_ACT_ELU, p=0.0) == E.IABN_ERR_INVALID_ARG
    assert _fwd(act=E.IABN_ACT_ELU, p=float("inf")) == E.IABN_ERR_INVALID_ARG
    assert _fwd(x=FAKE + 2) == E.IABN_ERR_MISALIGNED
    assert _fwd(ws=None) == E.IABN_ERR_WORKSPACE
    d = iabn.make_desc((2, 4, 3, 3), 0, 0)
    assert _fwd(desc=d, ws_bytes=iabn.iabn_workspace_size(d) - 1) == E.IABN_ERR_WORKSPACE
    assert iabn.lib().iabn_forward(None, FAKE, FAKE, FAKE, 1e-5, 0, 0.01, FAKE, FAKE, FAKE,
                                   1 << 20, None) == E.IABN_ERR_INVALID_ARG


@no_gpu_only
def test_backward_rejects_bad_arguments():
    E = iabn
    assert _bwd(desc=iabn.make_desc((1, 4, 1, 1), 1, 1)) == E.IABN_ERR_INVALID_ARG
    assert _bwd(z=None) == E.IABN_ERR_INVALID_ARG
    assert _bwd(dz=None) == E.IABN_ERR_INVALID_ARG
    assert _bwd(z=FAKE, dz=FAKE) == E.IABN_ERR_INVALID_ARG       # z and dz alias
    assert _bwd(dg=None) == E.IABN_ERR_INVALID_ARG
    assert _bwd(eps=-1.0) == E.IABN_ERR_INVALID_ARG
    assert _bwd(act=E.IABN_ACT_ELU, p=-1.0) == E.IABN_ERR_INVALID_ARG
    assert _bwd(dz=FAKE + 4096 + 8) == E.IABN_ERR_MISALIGNED
    assert _bwd(z=FAKE + 1) == E.IABN_ERR_MISALIGNED
    assert _bwd(ws_bytes=16) == E.IABN_ERR_WORKSPACE


def _inf(desc=None, x=FAKE, eps=1e-5, act=0, p=0.01, ws=FAKE + 8192, ws_bytes=None,
         rm=FAKE, rv=FAKE):
    desc = desc or iabn.make_desc((2, 4, 3, 3), iabn.IABN_NHWC, iabn.IABN_F16)
    if ws_bytes is None:
        ws_bytes = iabn.iabn_workspace_size(desc)
    return iabn.iabn_inference(desc, x, FAKE, FAKE, rm, rv, eps, act, p, ws, ws_bytes, None)


@no_gpu_only
def test_inference_rejects_bad_arguments():
    E = iabn
    assert _inf(desc=iabn.make_desc((0, 4, 1, 1), 0, 0)) == E.IABN_ERR_INVALID_ARG
    assert _inf(desc=iabn.make_desc((1, 4, 1, 1), 0, 3)) == E.IABN_ERR_INVALID_ARG
    assert _inf(x=None) == E.IABN_ERR_INVALID_ARG
    assert _inf(rm=None) == E.IABN_ERR_INVALID_ARG
    assert _inf(rv=None) == E.IABN_ERR_INVALID_ARG
    assert _inf(eps=-1.0) == E.IABN_ERR_INVALID_ARG
    assert _inf(act=E.IABN_ACT_ELU, p=0.0) == E.IABN_ERR_INVALID_ARG
    assert _inf(x=FAKE + 8) == E.IABN_ERR_MISALIGNED
    assert _inf(ws=None) == E.IABN_ERR_WORKSPACE
    assert _inf(ws_bytes=16) == E.IABN_ERR_WORKSPACE
    # M = 1 passes the host checks (and then finds no device here)
    assert _inf(desc=iabn.make_desc((1, 4, 1, 1), 0, 0)) == E.IABN_ERR_CUDA
    assert _inf() == E.IABN_ERR_CUDA


@no_gpu_only
def test_running_update_and_status_reject_bad_arguments():
    E = iabn
    f = iabn.iabn_update_running_stats
    assert f(0, 10, FAKE, FAKE, FAKE, FAKE, 0.1, None) == E.IABN_ERR_INVALID_ARG
    assert f(4, 1, FAKE, FAKE, FAKE, FAKE, 0.1, None) == E.IABN_ERR_INVALID_ARG
    assert f(4, 10, None, FAKE, FAKE, FAKE, 0.1, None) == E.IABN_ERR_INVALID_ARG
    assert f(4, 10, FAKE, FAKE, FAKE, FAKE, 1.5, None) == E.IABN_ERR_INVALID_ARG
    assert f(4, 10, FAKE, FAKE, FAKE, FAKE, float("nan"), None) == E.IABN_ERR_INVALID_ARG
    assert iabn.iabn_get_device_status(None, None) == E.IABN_ERR_INVALID_ARG


@no_gpu_only
def test_valid_call_without_gpu_reports_cuda_error():
    """With every argument valid, the host reaches the CUDA runtime, which has
    no device here: the call reports IABN_ERR_CUDA rather than computing on
    the CPU."""
    assert _fwd() == iabn.IABN_ERR_CUDA
    assert _bwd() == iabn.IABN_ERR_CUDA


def test_tensor_helpers_refuse_cpu_tensors():
    x = torch.zeros(2 * 4 * 9)
    g = torch.ones(4)
    with pytest.raises(iabn.IabnError):
        iabn.forward(x, g, g, g, g, torch.zeros(1 << 16, dtype=torch.uint8),
                     shape=(2, 4, 3, 3), layout=0, eps=1e-5, act=0, act_param=0.01)


@no_gpu_only
def test_probes_reject_bad_arguments_on_the_host():
    assert iabn.iabn_probe_empty(0, 320, 0, 0, None) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_probe_empty(148, 2048, 0, 0, None) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_probe_read(None, 1 << 20, 148, None) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_probe_read(FAKE, 17, 148, None) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_probe_read_write(FAKE + 8, 1 << 20, 148, None) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_probe_read_write(FAKE, 1 << 20, 0, None) == iabn.IABN_ERR_INVALID_ARG
    with pytest.raises(RuntimeError):
        iabn.iabn_probe_cluster_occupancy(0, 320, 0)
