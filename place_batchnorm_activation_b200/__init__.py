"""Python binding of libiabn.so -- In-Place Activated BatchNorm on B200.

Argument marshalling only: every step of the layer runs in the CUDA kernels
of libiabn.so (declared in include/iabn.h).  PyTorch is used for device
memory and streams.  There is no CPU fallback: if the library is missing or
no GPU is present, calls raise.

Two levels:
  * ``iabn_forward``, ``iabn_backward``, ``iabn_forward_standard``,
    ``iabn_backward_standard``, ``iabn_forward_checkpoint``,
    ``iabn_backward_checkpoint``, ``iabn_checkpoint_recompute``,
    ``iabn_inference``, ``iabn_update_running_stats``, ``iabn_workspace_size``,
    ``iabn_get_device_status``: the C entry points with the same names and
    arguments (raw device pointers as ints).
  * ``forward``, ``backward``, ``forward_standard``, ``backward_standard``,
    ``forward_checkpoint``, ``backward_checkpoint``, ``checkpoint_recompute``,
    ``inference``, ``update_running_stats``, ``workspace_size``,
    ``get_device_status``: the same calls taking torch tensors;
    ``describe_plan``: the launch plan of a call on a descriptor, as a dict.
  * INPLACE-ABNsync (statistics over a batch split across GPUs):
    ``sync_forward_stats`` / ``sync_forward_apply``,
    ``sync_backward_stats`` / ``sync_backward_apply`` (the C calls), and
    ``forward_sync`` / ``backward_sync``, which put ``gather_records`` (an
    all-gather over a torch.distributed group) between them.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libiabn.so")

# enums of include/iabn.h
IABN_OK = 0
IABN_ERR_INVALID_ARG = 1
IABN_ERR_UNSUPPORTED = 2
IABN_ERR_MISALIGNED = 3
IABN_ERR_WORKSPACE = 4
IABN_ERR_CUDA = 5
IABN_ERR_TIMEOUT = 6
IABN_ERR_SINGULAR_GAMMA = 7
STATUS_NAMES = {0: "IABN_OK", 1: "IABN_ERR_INVALID_ARG", 2: "IABN_ERR_UNSUPPORTED",
                3: "IABN_ERR_MISALIGNED", 4: "IABN_ERR_WORKSPACE", 5: "IABN_ERR_CUDA",
                6: "IABN_ERR_TIMEOUT", 7: "IABN_ERR_SINGULAR_GAMMA"}

IABN_NCHW, IABN_NHWC = 0, 1
IABN_F32, IABN_BF16, IABN_F16 = 0, 1, 2
IABN_ACT_LEAKY_RELU, IABN_ACT_ELU, IABN_ACT_IDENTITY = 0, 1, 2

# Symbols include/iabn.h declares (checked by the tests).
EXPORTS = ("iabn_workspace_size", "iabn_forward", "iabn_forward_with_running_stats",
           "iabn_backward",
           "iabn_update_running_stats", "iabn_get_device_status", "iabn_kernel_launches",
           "iabn_forward_static_ws", "iabn_get_static_ws_status", "iabn_describe_plan",
           "iabn_inference",
           "iabn_forward_standard", "iabn_backward_standard", "iabn_forward_checkpoint",
           "iabn_backward_checkpoint", "iabn_checkpoint_recompute",
           "iabn_sync_forward_stats", "iabn_sync_forward_apply", "iabn_sync_backward_stats",
           "iabn_sync_backward_apply")
# Symbols include/iabn_probe.h declares: measurement probes, not the method.
PROBE_EXPORTS = ("iabn_probe_empty", "iabn_probe_read", "iabn_probe_read_write",
                 "iabn_probe_cluster_occupancy")

# iabn_call values (iabn_describe_plan)
(IABN_CALL_FORWARD, IABN_CALL_BACKWARD, IABN_CALL_FORWARD_STANDARD, IABN_CALL_BACKWARD_STANDARD,
 IABN_CALL_FORWARD_CHECKPOINT, IABN_CALL_BACKWARD_CHECKPOINT) = range(6)

IABN_PLAN_TWOPHASE, IABN_PLAN_RESIDENT = 0, 1
PLAN_NAMES = {IABN_PLAN_TWOPHASE: "twophase", IABN_PLAN_RESIDENT: "resident"}


class IabnDesc(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("c", ctypes.c_int64), ("h", ctypes.c_int64),
                ("w", ctypes.c_int64), ("layout", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class IabnPlanInfo(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "plan", "launches", "grid", "threads", "smem_bytes", "tile_bytes", "slots", "ring",
        "vectors_per_row", "cols_per_thread", "row_phases", "planes_per_unit", "stash_rows",
        "stash_copy_engine")]


class IabnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libiabn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "place_batchnorm_activation_b200._build.build()")
            L = ctypes.CDLL(LIB_PATH)
            vp, f32, i32, i64 = ctypes.c_void_p, ctypes.c_float, ctypes.c_int32, ctypes.c_int64
            pd = ctypes.POINTER(IabnDesc)
            L.iabn_workspace_size.argtypes = [pd]
            L.iabn_workspace_size.restype = ctypes.c_size_t
            L.iabn_forward.argtypes = [pd, vp, vp, vp, f32, i32, f32, vp, vp, vp,
                                       ctypes.c_size_t, vp]
            L.iabn_forward.restype = i32
            L.iabn_forward_with_running_stats.argtypes = [pd, vp, vp, vp, f32, i32, f32, vp, vp,
                                                          vp, vp, f32, vp, ctypes.c_size_t, vp]
            L.iabn_forward_with_running_stats.restype = i32
            L.iabn_backward.argtypes = [pd, vp, vp, vp, vp, vp, f32, i32, f32, vp, vp, vp,
                                        ctypes.c_size_t, vp]
            L.iabn_backward.restype = i32
            L.iabn_forward_standard.argtypes = [pd, vp, vp, vp, vp, f32, i32, f32, vp, vp, vp,
                                                ctypes.c_size_t, vp]
            L.iabn_forward_standard.restype = i32
            L.iabn_forward_checkpoint.argtypes = [pd, vp, vp, vp, vp, f32, i32, f32, vp, vp, vp,
                                                  ctypes.c_size_t, vp]
            L.iabn_forward_checkpoint.restype = i32
            L.iabn_backward_standard.argtypes = [pd, vp, vp, vp, vp, vp, vp, f32, i32, f32, vp,
                                                 vp, vp, ctypes.c_size_t, vp]
            L.iabn_backward_standard.restype = i32
            L.iabn_backward_checkpoint.argtypes = [pd, vp, vp, vp, vp, vp, f32, i32, f32, vp, vp,
                                                   vp, ctypes.c_size_t, vp]
            L.iabn_backward_checkpoint.restype = i32
            L.iabn_checkpoint_recompute.argtypes = [pd, vp, vp, vp, vp, i32, f32, vp]
            L.iabn_checkpoint_recompute.restype = i32
            L.iabn_inference.argtypes = [pd, vp, vp, vp, vp, vp, f32, i32, f32, vp,
                                         ctypes.c_size_t, vp]
            L.iabn_inference.restype = i32
            L.iabn_update_running_stats.argtypes = [i64, i64, vp, vp, vp, vp, f32, vp]
            L.iabn_update_running_stats.restype = i32
            L.iabn_get_device_status.argtypes = [vp, vp]
            L.iabn_get_device_status.restype = i32
            L.iabn_kernel_launches.argtypes = []
            L.iabn_kernel_launches.restype = ctypes.c_uint64
            L.iabn_forward_static_ws.argtypes = [pd, vp, vp, vp, f32, i32, f32, vp, vp, vp]
            L.iabn_forward_static_ws.restype = i32
            L.iabn_get_static_ws_status.argtypes = [vp]
            L.iabn_get_static_ws_status.restype = i32
            L.iabn_describe_plan.argtypes = [pd, i32, i32, i32, ctypes.POINTER(IabnPlanInfo)]
            L.iabn_describe_plan.restype = i32
            L.iabn_sync_forward_stats.argtypes = [pd, vp, vp, vp, ctypes.c_size_t, vp]
            L.iabn_sync_forward_stats.restype = i32
            L.iabn_sync_forward_apply.argtypes = [pd, vp, vp, i32, vp, vp, f32, i32, f32, vp, vp,
                                                  vp, ctypes.c_size_t, vp]
            L.iabn_sync_forward_apply.restype = i32
            L.iabn_sync_backward_stats.argtypes = [pd, vp, vp, vp, vp, i32, f32, vp, vp,
                                                   ctypes.c_size_t, vp]
            L.iabn_sync_backward_stats.restype = i32
            L.iabn_sync_backward_apply.argtypes = [pd, vp, vp, vp, i32, vp, vp, vp, f32, i32, f32,
                                                   vp, vp, vp, ctypes.c_size_t, vp]
            L.iabn_sync_backward_apply.restype = i32
            L.iabn_probe_empty.argtypes = [i32, i32, i32, i32, vp]
            L.iabn_probe_empty.restype = i32
            L.iabn_probe_read.argtypes = [vp, ctypes.c_size_t, i32, vp]
            L.iabn_probe_read.restype = i32
            L.iabn_probe_read_write.argtypes = [vp, ctypes.c_size_t, i32, vp]
            L.iabn_probe_read_write.restype = i32
            L.iabn_probe_cluster_occupancy.argtypes = [i32, i32, i32, ctypes.POINTER(i32)]
            L.iabn_probe_cluster_occupancy.restype = i32
            _lib = L
    return _lib


def make_desc(shape, layout: int, dtype: int) -> IabnDesc:
    n, c, h, w = (int(v) for v in shape)
    return IabnDesc(n, c, h, w, int(layout), int(dtype))


# -------------------------------------------------------------- raw C calls

def iabn_workspace_size(desc: IabnDesc) -> int:
    return int(lib().iabn_workspace_size(ctypes.byref(desc)))


def iabn_forward(desc, x_inout, gamma, beta, eps, act, act_param, save_mean, save_var,
                 workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_forward(ctypes.byref(desc), x_inout, gamma, beta, eps, act,
                                  act_param, save_mean, save_var, workspace, ws_bytes, stream))


def iabn_forward_with_running_stats(desc, x_inout, gamma, beta, eps, act, act_param, save_mean,
                                    save_var, running_mean, running_var, momentum, workspace,
                                    ws_bytes, stream) -> int:
    return int(lib().iabn_forward_with_running_stats(ctypes.byref(desc), x_inout, gamma, beta,
                                                     eps, act, act_param, save_mean, save_var,
                                                     running_mean, running_var, momentum,
                                                     workspace, ws_bytes, stream))


def iabn_backward(desc, z, dz_inout, gamma, beta, save_var, eps, act, act_param, dgamma,
                  dbeta, workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_backward(ctypes.byref(desc), z, dz_inout, gamma, beta, save_var,
                                   eps, act, act_param, dgamma, dbeta, workspace, ws_bytes,
                                   stream))


def iabn_forward_standard(desc, x, z_out, gamma, beta, eps, act, act_param, save_mean, save_var,
                          workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_forward_standard(ctypes.byref(desc), x, z_out, gamma, beta, eps, act,
                                           act_param, save_mean, save_var, workspace, ws_bytes,
                                           stream))


def iabn_backward_standard(desc, x, dz_inout, gamma, beta, save_mean, save_var, eps, act,
                           act_param, dgamma, dbeta, workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_backward_standard(ctypes.byref(desc), x, dz_inout, gamma, beta,
                                            save_mean, save_var, eps, act, act_param, dgamma,
                                            dbeta, workspace, ws_bytes, stream))


def iabn_forward_checkpoint(desc, x_inout, z_out, gamma, beta, eps, act, act_param, save_mean,
                            save_var, workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_forward_checkpoint(ctypes.byref(desc), x_inout, z_out, gamma, beta,
                                             eps, act, act_param, save_mean, save_var, workspace,
                                             ws_bytes, stream))


def iabn_backward_checkpoint(desc, xhat, dz_inout, gamma, beta, save_var, eps, act, act_param,
                             dgamma, dbeta, workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_backward_checkpoint(ctypes.byref(desc), xhat, dz_inout, gamma, beta,
                                              save_var, eps, act, act_param, dgamma, dbeta,
                                              workspace, ws_bytes, stream))


def iabn_checkpoint_recompute(desc, xhat, z_out, gamma, beta, act, act_param, stream) -> int:
    return int(lib().iabn_checkpoint_recompute(ctypes.byref(desc), xhat, z_out, gamma, beta,
                                               act, act_param, stream))


def iabn_inference(desc, x_inout, gamma, beta, running_mean, running_var, eps, act, act_param,
                   workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_inference(ctypes.byref(desc), x_inout, gamma, beta, running_mean,
                                    running_var, eps, act, act_param, workspace, ws_bytes,
                                    stream))


def iabn_update_running_stats(c, count, save_mean, save_var, running_mean, running_var,
                              momentum, stream) -> int:
    return int(lib().iabn_update_running_stats(c, count, save_mean, save_var, running_mean,
                                               running_var, momentum, stream))


def iabn_get_device_status(workspace, stream) -> int:
    return int(lib().iabn_get_device_status(workspace, stream))


def iabn_kernel_launches() -> int:
    return int(lib().iabn_kernel_launches())


def iabn_forward_static_ws(desc, x_inout, gamma, beta, eps, act, act_param, save_mean,
                           save_var, stream) -> int:
    """iabn_forward with the library's own fixed 8 MiB scratch (no workspace
    argument) for callers that cannot allocate device memory."""
    return int(lib().iabn_forward_static_ws(ctypes.byref(desc), x_inout, gamma, beta, eps, act,
                                            act_param, save_mean, save_var, stream))


def iabn_get_static_ws_status(stream) -> int:
    """Reads and clears the status word of iabn_forward_static_ws's scratch
    on the current device (synchronises the stream)."""
    return int(lib().iabn_get_static_ws_status(stream))


def iabn_describe_plan(desc, call, sm_count, smem_optin, info) -> int:
    return int(lib().iabn_describe_plan(ctypes.byref(desc), call, sm_count, smem_optin,
                                        ctypes.byref(info)))


def iabn_sync_forward_stats(desc, x, stats, workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_sync_forward_stats(ctypes.byref(desc), x, stats, workspace, ws_bytes,
                                             stream))


def iabn_sync_forward_apply(desc, x_inout, gathered, world, gamma, beta, eps, act, act_param,
                            save_mean, save_var, workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_sync_forward_apply(ctypes.byref(desc), x_inout, gathered, world, gamma,
                                             beta, eps, act, act_param, save_mean, save_var,
                                             workspace, ws_bytes, stream))


def iabn_sync_backward_stats(desc, z, dz, gamma, beta, act, act_param, stats, workspace,
                             ws_bytes, stream) -> int:
    return int(lib().iabn_sync_backward_stats(ctypes.byref(desc), z, dz, gamma, beta, act,
                                              act_param, stats, workspace, ws_bytes, stream))


def iabn_sync_backward_apply(desc, z, dz_inout, gathered, world, gamma, beta, save_var, eps, act,
                             act_param, dgamma, dbeta, workspace, ws_bytes, stream) -> int:
    return int(lib().iabn_sync_backward_apply(ctypes.byref(desc), z, dz_inout, gathered, world,
                                              gamma, beta, save_var, eps, act, act_param, dgamma,
                                              dbeta, workspace, ws_bytes, stream))


def iabn_probe_empty(blocks, threads, smem_bytes, cooperative, stream) -> int:
    return int(lib().iabn_probe_empty(blocks, threads, smem_bytes, cooperative, stream))


def iabn_probe_read(src, nbytes, blocks, stream) -> int:
    return int(lib().iabn_probe_read(src, nbytes, blocks, stream))


def iabn_probe_read_write(buf, nbytes, blocks, stream) -> int:
    return int(lib().iabn_probe_read_write(buf, nbytes, blocks, stream))


def iabn_probe_cluster_occupancy(cluster_size, threads, smem_bytes) -> int:
    """The number of co-resident clusters (raises on an error status)."""
    n = ctypes.c_int32(0)
    _ok(int(lib().iabn_probe_cluster_occupancy(cluster_size, threads, smem_bytes,
                                               ctypes.byref(n))),
        "iabn_probe_cluster_occupancy")
    return int(n.value)


# ---------------------------------------------------------- tensor helpers

def _dtype_code(t) -> int:
    import torch
    try:
        return {torch.float32: IABN_F32, torch.bfloat16: IABN_BF16,
                torch.float16: IABN_F16}[t.dtype]
    except KeyError:
        raise IabnError(IABN_ERR_INVALID_ARG, f"unsupported storage dtype {t.dtype}") from None


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    if not t.is_cuda:
        raise IabnError(IABN_ERR_INVALID_ARG, "tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise IabnError(IABN_ERR_INVALID_ARG, "tensor is not contiguous")
    return int(t.data_ptr())


def _ok(status: int, what: str) -> None:
    if status != IABN_OK:
        raise IabnError(status, what)


def workspace_size(shape, layout: int, dtype: int) -> int:
    return iabn_workspace_size(make_desc(shape, layout, dtype))


def describe_plan(shape, layout: int, dtype: int, call: int, *, sm_count: int = 0,
                  smem_optin: int = 0) -> dict:
    """The launch plan and shape the training call ``call`` (IABN_CALL_*; 0 is
    iabn_forward, 1 iabn_backward) takes for this descriptor; sm_count and
    smem_optin describe the device (both 0: the current device)."""
    info = IabnPlanInfo()
    _ok(iabn_describe_plan(make_desc(shape, layout, dtype), int(call), int(sm_count),
                           int(smem_optin), info), "iabn_describe_plan")
    out = {name: int(getattr(info, name)) for name, _ in IabnPlanInfo._fields_}
    out["plan"] = PLAN_NAMES[out["plan"]]
    return out


def new_workspace(shape, layout: int, dtype: int, device=None):
    """A zero-filled workspace tensor (uint8) for this descriptor."""
    import torch
    return torch.zeros(workspace_size(shape, layout, dtype), dtype=torch.uint8, device=device)


def forward(x, gamma, beta, save_mean, save_var, workspace, *, shape, layout: int,
            eps: float, act: int, act_param: float, stream=None) -> None:
    """x (storage dtype, ``shape`` in ``layout``) is overwritten with z."""
    desc = make_desc(shape, layout, _dtype_code(x))
    _ok(iabn_forward(desc, _ptr(x), _ptr(gamma), _ptr(beta), float(eps), int(act),
                     float(act_param), _ptr(save_mean), _ptr(save_var), _ptr(workspace),
                     workspace.numel() * workspace.element_size(), _stream_ptr(stream)),
        "iabn_forward")


def forward_with_running_stats(x, gamma, beta, save_mean, save_var, running_mean, running_var,
                               workspace, *, shape, layout: int, eps: float, act: int,
                               act_param: float, momentum: float, stream=None) -> None:
    """``forward`` plus the running-statistics update, in the forward's own
    launch."""
    desc = make_desc(shape, layout, _dtype_code(x))
    _ok(iabn_forward_with_running_stats(desc, _ptr(x), _ptr(gamma), _ptr(beta), float(eps),
                                        int(act), float(act_param), _ptr(save_mean),
                                        _ptr(save_var), _ptr(running_mean), _ptr(running_var),
                                        float(momentum), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream_ptr(stream)), "iabn_forward_with_running_stats")


def backward(z, dz, gamma, beta, save_var, dgamma, dbeta, workspace, *, shape, layout: int,
             eps: float, act: int, act_param: float, stream=None) -> None:
    """dz is overwritten with dx; dgamma and dbeta are written."""
    desc = make_desc(shape, layout, _dtype_code(z))
    _ok(iabn_backward(desc, _ptr(z), _ptr(dz), _ptr(gamma), _ptr(beta), _ptr(save_var),
                      float(eps), int(act), float(act_param), _ptr(dgamma), _ptr(dbeta),
                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                      _stream_ptr(stream)), "iabn_backward")


def forward_standard(x, z, gamma, beta, save_mean, save_var, workspace, *, shape, layout: int,
                     eps: float, act: int, act_param: float, stream=None) -> None:
    """Standard BN+ACT forward: x is kept, z is written to its own buffer."""
    desc = make_desc(shape, layout, _dtype_code(x))
    _ok(iabn_forward_standard(desc, _ptr(x), _ptr(z), _ptr(gamma), _ptr(beta), float(eps),
                              int(act), float(act_param), _ptr(save_mean), _ptr(save_var),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream_ptr(stream)), "iabn_forward_standard")


def backward_standard(x, dz, gamma, beta, save_mean, save_var, dgamma, dbeta, workspace, *,
                      shape, layout: int, eps: float, act: int, act_param: float,
                      stream=None) -> None:
    """Standard backward from the stored x: dz is overwritten with dx."""
    desc = make_desc(shape, layout, _dtype_code(x))
    _ok(iabn_backward_standard(desc, _ptr(x), _ptr(dz), _ptr(gamma), _ptr(beta),
                               _ptr(save_mean), _ptr(save_var), float(eps), int(act),
                               float(act_param), _ptr(dgamma), _ptr(dbeta), _ptr(workspace),
                               workspace.numel() * workspace.element_size(),
                               _stream_ptr(stream)), "iabn_backward_standard")


def forward_checkpoint(x, z, gamma, beta, save_mean, save_var, workspace, *, shape,
                       layout: int, eps: float, act: int, act_param: float,
                       stream=None) -> None:
    """Checkpointing forward: x is overwritten with xhat, z written to its own buffer."""
    desc = make_desc(shape, layout, _dtype_code(x))
    _ok(iabn_forward_checkpoint(desc, _ptr(x), _ptr(z), _ptr(gamma), _ptr(beta), float(eps),
                                int(act), float(act_param), _ptr(save_mean), _ptr(save_var),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream_ptr(stream)), "iabn_forward_checkpoint")


def backward_checkpoint(xhat, dz, gamma, beta, save_var, dgamma, dbeta, workspace, *, shape,
                        layout: int, eps: float, act: int, act_param: float,
                        stream=None) -> None:
    """Checkpointing backward from the stored xhat: dz is overwritten with dx."""
    desc = make_desc(shape, layout, _dtype_code(xhat))
    _ok(iabn_backward_checkpoint(desc, _ptr(xhat), _ptr(dz), _ptr(gamma), _ptr(beta),
                                 _ptr(save_var), float(eps), int(act), float(act_param),
                                 _ptr(dgamma), _ptr(dbeta), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream)), "iabn_backward_checkpoint")


def checkpoint_recompute(xhat, z, gamma, beta, *, shape, layout: int, act: int,
                         act_param: float, stream=None) -> None:
    """z = phi(gamma*xhat + beta) from the stored xhat."""
    desc = make_desc(shape, layout, _dtype_code(xhat))
    _ok(iabn_checkpoint_recompute(desc, _ptr(xhat), _ptr(z), _ptr(gamma), _ptr(beta), int(act),
                                  float(act_param), _stream_ptr(stream)),
        "iabn_checkpoint_recompute")


def inference(x, gamma, beta, running_mean, running_var, workspace, *, shape, layout: int,
              eps: float, act: int, act_param: float, stream=None) -> None:
    """Evaluation mode: x is overwritten with z computed from the running
    statistics."""
    desc = make_desc(shape, layout, _dtype_code(x))
    _ok(iabn_inference(desc, _ptr(x), _ptr(gamma), _ptr(beta), _ptr(running_mean),
                       _ptr(running_var), float(eps), int(act), float(act_param),
                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                       _stream_ptr(stream)), "iabn_inference")


def update_running_stats(save_mean, save_var, running_mean, running_var, *, count: int,
                         momentum: float, stream=None) -> None:
    _ok(iabn_update_running_stats(save_mean.numel(), int(count), _ptr(save_mean),
                                  _ptr(save_var), _ptr(running_mean), _ptr(running_var),
                                  float(momentum), _stream_ptr(stream)),
        "iabn_update_running_stats")


# ------------------------------------------------------------ INPLACE-ABNsync
# The batch split along N over the ranks of a process group, one GPU each;
# the statistics are the whole batch's.  Records are float64 tensors of C*3
# values (see include/iabn.h); `gathered` holds all ranks' records in rank
# order, shape [world, C*3].

def sync_forward_stats(x, stats, workspace, *, shape, layout: int, stream=None) -> None:
    """This rank's forward record of its shard x into ``stats`` (float64, C*3)."""
    desc = make_desc(shape, layout, _dtype_code(x))
    _ok(iabn_sync_forward_stats(desc, _ptr(x), _ptr(stats), _ptr(workspace),
                                workspace.numel() * workspace.element_size(),
                                _stream_ptr(stream)), "iabn_sync_forward_stats")


def sync_forward_apply(x, gathered, gamma, beta, save_mean, save_var, workspace, *, shape,
                       layout: int, eps: float, act: int, act_param: float, stream=None) -> None:
    """x (this rank's shard) is overwritten with z under the whole batch's
    statistics, which are written to save_mean / save_var."""
    desc = make_desc(shape, layout, _dtype_code(x))
    world = gathered.numel() // (3 * int(shape[1]))
    _ok(iabn_sync_forward_apply(desc, _ptr(x), _ptr(gathered), world, _ptr(gamma), _ptr(beta),
                                float(eps), int(act), float(act_param), _ptr(save_mean),
                                _ptr(save_var), _ptr(workspace),
                                workspace.numel() * workspace.element_size(),
                                _stream_ptr(stream)), "iabn_sync_forward_apply")


def sync_backward_stats(z, dz, gamma, beta, stats, workspace, *, shape, layout: int, act: int,
                        act_param: float, stream=None) -> None:
    """This rank's backward record (n, sum dy, sum dy*xhat) into ``stats``."""
    desc = make_desc(shape, layout, _dtype_code(z))
    _ok(iabn_sync_backward_stats(desc, _ptr(z), _ptr(dz), _ptr(gamma), _ptr(beta), int(act),
                                 float(act_param), _ptr(stats), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream)), "iabn_sync_backward_stats")


def sync_backward_apply(z, dz, gathered, gamma, beta, save_var, dgamma, dbeta, workspace, *,
                        shape, layout: int, eps: float, act: int, act_param: float,
                        stream=None) -> None:
    """dz (this rank's shard) is overwritten with dx; dgamma and dbeta (the
    whole batch's) are written."""
    desc = make_desc(shape, layout, _dtype_code(z))
    world = gathered.numel() // (3 * int(shape[1]))
    _ok(iabn_sync_backward_apply(desc, _ptr(z), _ptr(dz), _ptr(gathered), world, _ptr(gamma),
                                 _ptr(beta), _ptr(save_var), float(eps), int(act),
                                 float(act_param), _ptr(dgamma), _ptr(dbeta), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(),
                                 _stream_ptr(stream)), "iabn_sync_backward_apply")


def gather_records(stats, group=None):
    """All ranks' records in rank order, shape [world, numel]: an all-gather
    over ``group`` (NCCL for CUDA tensors); without an initialised process
    group, this rank's record alone."""
    import torch
    import torch.distributed as dist
    flat = stats.reshape(-1).contiguous()
    if not (dist.is_available() and dist.is_initialized()):
        return flat.reshape(1, -1)
    world = dist.get_world_size(group)
    parts = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(parts, flat, group=group)
    return torch.stack(parts)


def forward_sync(x, gamma, beta, save_mean, save_var, stats, workspace, *, shape, layout: int,
                 eps: float, act: int, act_param: float, group=None, stream=None):
    """INPLACE-ABNsync forward of this rank's shard: record, all-gather,
    apply.  Returns the gathered records (their n column sums to the whole
    batch's values per channel, the count for the running statistics)."""
    sync_forward_stats(x, stats, workspace, shape=shape, layout=layout, stream=stream)
    gathered = gather_records(stats, group)
    sync_forward_apply(x, gathered, gamma, beta, save_mean, save_var, workspace, shape=shape,
                       layout=layout, eps=eps, act=act, act_param=act_param, stream=stream)
    return gathered


def backward_sync(z, dz, gamma, beta, save_var, dgamma, dbeta, stats, workspace, *, shape,
                  layout: int, eps: float, act: int, act_param: float, group=None,
                  stream=None):
    """INPLACE-ABNsync backward of this rank's shard: record, all-gather,
    apply.  Returns the gathered records."""
    sync_backward_stats(z, dz, gamma, beta, stats, workspace, shape=shape, layout=layout,
                        act=act, act_param=act_param, stream=stream)
    gathered = gather_records(stats, group)
    sync_backward_apply(z, dz, gathered, gamma, beta, save_var, dgamma, dbeta, workspace,
                        shape=shape, layout=layout, eps=eps, act=act, act_param=act_param,
                        stream=stream)
    return gathered


def get_static_ws_status(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the status of the
    iabn_forward_static_ws calls on the current device."""
    return iabn_get_static_ws_status(_stream_ptr(stream))


def get_device_status(workspace, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the workspace's device status."""
    return iabn_get_device_status(_ptr(workspace), _stream_ptr(stream))
