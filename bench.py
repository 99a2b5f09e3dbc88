"""Benchmark of the InPlace-ABN layer (training forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole layer over one batch:
iabn_forward_with_running_stats (x -> z in place, the batch statistics, and
the running-statistics update in the forward's finalize) and iabn_backward
(dz -> dx in place, dgamma, dbeta), on the ResNet-trunk workload: NHWC bf16 storage,
N=64 C=256 H=W=56, leaky-ReLU 0.01.  Inputs are synthetic (seeded, same value
recipe as the tests) and restored before every step (the layer is in place);
the L2 cache is flushed (a 2x-L2 write) before every forward and every
backward call, outside the timed events.

Metric: GB/s of compulsory traffic, 5*E*s bytes per step (the forward reads x
and writes z; the backward reads z and dz and writes dx), divided by the
device time of the two calls (CUDA events on the launching stream).  Under
torchrun (N > 1) every rank runs its own replica (no cross-GPU statistics):
value = N * bytes / max-over-ranks time ("weak" scaling).

Prints ONE JSON line on rank 0.  ``--impl reference`` times the fp64 CPU
oracle (test infrastructure) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "InPlace-ABN fwd+bwd GB/s and % of B200 HBM roofline per config; elements/s"
# DRAM bytes per launch (dram__bytes_read.sum, dram__bytes_write.sum) of the
# resident kernels on the ResNet-trunk layer, from one ncu capture:
#   python bench.py --profile 1 --steps 1 --warmup 1
#   ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum,\
#   lts__t_sector_hit_rate.pct,dram__throughput.avg.pct_of_peak_sustained_elapsed \
#       --clock-control none -k regex:k_resident -s 2 -c 2 --csv \
#       python bench.py --profile 1 --steps 1 --warmup 1
# Reported only while the resident kernels' sources (KERNEL_SOURCES) hash to the value
# they were captured on; otherwise "traffic" and "dram_bytes" are null.
NCU_TRAFFIC = {
    "sources_sha256": "bbdc62027627e6b1321072c2715d14102e149c15a87bb35033754587b1702b6b",
    "backward": {"read": 272967424, "write": 32150272},
    "forward": {"read": 102939392, "write": 21014784},
}
# the resident kernels' phase trace in the workspace (IABN_TRACE=1): up to 256
# CTAs x 16 slots of 8 bytes, right after the 256-byte control block
TRACE_SLOTS = 16
TRACE_BYTES = 256 * TRACE_SLOTS * 8
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def measured_hbm_gbs():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The sources the captured resident kernels and their launch plans are built
# from (the kernel template, its instantiations and plan, the device headers).
KERNEL_SOURCES = ("iabn_resident", "iabn_device.cuh", "iabn_bulk.cuh", "iabn_tmem.cuh",
                  "iabn_internal.h")


def kernel_sources_sha256() -> str:
    """sha256 over the sources of the resident kernels (file names and bytes)."""
    import hashlib
    d = os.path.join(ROOT, "place_batchnorm_activation_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(d)):
        if name.endswith((".cu", ".cuh", ".h")) and name.startswith(KERNEL_SOURCES):
            h.update(name.encode())
            with open(os.path.join(d, name), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()


def ncu_traffic(direction: str):
    """Captured DRAM bytes (read + write) per launch, or None if the kernels
    changed since."""
    if kernel_sources_sha256() != NCU_TRAFFIC["sources_sha256"]:
        return None
    return NCU_TRAFFIC[direction]["read"] + NCU_TRAFFIC[direction]["write"]


def ncu_dram(direction: str):
    """The captured DRAM read and write bytes per launch (None if stale)."""
    if kernel_sources_sha256() != NCU_TRAFFIC["sources_sha256"]:
        return None
    return dict(NCU_TRAFFIC[direction])


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads and the CPU baseline")
    ap.add_argument("--profile", type=int, default=0, metavar="WORKLOAD",
                    help="profiling run: only `warmup` + `steps` fwd/bwd/running steps of "
                         "workload 1, 2, 3 or 4 (no e2e, extras or JSON line)")
    ap.add_argument("--layer", type=int, default=0,
                    help="with --profile 4: the layer of the sweep")
    ap.add_argument("--layer-kind", choices=["inplace", "standard", "checkpoint", "inference"],
                    default="inplace",
                    help="with --profile: which layer's calls to run (default: in-place)")
    ap.add_argument("--probe", action="store_true",
                    help="run the measurement probes of include/iabn_probe.h (launch floor, "
                         "L2 retention and read rates, cluster occupancy) and print them")
    return ap.parse_args()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz, self.error = [], set(), None, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(pynvml, device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # no NVML: report why
            self.nv, self.error = None, repr(e)

    @staticmethod
    def _handle(pynvml, idx):
        import torch
        try:
            p = torch.cuda.get_device_properties(idx)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for b, name in self.REASONS.items():
            if bits & b:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:
                self.error = repr(e)
                return
            time.sleep(0.002)

    def __enter__(self):
        if self.nv is not None:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.nv is not None:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
               "samples": len(self.samples)}
        if self.error:
            out["error"] = self.error
        return out


# ------------------------------------------------------------------ inputs

def device_inputs(sp, seed, gen_device):
    """Synthetic layer inputs drawn on the device (same recipe as the tests:
    mu_c ~ U(-2,2), sigma_c ~ U(0.5,3), x = mu + sigma*N(0,1) (Student-t(3)
    for the segmentation workload), gamma = +-U(lo,1.5), beta ~ N(0, 0.1),
    dz ~ N(0,1))."""
    import torch
    import workloads as wl
    g = torch.Generator(device=gen_device).manual_seed(seed)
    n, c, h, w = sp.shape
    dev = gen_device
    mu = torch.rand(c, generator=g, device=dev, dtype=torch.float32) * 4 - 2
    sig = torch.rand(c, generator=g, device=dev) * 2.5 + 0.5
    sign = torch.where(torch.rand(c, generator=g, device=dev) < 0.5, -1.0, 1.0)
    gamma = sign * (torch.rand(c, generator=g, device=dev) * (1.5 - sp.gamma_lo) + sp.gamma_lo)
    beta = torch.randn(c, generator=g, device=dev) * (0.1 ** 0.5)
    shape_l = (n, h, w, c) if sp.layout == wl.NHWC else (n, c, h, w)
    bshape = (1, 1, 1, c) if sp.layout == wl.NHWC else (1, c, 1, 1)
    if sp.x_dist == "student_t3":
        z = torch.randn(shape_l, generator=g, device=dev)
        chi = sum(torch.randn(shape_l, generator=g, device=dev) ** 2 for _ in range(3))
        e = z / torch.sqrt(chi / 3.0)
    else:
        e = torch.randn(shape_l, generator=g, device=dev)
    x = (mu.view(bshape) + sig.view(bshape) * e).to(wl.torch_dtype(sp.dtype)).reshape(-1)
    dz = torch.randn(shape_l, generator=g, device=dev).to(wl.torch_dtype(sp.dtype)).reshape(-1)
    return x, dz, gamma.contiguous(), beta.contiguous()


class Layer:
    """Device buffers of one layer plus its pristine inputs."""

    def __init__(self, sp, seed, device):
        import torch
        import place_batchnorm_activation_b200 as iabn
        self.iabn, self.sp = iabn, sp
        self.x0, self.dz0, self.gamma, self.beta = device_inputs(sp, seed, device)
        self.x = self.x0.clone()
        self.dz = self.dz0.clone()
        c = sp.c
        self.mean = torch.empty(c, device=device)
        self.var = torch.empty(c, device=device)
        self.dgamma = torch.empty(c, device=device)
        self.dbeta = torch.empty(c, device=device)
        self.rmean = torch.zeros(c, device=device)
        self.rvar = torch.ones(c, device=device)
        self.ws = iabn.new_workspace(sp.shape, sp.layout, sp.dtype, device=device)
        self.bytes = 5 * sp.numel * sp.itemsize

    def restore(self):
        self.x.copy_(self.x0)
        self.dz.copy_(self.dz0)

    def fwd(self):
        sp = self.sp
        self.iabn.forward(self.x, self.gamma, self.beta, self.mean, self.var, self.ws,
                          shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act,
                          act_param=sp.act_param)

    def bwd(self):
        sp = self.sp
        self.iabn.backward(self.x, self.dz, self.gamma, self.beta, self.var, self.dgamma,
                           self.dbeta, self.ws, shape=sp.shape, layout=sp.layout, eps=sp.eps,
                           act=sp.act, act_param=sp.act_param)

    def run(self):
        self.iabn.update_running_stats(self.mean, self.var, self.rmean, self.rvar,
                                       count=self.sp.per_channel, momentum=self.sp.momentum)

    def fwd_train(self):
        """The training step's forward: z over x, the batch statistics and the
        running-statistics update, in one call."""
        sp = self.sp
        self.iabn.forward_with_running_stats(self.x, self.gamma, self.beta, self.mean, self.var,
                                             self.rmean, self.rvar, self.ws, shape=sp.shape,
                                             layout=sp.layout, eps=sp.eps, act=sp.act,
                                             act_param=sp.act_param, momentum=sp.momentum)


class L2Flush:
    """Evicts the L2 before a timed call: writes a buffer of twice the L2 size,
    then reads another one as large, so the L2 holds only clean lines and the
    timed kernel is not charged for writing back the flush's own dirty data.
    ``write_only=True`` skips the read (the timed kernel then pays for that
    write-back)."""

    def __init__(self, device, write_only=False):
        import torch
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        n = 2 * max(l2, 64 << 20)
        self.w = torch.empty(n, dtype=torch.uint8, device=device)
        self.r = torch.ones(n // 4, dtype=torch.float32, device=device)
        self.write_only = write_only

    def zero_(self):
        self.w.zero_()
        if not self.write_only:
            self.r.sum()

    def read_(self):
        """The clean-read half alone: reading 2x L2 of other data evicts every
        line the previous kernel left in L2 (dirty ones are written back)."""
        self.r.sum()


def timed_layer_steps(layer, flush, steps, warmup, dist_barrier=None, sampler=None):
    """Warm-up, then `steps` timed steps; returns per-step event times (ms) of
    the forward (with the running-statistics update in its finalize) and the
    backward, a list of zeros for a separate running update (there is none),
    and the launch count in between."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(warmup):
        layer.restore()
        flush.zero_()
        layer.fwd_train()
        flush.zero_()
        layer.bwd()
    records = [(ev(), ev(), ev(), ev()) for _ in range(steps)]
    if dist_barrier:
        dist_barrier()
    torch.cuda.synchronize()
    l0 = layer.iabn.iabn_kernel_launches()
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        t0 = time.perf_counter()
        for r in records:
            layer.restore()
            flush.zero_()
            r[0].record()
            layer.fwd_train()
            r[1].record()
            flush.zero_()
            r[2].record()
            layer.bwd()
            r[3].record()
        if dist_barrier:
            dist_barrier()
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    launches = layer.iabn.iabn_kernel_launches() - l0
    f = [r[0].elapsed_time(r[1]) for r in records]
    b = [r[2].elapsed_time(r[3]) for r in records]
    u = [0.0 for _ in records]
    return f, b, u, launches, wall


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def e2e_steps(layer, steps, warmup):
    """Through the public API with host buffers, every step: pinned host x and
    dz -> device, the forward (with the running-statistics update) and the
    backward, z and dx (and dgamma, dbeta) -> host.  Copies and compute run on
    three streams over two device buffer sets, so step i+1's host-to-device
    copies overlap step i's kernels and device-to-host copies (PCIe carries
    both directions at once), and z goes back while the backward reads it.
    Returns per-step ms (the whole run's device time over the steps) and the
    bytes moved each way per step."""
    import torch
    sp = layer.sp
    hx = layer.x0.cpu().pin_memory()
    hdz = layer.dz0.cpu().pin_memory()
    hz = torch.empty_like(hx).pin_memory()
    hdx = torch.empty_like(hdz).pin_memory()
    hg = torch.empty_like(layer.dgamma, device="cpu").pin_memory()
    hb = torch.empty_like(layer.dbeta, device="cpu").pin_memory()
    dev = layer.x.device
    slots = [dict(x=layer.x, dz=layer.dz, dg=layer.dgamma, db=layer.dbeta),
             dict(x=torch.empty_like(layer.x), dz=torch.empty_like(layer.dz),
                  dg=torch.empty_like(layer.dgamma), db=torch.empty_like(layer.dbeta))]
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    freed = [None, None]   # event: the slot's device-to-host copies are done
    kw = dict(shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act, act_param=sp.act_param)

    def step(i):
        k = slots[i % 2]
        with torch.cuda.stream(s_in):
            if freed[i % 2] is not None:
                s_in.wait_event(freed[i % 2])
            k["x"].copy_(hx, non_blocking=True)
            x_in = ev()
            x_in.record(s_in)
            k["dz"].copy_(hdz, non_blocking=True)
            dz_in = ev()
            dz_in.record(s_in)
        s_run.wait_event(x_in)
        layer.iabn.forward_with_running_stats(k["x"], layer.gamma, layer.beta, layer.mean,
                                              layer.var, layer.rmean, layer.rvar, layer.ws,
                                              momentum=sp.momentum, stream=s_run, **kw)
        fwd_done = ev()
        fwd_done.record(s_run)
        s_run.wait_event(dz_in)
        layer.iabn.backward(k["x"], k["dz"], layer.gamma, layer.beta, layer.var, k["dg"],
                            k["db"], layer.ws, stream=s_run, **kw)
        bwd_done = ev()
        bwd_done.record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(fwd_done)
            hz.copy_(k["x"], non_blocking=True)      # z, while the backward reads it
            s_out.wait_event(bwd_done)
            hdx.copy_(k["dz"], non_blocking=True)
            hg.copy_(k["dg"], non_blocking=True)
            hb.copy_(k["db"], non_blocking=True)
            freed[i % 2] = ev()
            freed[i % 2].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(warmup, warmup + steps):
        step(i)
    s_in.wait_stream(s_out)
    s_in.wait_stream(s_run)
    t1.record(s_in)
    torch.cuda.synchronize()
    ms = [t0.elapsed_time(t1) / steps] * steps
    h2d = hx.numel() * hx.element_size() + hdz.numel() * hdz.element_size()
    d2h = (hz.numel() * hz.element_size() + hdx.numel() * hdx.element_size()
           + hg.numel() * 4 + hb.numel() * 4)
    return ms, h2d, d2h


def drained_steps(layer, flush, steps, warmup):
    """The same steps with each call's dirty output drained inside its own
    events: call, then the clean-read half of the flush (which writes back
    whatever the call left dirty in L2), minus that read's time on an L2 that
    holds only clean lines.  Returns (fwd_ms, bwd_ms, read_ms) medians."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)
    recs = []
    for i in range(warmup + steps):
        layer.restore()
        r = [ev() for _ in range(6)]
        flush.zero_()
        r[0].record()
        flush.read_()
        r[1].record()
        flush.zero_()
        r[2].record()
        layer.fwd_train()
        flush.read_()
        r[3].record()
        flush.zero_()
        r[4].record()
        layer.bwd()
        flush.read_()
        r[5].record()
        if i >= warmup:
            recs.append(r)
    torch.cuda.synchronize()
    rd = statistics.median(r[0].elapsed_time(r[1]) for r in recs)
    f = statistics.median(r[2].elapsed_time(r[3]) for r in recs) - rd
    b = statistics.median(r[4].elapsed_time(r[5]) for r in recs) - rd
    return f, b, rd


class LayerVariants(Layer):
    """One workload's buffers for the three layers the pages compare: the
    in-place layer (keeps z), the standard BN+ACT layer (keeps x and z) and
    the optimized-checkpointing layer (keeps xhat)."""

    def __init__(self, sp, seed, device):
        import torch
        super().__init__(sp, seed, device)
        self.z = torch.empty_like(self.x)

    def kw(self):
        sp = self.sp
        return dict(shape=sp.shape, layout=sp.layout, eps=sp.eps, act=sp.act,
                    act_param=sp.act_param)

    def calls(self, variant):
        """(name, callable) of one step of `variant`, in order."""
        io = self.iabn
        if variant == "inplace":
            return [("fwd", self.fwd), ("bwd", self.bwd)]
        if variant == "standard":
            return [("fwd", lambda: io.forward_standard(self.x, self.z, self.gamma, self.beta,
                                                        self.mean, self.var, self.ws,
                                                        **self.kw())),
                    ("bwd", lambda: io.backward_standard(self.x, self.dz, self.gamma, self.beta,
                                                         self.mean, self.var, self.dgamma,
                                                         self.dbeta, self.ws, **self.kw()))]
        kw = self.kw()
        return [("fwd", lambda: io.forward_checkpoint(self.x, self.z, self.gamma, self.beta,
                                                      self.mean, self.var, self.ws, **kw)),
                ("recompute", lambda: io.checkpoint_recompute(
                    self.x, self.z, self.gamma, self.beta, shape=kw["shape"],
                    layout=kw["layout"], act=kw["act"], act_param=kw["act_param"])),
                ("bwd", lambda: io.backward_checkpoint(self.x, self.dz, self.gamma, self.beta,
                                                       self.var, self.dgamma, self.dbeta,
                                                       self.ws, **kw))]


# bytes each layer reads and writes per step, in units of E*s
LAYER_TRAFFIC = {"inplace": {"fwd": 2, "bwd": 3}, "standard": {"fwd": 2, "bwd": 3},
                 "checkpoint": {"fwd": 3, "recompute": 2, "bwd": 3}}
# activation buffers a layer keeps from its forward to its backward, in units of E*s
LAYER_KEPT = {"inplace": 1, "standard": 2, "checkpoint": 1}


def bench_layer_variants(flush, steps, warmup, device):
    """The in-place layer against the standard BN+ACT layer and the
    optimized-checkpointing layer on workloads 1-3 (same protocol: L2
    flushed before every call, inputs restored before every step)."""
    import torch
    import workloads as wl
    ev = lambda: torch.cuda.Event(enable_timing=True)
    out = {}
    for wid in (1, 2, 3):
        sp = wl.spec(wid)
        L = LayerVariants(sp, sp.seed, device)
        es = sp.numel * sp.itemsize
        res = {}
        for variant in ("inplace", "standard", "checkpoint"):
            calls = L.calls(variant)
            times = {name: [] for name, _ in calls}
            for i in range(warmup + steps):
                L.restore()
                for name, fn in calls:
                    flush.zero_()
                    a, b = ev(), ev()
                    a.record()
                    fn()
                    b.record()
                    if i >= warmup:
                        times[name].append((a, b))
            torch.cuda.synchronize()
            us = {k: statistics.median(a.elapsed_time(b) for a, b in v) * 1e3
                  for k, v in times.items()}
            total = sum(us.values())
            nbytes = sum(LAYER_TRAFFIC[variant].values()) * es
            res[variant] = {**{f"{k}_us": round(v, 2) for k, v in us.items()},
                            "step_us": round(total, 2),
                            "compulsory_bytes": nbytes,
                            "gbs": round(nbytes / (total * 1e-6) / 1e9, 1),
                            "kept_for_backward_bytes": LAYER_KEPT[variant] * es}
        std = res["standard"]
        for variant in ("inplace", "checkpoint"):
            r = res[variant]
            r["time_vs_standard_pct"] = round(100.0 * (r["step_us"] / std["step_us"] - 1.0), 2)
            r["memory_saving_vs_standard_pct"] = round(
                100.0 * (1.0 - r["kept_for_backward_bytes"] / std["kept_for_backward_bytes"]), 1)
        out[sp.name] = res
        del L
        torch.cuda.empty_cache()
    out["pages"] = ("InPlace-ABN vs standard BN+ACT on 4x Titan Xp (Pascal): up to 50% training "
                    "memory saved, 0.8-2% more computation time (whole networks)")
    return out


# -------------------------------------------------------- other workloads

def bench_other_workloads(flush, steps, warmup, hbm_peak, device):
    """Workloads 2-4 of the layer's benchmark set, same protocol (L2 flushed
    before every call).  The layer sweep chains 16 layers (x_{l+1} is a
    subsampled, channel-cycled copy of z_l, made outside the timed events),
    forward l = 0..15 then backward l = 15..0 with a fresh dz per layer."""
    import torch
    import workloads as wl
    out = {}
    for wid in (2, 3):
        sp = wl.spec(wid)
        L = Layer(sp, sp.seed, device)
        f, b, u, _, _ = timed_layer_steps(L, flush, steps, warmup)
        tf, tb = statistics.median(f), statistics.median(b)
        gbs = L.bytes / ((tf + tb) * 1e-3) / 1e9
        out[sp.name] = {"fwd_us": round(tf * 1e3, 2), "bwd_us": round(tb * 1e3, 2),
                        "gbs": round(gbs, 1), "frac_hbm_peak": round(gbs / hbm_peak, 4),
                        "frac_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                        "elements_per_s": sp.numel / ((tf + tb) * 1e-3)}
        del L
        torch.cuda.empty_cache()
    # layer sweep
    layers = []
    for l in range(len(wl.SWEEP_SHAPES)):
        sp = wl.spec(4, l)
        layers.append(Layer(sp, sp.seed, device))
    base0 = layers[0].x0.clone()

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def one_pass(rec):
        layers[0].x.copy_(base0)
        for l, L in enumerate(layers):
            if l > 0:
                a, b = layers[l - 1], L
                za = a.x.view(a.sp.n, a.sp.h, a.sp.w, a.sp.c)
                r = a.sp.h // b.sp.h
                idx = torch.arange(b.sp.c, device=device) % a.sp.c
                b.x.copy_(za[:, ::r, ::r, :][..., idx].reshape(-1))
            flush.zero_()
            rec[2 * l][0].record()
            L.fwd()
            rec[2 * l][1].record()
        for l in range(len(layers) - 1, -1, -1):
            L = layers[l]
            L.dz.copy_(L.dz0)
            flush.zero_()
            rec[2 * l + 1][0].record()
            L.bwd()
            rec[2 * l + 1][1].record()

    for _ in range(warmup):
        one_pass([(ev(), ev()) for _ in range(2 * len(layers))])
    torch.cuda.synchronize()
    totals = []
    for _ in range(max(3, steps // 4)):
        rec = [(ev(), ev()) for _ in range(2 * len(layers))]
        one_pass(rec)
        torch.cuda.synchronize()
        totals.append(sum(a.elapsed_time(b) for a, b in rec))
    t = statistics.median(totals)
    total_bytes = sum(L.bytes for L in layers)
    gbs = total_bytes / (t * 1e-3) / 1e9
    out["layer_sweep"] = {"sum_of_32_calls_us": round(t * 1e3, 2), "gbs": round(gbs, 1),
                          "frac_hbm_peak": round(gbs / hbm_peak, 4),
                          "frac_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                          "elements_per_s": sum(L.sp.numel for L in layers) / (t * 1e-3),
                          "dz": "fresh N(0,1) per layer"}
    del layers
    torch.cuda.empty_cache()
    return out


def bench_inference(flush, steps, warmup, hbm_peak, device):
    """Evaluation mode (iabn_inference) on the ResNet-trunk layer, with the
    running statistics of three training steps; L2 flushed before every
    call, x restored between calls (outside the timed events).  Traffic:
    read x, write z = 2*E*s."""
    import torch
    import workloads as wl
    sp = wl.spec(1)
    L = Layer(sp, sp.seed, device)
    for _ in range(3):
        L.restore()
        L.fwd()
        L.run()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    recs = []
    l0 = L.iabn.iabn_kernel_launches()
    for i in range(warmup + steps):
        L.restore()
        flush.zero_()
        a, b = ev(), ev()
        a.record()
        L.iabn.inference(L.x, L.gamma, L.beta, L.rmean, L.rvar, L.ws, shape=sp.shape,
                         layout=sp.layout, eps=sp.eps, act=sp.act, act_param=sp.act_param)
        b.record()
        if i >= warmup:
            recs.append((a, b))
    torch.cuda.synchronize()
    calls = warmup + steps
    launches = (L.iabn.iabn_kernel_launches() - l0) / calls
    t = statistics.median(a.elapsed_time(b) for a, b in recs)
    nbytes = 2 * sp.numel * sp.itemsize
    gbs = nbytes / (t * 1e-3) / 1e9
    del L
    torch.cuda.empty_cache()
    return {"us": round(t * 1e3, 2), "gbs": round(gbs, 1),
            "frac_hbm_peak": round(gbs / hbm_peak, 4), "bytes_per_call": nbytes,
            "launches_per_call": launches,
            "plan": "one launch: coefficients formed in the elementwise pass"}


def bench_twophase(flush, steps, warmup, hbm_peak, device):
    """The fallback plan (three launches per call, for the shapes the
    resident plan declines) forced on the ResNet-trunk layer, same protocol."""
    import torch
    import workloads as wl
    old = os.environ.get("IABN_FORCE_PLAN")
    os.environ["IABN_FORCE_PLAN"] = "twophase"
    try:
        sp = wl.spec(1)
        L = Layer(sp, sp.seed, device)
        f, b, u, launches, _ = timed_layer_steps(L, flush, steps, warmup)
    finally:
        if old is None:
            os.environ.pop("IABN_FORCE_PLAN", None)
        else:
            os.environ["IABN_FORCE_PLAN"] = old
    tf, tb = statistics.median(f), statistics.median(b)
    gbs = L.bytes / ((tf + tb) * 1e-3) / 1e9
    del L
    torch.cuda.empty_cache()
    return {"fwd_us": round(tf * 1e3, 2), "bwd_us": round(tb * 1e3, 2), "gbs": round(gbs, 1),
            "frac_hbm_peak": round(gbs / hbm_peak, 4),
            "launches_per_step": launches / max(1, steps),
            "plan": "IABN_FORCE_PLAN=twophase"}


def bench_sync(flush, steps, warmup, hbm_peak, device):
    """INPLACE-ABNsync on the ResNet-trunk layer with one rank: the record
    and apply calls of each direction through the C ABI, with the GPU's own
    record as the gathered array (with more GPUs an all-gather of 24*C bytes
    per GPU sits between the two calls); L2 flushed before each direction,
    x and dz restored between steps, outside the timed events."""
    import torch
    import workloads as wl
    sp = wl.spec(1)
    L = Layer(sp, sp.seed, device)
    iabn = L.iabn
    rec = torch.empty(sp.c * 3, dtype=torch.float64, device=device)
    kw = dict(shape=sp.shape, layout=sp.layout)
    act = dict(eps=sp.eps, act=sp.act, act_param=sp.act_param)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    recs = []
    l0 = iabn.iabn_kernel_launches()
    for i in range(warmup + steps):
        L.restore()
        r = [ev() for _ in range(4)]
        flush.zero_()
        r[0].record()
        iabn.sync_forward_stats(L.x, rec, L.ws, **kw)
        iabn.sync_forward_apply(L.x, rec.view(1, -1), L.gamma, L.beta, L.mean, L.var, L.ws,
                                **kw, **act)
        r[1].record()
        flush.zero_()
        r[2].record()
        iabn.sync_backward_stats(L.x, L.dz, L.gamma, L.beta, rec, L.ws, **kw, act=sp.act,
                                 act_param=sp.act_param)
        iabn.sync_backward_apply(L.x, L.dz, rec.view(1, -1), L.gamma, L.beta, L.var, L.dgamma,
                                 L.dbeta, L.ws, **kw, **act)
        r[3].record()
        if i >= warmup:
            recs.append(r)
    torch.cuda.synchronize()
    launches = (iabn.iabn_kernel_launches() - l0) / (warmup + steps)
    tf = statistics.median(r[0].elapsed_time(r[1]) for r in recs)
    tb = statistics.median(r[2].elapsed_time(r[3]) for r in recs)
    gbs = L.bytes / ((tf + tb) * 1e-3) / 1e9
    del L
    torch.cuda.empty_cache()
    return {"fwd_us": round(tf * 1e3, 2), "bwd_us": round(tb * 1e3, 2), "gbs": round(gbs, 1),
            "frac_hbm_peak": round(gbs / hbm_peak, 4), "launches_per_step": launches,
            "world": 1,
            "plan": "record call (two-phase statistics / reduce kernel + record kernel), "
                    "apply call (rank-order combine + elementwise pass), per direction"}


# ------------------------------------------------------------ CPU (oracle)

def oracle_pass(sp_sample):
    """One forward + backward + running update of the oracle on a sample."""
    import numpy as np
    import oracle
    import workloads as wl
    inp = wl.draw(sp_sample)
    g, b = inp.gamma.astype(np.float64), inp.beta.astype(np.float64)
    eps, p = float(np.float32(sp_sample.eps)), float(np.float32(sp_sample.act_param))
    t0 = time.perf_counter()
    fw = oracle.forward(sp_sample.shape, sp_sample.layout, inp.x64, g, b, eps, sp_sample.act, p)
    z = oracle.round_to(fw["z"], sp_sample.dtype)
    bw = oracle.backward_inplace(sp_sample.shape, sp_sample.layout, z, inp.dz64, g, b,
                                 fw["var"], eps, sp_sample.act, p)
    oracle.round_to(bw["dx"], sp_sample.dtype)
    oracle.running_update(sp_sample.per_channel, fw["mean"], fw["var"], 0.1,
                          inp.running_mean, inp.running_var)
    return time.perf_counter() - t0


def host_cpu():
    """(logical cores, CPU model) of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def cpu_baseline():
    """The fp64 C oracle on the bench workload itself (N=64), one
    fwd+bwd+running update: the -fopenmp build on all host cores (the
    reported value) and the plain build on one core."""
    import oracle
    import workloads as wl
    sp = wl.spec(1)
    cores, model = host_cpu()
    nbytes = 5 * sp.numel * sp.itemsize
    oracle.openmp(True)
    try:
        t_all = oracle_pass(sp)
    finally:
        oracle.openmp(False)
    t_one = oracle_pass(sp)
    return {"value": round(nbytes / t_all / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle", "cpu_model": model,
            "sample": f"the resnet_trunk workload itself (N=64, {sp.numel} elements), one "
                      f"fwd+bwd+running update of the fp64 C oracle built with -fopenmp, "
                      f"channel loops over all {cores} host threads: {t_all:.2f} s",
            "single_thread": {"value": round(nbytes / t_one / 1e9, 4), "unit": "GB/s",
                              "cores": 1, "seconds": round(t_one, 2)}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import workloads as wl
    sp = wl.spec(1).with_(n=8)
    cores, model = host_cpu()
    oracle.openmp(True)
    for _ in range(args.warmup):
        oracle_pass(sp)
    times = [oracle_pass(sp) for _ in range(args.steps)]
    oracle.openmp(False)
    t = statistics.mean(times)
    gbs = 5 * sp.numel * sp.itemsize / t / 1e9
    line = {"metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "resnet_trunk NHWC bf16 N=64 C=256 H=W=56 leaky_relu 0.01, "
                                   "fwd+bwd+running stats; each step a bounded sample N=8",
                       "sample_elements": sp.numel},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "cpu_model": model,
                             "sample": f"N=8 slice of the resnet_trunk workload "
                                       f"({sp.numel} elements) per step, fp64 C oracle built "
                                       f"with -fopenmp on all {cores} host threads"},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------- multi-rank

def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (plain value when world == 1)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processed its own replica of the work;
    the job took as long as the slowest rank."""
    return world * bytes_per_rank / (max_ms * 1e-3) / 1e9


# ------------------------------------------------------------------- main

def run_profile(args):
    """Warm-up plus `steps` timed steps of one workload; prints per-call times."""
    import torch
    import workloads as wl
    device = torch.device("cuda", 0)
    flush = L2Flush(device, write_only=os.environ.get("IABN_BENCH_WRITE_FLUSH") == "1")
    sp = wl.spec(args.profile, args.layer if args.profile == 4 else 0)
    if args.layer_kind != "inplace":
        # per-call times of the other layers' calls, same protocol
        L = LayerVariants(sp, sp.seed, device)
        if args.layer_kind == "inference":
            for _ in range(3):
                L.restore()
                L.fwd()
                L.run()
            calls = [("inference", lambda: L.iabn.inference(
                L.x, L.gamma, L.beta, L.rmean, L.rvar, L.ws, **L.kw()))]
        else:
            calls = L.calls(args.layer_kind)
        times = {name: [] for name, _ in calls}
        for i in range(args.warmup + args.steps):
            L.restore()
            for name, fn in calls:
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                if i >= args.warmup:
                    times[name].append((a, b))
        torch.cuda.synchronize()
        print(f"profile {sp.name} {args.layer_kind}: " + " ".join(
            f"{k}_us={statistics.mean(x.elapsed_time(y) for x, y in v) * 1e3:.2f}"
            for k, v in times.items()), flush=True)
        return 0
    layer = Layer(sp, sp.seed, device)
    f, b, u, launches, _ = timed_layer_steps(layer, flush, args.steps, args.warmup)
    print(f"profile {sp.name}: fwd_us={statistics.mean(f) * 1e3:.2f} "
          f"bwd_us={statistics.mean(b) * 1e3:.2f} launches={launches}", flush=True)
    if os.environ.get("IABN_TRACE") == "1":
        # phase stamps of the resident kernels (see k_resident): per-CTA times
        # relative to the earliest CTA start, median / min / max over CTAs (us)
        names = ["start", "phaseA", "merged", "barrier1", "finalize", "barrier2",
                 "merge_rounds", "last_refill", "exit"]
        for what, call in (("fwd", layer.fwd), ("bwd", layer.bwd)):
            layer.restore()
            flush.zero_()
            if what == "bwd":
                layer.fwd()
                flush.zero_()
                layer.ws[256:256 + TRACE_BYTES].zero_()
            else:
                layer.ws[256:256 + TRACE_BYTES].zero_()
            call()
            torch.cuda.synchronize()
            tr = layer.ws[256:256 + TRACE_BYTES].view(torch.int64).view(256, TRACE_SLOTS).cpu()
            rows = [r for r in tr.tolist() if r[0] != 0]
            if not rows:
                print(f"trace {sp.name} {what}: no resident-kernel stamps (two-phase plan)",
                      flush=True)
                continue
            t0 = min(r[0] for r in rows)
            parts = []
            for k, nm in enumerate(names):
                # a stamp this kernel does not take (the NCHW kernels have no
                # in-CTA merge rounds) stays 0
                if any(r[k] == 0 for r in rows):
                    parts.append(f"{nm}=n/a")
                    continue
                v = sorted((r[k] - t0) / 1e3 for r in rows)
                parts.append(f"{nm}={v[len(v) // 2]:.1f}[{v[0]:.1f},{v[-1]:.1f}]")
            for k, nm in ((9, "A.wait_kcyc"), (10, "A.work_kcyc"), (13, "A.comp_kcyc"),
                          (11, "B.wait_kcyc"), (12, "B.work_kcyc"), (15, "B.comp_kcyc")):
                v = sorted(r[k] / 1e3 for r in rows)
                parts.append(f"{nm}={v[len(v) // 2]:.1f}")
            print(f"trace {sp.name} {what} ({len(rows)} CTAs): " + " ".join(parts), flush=True)
    return 0


def run_probe(args):
    """The measurement probes of include/iabn_probe.h on GPU 0.

    * launch floor: CUDA events around nothing, around one empty kernel of the
      resident kernel's shape (148 x 320; without and with the cooperative
      attribute and the resident kernel's dynamic shared memory) and around
      two; the bench's L2 flush before every window; median of 40.
    * L2: for a buffer of S MB, a read after the flush (cold), a second read
      of the same bytes in the same order (what L2 kept), then an in-place
      read + write; mean of 3 after one discarded round.  Marginal rates come
      from the difference between two sizes, which cancels the launch cost.
    * cluster occupancy: co-resident clusters of 1..16 blocks of 320 threads
      with the resident kernel's dynamic shared memory (a host query).
    """
    import torch
    import place_batchnorm_activation_b200 as iabn
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    sms = props.multi_processor_count
    optin = int(getattr(props, "shared_memory_per_block_optin", 232448))
    smem = optin - 1024
    flush = L2Flush(device)
    st = torch.cuda.current_stream(device)
    sh = ctypes.c_void_p(st.cuda_stream)

    def ok(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what}: status {rc}")

    def timed(fn, reps, discard=0):
        ts = []
        for r in range(reps + discard):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            b.synchronize()
            if r >= discard:
                ts.append(a.elapsed_time(b) * 1e3)
        return ts

    floor = {}
    cases = [("events only", []),
             ("empty 148x320, no shared memory, plain", [(0, 0)]),
             ("the same, cooperative", [(0, 1)]),
             (f"the same with {smem // 1024} KB dynamic shared memory, plain", [(smem, 0)]),
             ("the same, cooperative", [(smem, 1)]),
             (f"two {smem // 1024} KB cooperative empty kernels", [(smem, 1), (smem, 1)])]
    for i, (name, launches) in enumerate(cases):
        def fn(launches=launches):
            for sm_bytes, coop in launches:
                ok(iabn.iabn_probe_empty(sms, 320, sm_bytes, coop, sh), "iabn_probe_empty")
        floor[f"{i}: {name}"] = round(statistics.median(timed(fn, 40, 3)), 2)

    MB = 1 << 20
    sizes = [24, 40, 56, 72, 88, 104, 120, 160]
    buf = torch.zeros(max(sizes) * MB, dtype=torch.uint8, device=device)
    l2 = {}
    for S in sizes:
        nb = S * MB
        cold, warm, rw = [], [], []
        for r in range(4):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record(st)
            ok(iabn.iabn_probe_read(buf.data_ptr(), nb, sms, sh), "iabn_probe_read")
            ev[1].record(st)
            ok(iabn.iabn_probe_read(buf.data_ptr(), nb, sms, sh), "iabn_probe_read")
            ev[2].record(st)
            ok(iabn.iabn_probe_read_write(buf.data_ptr(), nb, sms, sh), "iabn_probe_read_write")
            ev[3].record(st)
            ev[3].synchronize()
            if r > 0:
                cold.append(ev[0].elapsed_time(ev[1]) * 1e3)
                warm.append(ev[1].elapsed_time(ev[2]) * 1e3)
                rw.append(ev[2].elapsed_time(ev[3]) * 1e3)
        l2[S] = {"cold_read_us": round(statistics.mean(cold), 2),
                 "re_read_us": round(statistics.mean(warm), 2),
                 "read_write_us": round(statistics.mean(rw), 2)}
    lo, hi = 24, 72

    def marginal(key, factor=1):
        dt = l2[hi][key] - l2[lo][key]
        return round(factor * (hi - lo) * MB / (dt * 1e3), 1) if dt > 0 else None

    rates = {"dram_read_gbs": marginal("cold_read_us"),
             "l2_hit_read_gbs": marginal("re_read_us"),
             "l2_read_plus_write_gbs": marginal("read_write_us", 2),
             "sizes_mb": [lo, hi]}
    clusters = {k: iabn.iabn_probe_cluster_occupancy(k, 320, smem) for k in (1, 2, 4, 8, 16)}
    for name, us in floor.items():
        print(f"floor  {name}: {us} us", flush=True)
    for S, v in l2.items():
        print(f"l2     {S:4d} MB: cold {v['cold_read_us']:.2f} us  re-read {v['re_read_us']:.2f} us"
              f"  read+write {v['read_write_us']:.2f} us", flush=True)
    print(f"rates  {rates}", flush=True)
    for k, n in clusters.items():
        print(f"clusters of {k:2d}: {n} resident ({n * k} blocks of {sms} SMs)", flush=True)
    print(json.dumps({"probe": {"sms": sms, "launch_floor_us": floor, "l2_mb": l2,
                                "marginal_rates": rates,
                                "clusters": {str(k): v for k, v in clusters.items()},
                                "smem_bytes": smem}}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.probe:
        return run_probe(args)
    if args.profile:
        return run_profile(args)
    import torch
    import torch.distributed as dist
    import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    barrier = None
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        barrier = dist.barrier

    hbm_peak, peak_kind = measured_hbm_gbs()
    flush = L2Flush(device)
    sp = wl.spec(1)
    layer = Layer(sp, sp.seed + 1000 * rank, device)

    sampler = ClockSampler(local)
    f, b, u, launches, wall = timed_layer_steps(layer, flush, args.steps, args.warmup,
                                                barrier, sampler)
    t_step = [x + y + z for x, y, z in zip(f, b, u)]
    mean_ms = statistics.mean(t_step)
    # the same steps with a write-only flush (the kernels then also pay for
    # writing back the flush's dirty lines)
    fw, bw, uw, _, _ = timed_layer_steps(layer, L2Flush(device, write_only=True),
                                         max(5, args.steps // 5), 2, barrier)
    wf_ms = reduce_max(statistics.mean([x + y + z for x, y, z in zip(fw, bw, uw)]), world,
                       device)
    t_max = reduce_max(mean_ms, world, device)
    value = whole_job_gbs(layer.bytes, world, t_max)
    fwd_us, bwd_us = statistics.mean(f) * 1e3, statistics.mean(b) * 1e3
    # the same steps with each call's dirty output written back inside its events
    df, db, drd = drained_steps(layer, flush, max(5, args.steps // 5), 2)
    d_ms = reduce_max(df + db + statistics.mean(u), world, device)

    # e2e through host buffers
    e_ms, h2d, d2h = e2e_steps(layer, max(5, args.steps // 5), 2)
    e_max = reduce_max(statistics.mean(e_ms), world, device)
    e2e_value = whole_job_gbs(layer.bytes, world, e_max)

    extra = {}
    if not args.no_extra and world == 1:
        extra = bench_other_workloads(flush, max(5, args.steps // 5), 3, hbm_peak, device)
        try:
            extra["inference_resnet_trunk"] = bench_inference(flush, max(5, args.steps // 5), 3,
                                                              hbm_peak, device)
        except Exception as e:  # reported in the line; never fatal for the headline
            extra["inference_resnet_trunk"] = {"error": f"{type(e).__name__}: {e}"}
        try:
            extra["twophase_resnet_trunk"] = bench_twophase(flush, max(5, args.steps // 5), 3,
                                                            hbm_peak, device)
        except Exception as e:
            extra["twophase_resnet_trunk"] = {"error": f"{type(e).__name__}: {e}"}
        try:
            extra["sync_resnet_trunk"] = bench_sync(flush, max(5, args.steps // 5), 3, hbm_peak,
                                                    device)
        except Exception as e:
            extra["sync_resnet_trunk"] = {"error": f"{type(e).__name__}: {e}"}
        try:
            extra["layers_vs_standard"] = bench_layer_variants(flush, max(5, args.steps // 5), 3,
                                                               device)
        except Exception as e:
            extra["layers_vs_standard"] = {"error": f"{type(e).__name__}: {e}"}

    if rank == 0:
        bwd_bytes = 3 * sp.numel * sp.itemsize
        achieved = bwd_bytes / (bwd_us * 1e-6) / 1e9
        fwd_achieved = 2 * sp.numel * sp.itemsize / (fwd_us * 1e-6) / 1e9
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_max, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "resnet_trunk: NHWC, bf16 storage, N=64 C=256 H=W=56, "
                                   "leaky_relu 0.01, eps 1e-5, fwd+bwd+running stats",
                       "storage_dtype": "bf16", "elements": sp.numel,
                       "compulsory_bytes_per_step": layer.bytes,
                       "l2": "flushed before every fwd and every bwd call: write 2x L2, then "
                             "read another 2x L2 so only clean lines remain (outside the "
                             "timed events); value_write_only_flush: same steps after a "
                             "write-only flush",
                       "inputs": "restored from pristine device copies before each step",
                       "parallelism": f"replicas x{world} (no cross-GPU statistics)",
                       "plan": os.environ.get("IABN_FORCE_PLAN", "auto")},
            "elements_per_s": world * sp.numel / (t_max * 1e-3),
            "value_write_only_flush": round(whole_job_gbs(layer.bytes, world, wf_ms), 1),
            "value_drained": round(whole_job_gbs(layer.bytes, world, d_ms), 1),
            "drained": {"fwd_us": round(df * 1e3, 2), "bwd_us": round(db * 1e3, 2),
                        "flush_read_us": round(drd * 1e3, 2),
                        "how": "each call followed, inside its events, by a read of 2x L2 of "
                               "other data (which writes back what the call left dirty), "
                               "minus that read's time on an L2 holding only clean lines"},
            "fwd_us": round(fwd_us, 2), "bwd_us": round(bwd_us, 2),
            "running_update": "in the forward's finalize (iabn_forward_with_running_stats)",
            "frac_of_8tbs": round(value / world / NOMINAL_HBM_GBS, 4),
            "frac_of_hbm_peak": round(value / world / hbm_peak, 4),
            "hbm_peak": {"gbs": hbm_peak,
                         "source": ("measured copy bandwidth (MEASURED_PEAKS.json)"
                                    if peak_kind == "measured" else
                                    "fallback: no MEASURED_PEAKS.json beside bench.py")},
            "roofline": {"bound": "hbm", "kernel": "backward (iabn_backward)",
                         "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(achieved / hbm_peak, 4),
                         "traffic": ncu_traffic("backward"),
                         "dram_bytes": ncu_dram("backward"),
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "algorithmic_bytes_per_launch": bwd_bytes},
            "roofline_fwd": {"bound": "hbm", "achieved": round(fwd_achieved, 1),
                             "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(fwd_achieved / hbm_peak, 4),
                             "traffic": ncu_traffic("forward"),
                             "dram_bytes": ncu_dram("forward"),
                             "algorithmic_bytes_per_launch": 2 * sp.numel * sp.itemsize},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e_max, 3),
                    "how": "public API, pinned host buffers; host-to-device copies, kernels "
                           "and device-to-host copies on three streams over two device "
                           "buffer sets (step i+1's copies overlap step i)"},
            "gpu_launches": int(launches),
            "clocks": sampler.summary(),
            "timed_wall_s": round(wall, 4),
        }
        try:   # host-side description of the launches timed above
            line["launch_plan"] = {
                d: layer.iabn.describe_plan(sp.shape, sp.layout, sp.dtype, i)
                for i, d in enumerate(("forward", "backward"))}
        except Exception as e:
            line["launch_plan"] = {"error": f"{type(e).__name__}: {e}"}
        if extra:
            line["workloads"] = extra
        if not args.no_extra and world == 1:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
