"""The host-side launch planner, through iabn_describe_plan, without a GPU.

The plan decides the launch shape of every call -- the in-place layer's
forward and backward, the standard layer's and the checkpointing layer's:
grid, shared memory, tile sizes, the Tensor Memory stash.  A planning error would reach the device as
an oversized launch or an out-of-range slot, so its invariants are checked
here on the CPU over a sweep of shapes, at the B200's limits (148 SMs,
232448 bytes of opt-in shared memory per block) and at smaller ones.  The
qualification rule of the resident plan (documented in iabn_resident.cu) is
checked against an independent restatement, and the five benchmark
workloads must all take the resident plan.
"""
import itertools
import math

import pytest
import torch

import place_batchnorm_activation_b200 as iabn
import workloads as wl

B200 = dict(sm_count=148, smem_optin=232448)
KNOBS = ("IABN_FORCE_PLAN", "IABN_TILE_KB_FWD", "IABN_TILE_KB_BWD", "IABN_RING_FWD",
         "IABN_RING_BWD", "IABN_TMEM_STASH", "IABN_STASH_CP", "IABN_NCHW_SMEM_COEF",
         "IABN_STASH_FIRST")


@pytest.fixture(autouse=True)
def default_knobs(monkeypatch):
    for k in KNOBS:
        monkeypatch.delenv(k, raising=False)


def esize(dtype):
    return 4 if dtype == wl.F32 else 2


CALLS = range(6)          # IABN_CALL_*: layer = call // 2, direction = call % 2


def qualifies(shape, layout, dtype, call=0):
    """The resident plan's shape rule, restated: NHWC rows of C channels are a
    multiple of 16 bytes and at most 16 KiB (at most 4 KiB, one 16-byte
    column per consumer thread, for the standard and the checkpointing
    layers); NCHW units of g whole planes (g = 16 / gcd(16, H*W*s)) start on
    16-byte boundaries, N*C is a multiple of g and a unit is at most 32 KiB."""
    n, c, h, w = shape
    s = esize(dtype)
    if layout == wl.NHWC:
        return (c * s) % 16 == 0 and c * s <= (16384 if call < 2 else 4096)
    g = 16 // math.gcd(h * w * s, 16)
    return (n * c) % g == 0 and g * h * w * s <= 32768


def check_resident(info, shape, layout, dtype, call, sm_count, smem_optin):
    n, c, h, w = shape
    s = esize(dtype)
    nt = 1 if call % 2 == 0 else 2           # tensors streamed: x; or z (x, xhat) and dz
    # 8 consumer warps, a producer and a copier; the NCHW forward (no Tensor
    # Memory stash): 15 consumer warps and a producer
    threads = 512 if layout == wl.NCHW and call % 2 == 0 else 320
    assert info["launches"] == 1 and info["threads"] == threads
    units = n * h * w if layout == wl.NHWC else n * c // info["planes_per_unit"]
    assert 1 <= info["grid"] <= min(sm_count, 256, units)
    assert 0 < info["smem_bytes"] <= smem_optin - 1024
    assert 2 <= info["ring"] <= info["slots"] <= 32
    tb = info["tile_bytes"]
    assert tb > 0 and tb % 16 == 0
    half = (tb + 127) // 128 * 128
    assert 1024 + info["slots"] * half * nt <= info["smem_bytes"]
    if layout == wl.NHWC:
        vc, cpt, rp = info["vectors_per_row"], info["cols_per_thread"], info["row_phases"]
        assert vc * 16 == c * s
        assert cpt in (1, 2, 4) and vc <= 256 * cpt and (cpt == 1 or vc > 256 * cpt // 2)
        assert cpt == 1 or call < 2
        assert rp == (256 // vc if cpt == 1 else 1)
        assert tb % (c * s) == 0 and (tb // (c * s)) % rp == 0
        assert info["planes_per_unit"] == 0
        # Tensor Memory: 1 KiB (64 16-byte vectors) per consumer thread
        assert info["stash_rows"] * cpt * nt <= 64
        if info["stash_copy_engine"]:
            assert info["stash_rows"] > 0 and rp * vc == 256 * cpt
    else:
        g = info["planes_per_unit"]
        assert g == 16 // math.gcd(h * w * s, 16)
        assert tb % (g * h * w * s) == 0
        assert info["stash_rows"] == 0 and info["stash_copy_engine"] == 0
        assert info["vectors_per_row"] == info["cols_per_thread"] == info["row_phases"] == 0


def check_twophase(info):
    assert info["launches"] == 3
    assert all(v == 0 for k, v in info.items() if k not in ("plan", "launches"))


CS = [1, 2, 3, 4, 6, 8, 12, 16, 24, 40, 64, 100, 256, 264, 512, 1000, 2048, 4096, 4104,
      8192, 8200, 16384]
HWS = [(1, 1), (1, 2), (3, 3), (5, 7), (7, 7), (14, 14), (56, 56), (1000, 37)]
NS = [1, 2, 3, 8, 64]


def sweep():
    for c, (h, w), n, layout, dtype in itertools.product(CS, HWS, NS, (wl.NCHW, wl.NHWC),
                                                         (wl.F32, wl.BF16, wl.F16)):
        if n * h * w >= 2 and n * c * h * w <= 1 << 31:
            yield (n, c, h, w), layout, dtype


@pytest.mark.parametrize("limits,tiles", [(B200, None),
                                           (dict(sm_count=132, smem_optin=232448), None),
                                           (dict(sm_count=8, smem_optin=101376), (16, 8))],
                         ids=["b200", "132sm", "8sm_99k_small_tiles"])
def test_plan_invariants_over_shapes(limits, tiles, monkeypatch):
    if tiles:
        monkeypatch.setenv("IABN_TILE_KB_FWD", str(tiles[0]))
        monkeypatch.setenv("IABN_TILE_KB_BWD", str(tiles[1]))
    seen = {"resident": 0, "twophase": 0}
    for shape, layout, dtype in sweep():
        for call in CALLS:
            info = iabn.describe_plan(shape, layout, dtype, call, **limits)
            seen[info["plan"]] += 1
            if info["plan"] == "resident":
                assert qualifies(shape, layout, dtype, call), (shape, layout, dtype, call)
                check_resident(info, shape, layout, dtype, call, **limits)
            else:
                check_twophase(info)
                if limits is B200:
                    # at the B200's limits every qualifying shape fits
                    assert not qualifies(shape, layout, dtype, call), (shape, layout, dtype, call)
    assert seen["resident"] > 0 and seen["twophase"] > 0


def test_both_calls_of_a_layer_agree_on_the_plan():
    for shape, layout, dtype in sweep():
        for layer in range(3):
            f = iabn.describe_plan(shape, layout, dtype, 2 * layer, **B200)
            b = iabn.describe_plan(shape, layout, dtype, 2 * layer + 1, **B200)
            assert f["plan"] == b["plan"] and f["grid"] == b["grid"]


def test_benchmark_workloads_take_the_resident_plan():
    specs = [wl.spec(i) for i in range(4)] + [wl.spec(4, l) for l in range(16)]
    for sp in specs:
        # every call of the in-place layer; the standard and the checkpointing
        # layers wherever a row is at most 4 KiB (all but the two widest
        # layers of the sweep)
        calls = CALLS if sp.layout == wl.NCHW or sp.c * sp.itemsize <= 4096 else (0, 1)
        for call in calls:
            info = iabn.describe_plan(sp.shape, sp.layout, sp.dtype, call, **B200)
            assert info["plan"] == "resident", (sp.name, call)
            if sp.n * sp.h * sp.w >= 148 * 8 or sp.layout == wl.NCHW and sp.n * sp.c >= 148 * 8:
                assert info["grid"] == 148
    # the ResNet-trunk layer keeps rows in Tensor Memory, filled by the copy engine
    trunk = wl.spec(1)
    for direction, rows in ((0, 64), (1, 32)):
        info = iabn.describe_plan(trunk.shape, trunk.layout, trunk.dtype, direction, **B200)
        assert (info["stash_rows"], info["stash_copy_engine"], info["row_phases"]) == (rows, 1, 8)


def test_nchw_forward_tiles_hold_whole_rounds_of_planes():
    """NCHW forward tiles hold a whole number of the planes its 480 consumer
    threads take at once (480 / lanes per plane) where the tile size target
    allows: the many-channel layer (7x7 fp16 planes, 8 planes per 16-byte
    aligned unit of 784 bytes) forward 60 units (480 planes, one lane each);
    the backward keeps 256 consumer threads and the plain target, 31 units."""
    mc = wl.spec(3)
    fwd = iabn.describe_plan(mc.shape, mc.layout, mc.dtype, 0, **B200)
    bwd = iabn.describe_plan(mc.shape, mc.layout, mc.dtype, 1, **B200)
    assert fwd["plan"] == bwd["plan"] == "resident"
    assert fwd["planes_per_unit"] == bwd["planes_per_unit"] == 8
    assert fwd["tile_bytes"] == 60 * 784 and bwd["tile_bytes"] == 31 * 784
    assert (fwd["threads"], bwd["threads"]) == (512, 320)


def test_small_shared_memory_declines_the_resident_plan():
    shape = (64, 256, 56, 56)
    info = iabn.describe_plan(shape, wl.NHWC, wl.BF16, 0, sm_count=148, smem_optin=65536)
    assert info["plan"] == "twophase"
    one = iabn.describe_plan(shape, wl.NHWC, wl.BF16, 0, sm_count=1, smem_optin=232448)
    assert one["plan"] == "resident" and one["grid"] == 1


def test_environment_knobs(monkeypatch):
    shape = (64, 256, 56, 56)
    monkeypatch.setenv("IABN_FORCE_PLAN", "twophase")
    check_twophase(iabn.describe_plan(shape, wl.NHWC, wl.BF16, 0, **B200))
    monkeypatch.delenv("IABN_FORCE_PLAN")
    monkeypatch.setenv("IABN_TILE_KB_FWD", "32")
    info = iabn.describe_plan(shape, wl.NHWC, wl.BF16, 0, **B200)
    assert info["plan"] == "resident" and info["tile_bytes"] == 32768
    check_resident(info, shape, wl.NHWC, wl.BF16, 0, **B200)
    monkeypatch.setenv("IABN_TMEM_STASH", "0")
    info = iabn.describe_plan(shape, wl.NHWC, wl.BF16, 0, **B200)
    assert info["stash_rows"] == 0 and info["stash_copy_engine"] == 0
    assert info["slots"] > info["ring"]        # without the stash, extra slots keep tiles


def test_describe_rejects_bad_arguments():
    d = iabn.make_desc((2, 8, 4, 4), wl.NHWC, wl.BF16)
    info = iabn.IabnPlanInfo()
    assert iabn.iabn_describe_plan(d, 6, 148, 232448, info) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_describe_plan(d, -1, 148, 232448, info) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_describe_plan(d, 0, 148, 0, info) == iabn.IABN_ERR_INVALID_ARG
    assert iabn.iabn_describe_plan(d, 0, -1, 232448, info) == iabn.IABN_ERR_INVALID_ARG
    bad = iabn.make_desc((1, 8, 1, 1), wl.NHWC, wl.BF16)          # M = 1
    assert iabn.iabn_describe_plan(bad, 0, 148, 232448, info) == iabn.IABN_ERR_INVALID_ARG
    huge = iabn.make_desc((1, 1 << 25, 1, 2), wl.NHWC, wl.BF16)    # beyond the grid limit
    assert iabn.iabn_describe_plan(huge, 0, 148, 232448, info) == iabn.IABN_ERR_UNSUPPORTED
    # channels: at most 65535 blocks of 256 on the grid's y dimension
    edge = iabn.make_desc((1, 65535 * 256, 1, 2), wl.NHWC, wl.BF16)
    assert iabn.iabn_describe_plan(edge, 0, 148, 232448, info) == iabn.IABN_OK
    assert info.plan == iabn.IABN_PLAN_TWOPHASE
    over = iabn.make_desc((1, 65535 * 256 + 8, 1, 2), wl.NHWC, wl.BF16)
    assert iabn.iabn_describe_plan(over, 0, 148, 232448, info) == iabn.IABN_ERR_UNSUPPORTED
    assert iabn.iabn_workspace_size(over) == 0
    lib = iabn.lib()
    assert lib.iabn_describe_plan(iabn.ctypes.byref(d), 0, 148, 232448, None) == \
        iabn.IABN_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_device_query_without_a_gpu_reports_cuda_error():
    d = iabn.make_desc((2, 8, 4, 4), wl.NHWC, wl.BF16)
    assert iabn.iabn_describe_plan(d, 0, 0, 0, iabn.IabnPlanInfo()) == iabn.IABN_ERR_CUDA


@pytest.mark.gpu
@pytest.mark.parametrize("shape,layout,dtype", [((8, 256, 14, 14), wl.NHWC, wl.BF16),
                                                ((3, 100, 5, 5), wl.NHWC, wl.BF16),
                                                ((16, 64, 7, 7), wl.NCHW, wl.F16)])
def test_described_plan_is_the_one_that_runs(shape, layout, dtype):
    """On the device: the current-device query matches the device's own
    limits, and a forward and a backward launch the described number of
    kernels."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from gpu_util import GpuLayer
    props = torch.cuda.get_device_properties(0)
    here = [iabn.describe_plan(shape, layout, dtype, d) for d in (0, 1)]
    explicit = [iabn.describe_plan(shape, layout, dtype, d, sm_count=props.multi_processor_count,
                                   smem_optin=props.shared_memory_per_block_optin)
                for d in (0, 1)]
    assert here == explicit
    n, c, h, w = shape
    sp = wl.LayerSpec("plan", n, c, h, w, layout, dtype, wl.LEAKY_RELU, 0.01, seed=31 + c)
    L = GpuLayer(wl.draw(sp))
    torch.cuda.synchronize()
    k0 = iabn.iabn_kernel_launches()
    L.forward()
    k1 = iabn.iabn_kernel_launches()
    L.backward()
    k2 = iabn.iabn_kernel_launches()
    torch.cuda.synchronize()
    assert (k1 - k0, k2 - k1) == (here[0]["launches"], here[1]["launches"])
    assert L.status() == 0
