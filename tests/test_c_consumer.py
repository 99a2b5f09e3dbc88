"""include/iabn.h consumed from plain C (and C++): tests/c/abi_consumer.c is
compiled with warnings as errors, linked against libiabn.so and run.  Its
results must match what the Python binding gets from the same library, so
the header's types (iabn_desc, iabn_plan_info, the enums) have the layout the
library uses.  Only host-side entry points are called."""
import os
import shutil
import subprocess

import pytest

import place_batchnorm_activation_b200 as iabn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "abi_consumer.c")


def _build_and_run(tmp_path, compiler, lang_flags):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    exe = tmp_path / f"consumer_{compiler.replace('+', 'p')}"
    libdir = os.path.dirname(iabn.LIB_PATH)
    cmd = [compiler, *lang_flags, "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), SRC, "-o", str(exe),
           "-L", libdir, "-l:libiabn.so", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return dict(line.split(" ", 1) for line in out.strip().splitlines())


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-std=c11"]),
                                            ("g++", ["-x", "c++", "-std=c++17"])])
def test_c_consumer_matches_the_binding(tmp_path, compiler, flags, monkeypatch):
    for k in ("IABN_FORCE_PLAN", "IABN_TILE_KB_FWD", "IABN_TILE_KB_BWD", "IABN_RING_FWD",
              "IABN_RING_BWD", "IABN_TMEM_STASH", "IABN_STASH_CP", "IABN_NCHW_SMEM_COEF"):
        monkeypatch.delenv(k, raising=False)
    iabn.lib()   # the library must exist (built by the package's build step)
    got = _build_and_run(tmp_path, compiler, flags)
    assert int(got["sizeof_desc"]) == 40
    assert int(got["sizeof_plan_info"]) == 4 * len(iabn.IabnPlanInfo._fields_)
    assert int(got["ws_trunk"]) == iabn.workspace_size((64, 256, 56, 56), iabn.IABN_NHWC,
                                                       iabn.IABN_BF16)
    assert int(got["ws_many"]) == iabn.workspace_size((128, 2048, 7, 7), iabn.IABN_NCHW,
                                                      iabn.IABN_F16)
    assert int(got["ws_bad"]) == 0
    for tag, shape, layout, dtype, direction in (
            ("trunk_fwd", (64, 256, 56, 56), iabn.IABN_NHWC, iabn.IABN_BF16, 0),
            ("trunk_bwd", (64, 256, 56, 56), iabn.IABN_NHWC, iabn.IABN_BF16, 1),
            ("many_fwd", (128, 2048, 7, 7), iabn.IABN_NCHW, iabn.IABN_F16, 0),
            ("trunk_std_bwd", (64, 256, 56, 56), iabn.IABN_NHWC, iabn.IABN_BF16,
             iabn.IABN_CALL_BACKWARD_STANDARD),
            ("trunk_ckpt_fwd", (64, 256, 56, 56), iabn.IABN_NHWC, iabn.IABN_BF16,
             iabn.IABN_CALL_FORWARD_CHECKPOINT)):
        want = iabn.describe_plan(shape, layout, dtype, direction, sm_count=148,
                                  smem_optin=232448)
        want["plan"] = {"twophase": 0, "resident": 1}[want["plan"]]
        for k, v in want.items():
            assert int(got[f"{tag}.{k}"]) == v, (tag, k)
    for k in ("describe_fwd_status", "describe_bwd_status", "describe_many_status",
              "describe_std_bwd_status", "describe_ckpt_fwd_status"):
        assert int(got[k]) == iabn.IABN_OK
    assert int(got["describe_bad_call"]) == iabn.IABN_ERR_INVALID_ARG
    for k in ("forward_standard_null_z", "backward_standard_null_mean",
              "forward_checkpoint_bad_eps", "backward_checkpoint_bad_desc",
              "recompute_null_xhat", "sync_forward_stats_null_stats",
              "forward_running_null_rmean",
              "sync_forward_apply_bad_world", "sync_backward_stats_bad_act",
              "sync_backward_apply_null_gathered"):
        assert int(got[k]) == iabn.IABN_ERR_INVALID_ARG, k
    assert int(got["forward_null_x"]) == iabn.IABN_ERR_INVALID_ARG
    assert int(got["backward_bad_desc"]) == iabn.IABN_ERR_INVALID_ARG
    assert int(got["inference_bad_act"]) == iabn.IABN_ERR_INVALID_ARG
    assert int(got["running_bad_count"]) == iabn.IABN_ERR_INVALID_ARG
    assert int(got["status_null_ws"]) == iabn.IABN_ERR_INVALID_ARG
    assert int(got["launches"]) == 0
