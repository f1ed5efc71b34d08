"""The checked build of the library (libmoe_checked.so, compiled with
-DMOE_DEBUG_CHECKS): every kernel that reads an index from the routing
outputs (row_token, tok_row, offsets, counts, idx) reports an out-of-range
value as kErrBadIndex | site in the error word, besides skipping it as every
build does. It stands in for a memory checker, which is not run here.

test_checked_build_parity_suite runs the small parity suite, the edge cases
and the backward's small layers in a subprocess that loads the checked build
(MOE_LIBRARY=checked): every one of those tests asserts a clear error word.
The tests below it run only inside that subprocess: they plant an
out-of-range slot entry, which every build skips, and check that the
checked build names it.
"""
import os
import subprocess
import sys

import pytest
import torch

from expert_dispatch_gemm_b200 import moe
from expert_dispatch_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.environ.get("MOE_LIBRARY") == "checked"


@pytest.mark.skipif(CHECKED, reason="the driver of the checked run")
def test_checked_build_parity_suite():
    assert os.path.exists(moe.CHECKED_LIB_PATH), "build libmoe_checked.so first"
    env = dict(os.environ, MOE_LIBRARY="checked")
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_gpu_checked.py"),
           os.path.join(ROOT, "tests", "test_gpu_parity.py"),
           os.path.join(ROOT, "tests", "test_gpu_backward.py"),
           "-k", "checked_build_reports or checked_library_is_loaded or layer_small or "
                 "edge_cases or dispatch_exact_copy or backward_small"]
    r = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=1500)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail


@pytest.mark.skipif(not CHECKED, reason="runs under the checked build (MOE_LIBRARY=checked)")
def test_checked_library_is_loaded():
    moe.lib()
    assert moe.LIB_PATH == moe.CHECKED_LIB_PATH
    maps = open("/proc/self/maps").read()
    assert "libmoe_checked.so" in maps and "/libmoe.so" not in maps


@pytest.mark.skipif(not CHECKED, reason="runs under the checked build (MOE_LIBRARY=checked)")
def test_checked_build_reports_out_of_range_slot_entries():
    # top-8 of 64 with a shared expert: the staged gather (it reads tok_row)
    # and Y rows past the routed bound (the shared expert's), so the planted
    # entry stays inside every buffer even if a check were missing
    w = wl.SMALL[4]
    inp = wl.make_inputs(w, DEV)
    cfg = moe.config(w)
    sz = moe.sizes(cfg)
    rb = moe.RouteBuffers(cfg, DEV)
    ws = moe.workspace(cfg, DEV, layer=False)
    dt = w.torch_dtype
    X_perm = torch.zeros((sz.rows, w.d), dtype=dt, device=DEV)
    H = torch.empty((sz.rows, w.h), dtype=dt, device=DEV)
    Y = torch.empty((sz.rows, w.d), dtype=dt, device=DEV)
    out = torch.empty((w.n, w.d), dtype=dt, device=DEV)
    moe.moe_route(cfg, inp["X"], inp["Wg"], None, inp["sel_bias"], rb, ws)
    moe.moe_dispatch(cfg, inp["X"], rb, X_perm)
    moe.moe_expert_ffn(cfg, inp["X"], X_perm, rb.offsets, inp["W1"], inp["W3"], inp["W2"],
                       inp["sW1"], inp["sW3"], inp["sW2"], H, Y, ws, counts=rb.counts)
    moe.moe_combine(cfg, Y, rb, out)
    assert moe.moe_read_error(ws) == (moe.MOE_OK, 0)
    assert moe.moe_read_error(None) == (moe.MOE_OK, 0)  # standalone dispatch / combine word
    routed = int(rb.offsets[-1])
    assert sz.shared_row_base >= routed and sz.rows > sz.shared_row_base
    t = 7
    saved = rb.tok_row[t, 0].item()
    rb.tok_row[t, 0] = sz.shared_row_base + 3  # past the routed rows, inside X_perm and Y
    moe.moe_dispatch(cfg, inp["X"], rb, X_perm)
    st, detail = moe.moe_read_error(None)
    assert st == moe.MOE_ERR_CUDA and detail == 0x201, hex(detail)  # gather, tok_row
    moe.moe_combine(cfg, Y, rb, out)
    st, detail = moe.moe_read_error(None)
    assert st == moe.MOE_ERR_CUDA and detail == 0x204, hex(detail)  # combine, tok_row
    rb.tok_row[t, 0] = saved
    moe.moe_combine(cfg, Y, rb, out)
    assert moe.moe_read_error(None) == (moe.MOE_OK, 0)
