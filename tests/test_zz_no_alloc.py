"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Callers such as an application whose device memory budget is fixed at
start-up, or a plugin inside a framework that owns every device allocation,
cannot pass moe_route a workspace. moe_route_noalloc runs the same routing
with its scratch in a library-owned static device array. These tests call it
through the C ABI and check that it returns what moe_route (with a
caller-provided workspace) returns, on two calls in a row, and that a config
needing more scratch than the array holds is refused.

This file is collected last on purpose, so a run that stops at the first
failure has run every other test before it; it also passes when run alone.
"""
import ctypes

import numpy as np
import pytest
import torch

from expert_dispatch_gemm_b200 import moe
from expert_dispatch_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [wl.SMALL[1], wl.SMALL[2], wl.SMALL[4], wl.EC_BF16, wl.TC_DROPLESS]


def _compare(ref: moe.RouteBuffers, got: moe.RouteBuffers):
    for name in ("idx", "load", "counts", "offsets", "tok_row", "drop", "ec_hist"):
        a, b = getattr(ref, name), getattr(got, name)
        if a is None:
            continue
        assert torch.equal(a, b), name
    used = int(ref.offsets[-1])
    assert torch.equal(ref.row_token[:used], got.row_token[:used])
    for name in ("gate", "tok_gate", "scores", "logits", "lse", "aux"):
        a, b = getattr(ref, name), getattr(got, name)
        np.testing.assert_allclose(b.cpu().numpy(), a.cpu().numpy(), rtol=1e-6, atol=0,
                                   err_msg=name)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_route_matches_workspace_route(w):
    sz = moe.sizes(moe.config(w))
    assert sz.route_ws <= moe.MOE_ROUTE_NOALLOC_SCRATCH_BYTES
    inp = wl.make_inputs(w, DEV, experts=False)
    cfg = moe.config(w)
    ref = moe.RouteBuffers(cfg, DEV)
    ws = moe.workspace(cfg, DEV, layer=False)
    moe.moe_route(cfg, inp["X"], inp["Wg"], inp["logit_bias"], inp["sel_bias"], ref, ws)
    L = moe.lib()
    for call in range(2):
        got = moe.RouteBuffers(cfg, DEV)
        st = L.moe_route_noalloc(ctypes.byref(cfg), ctypes.c_void_p(inp["X"].data_ptr()),
                                 ctypes.c_void_p(inp["Wg"].data_ptr()),
                                 None if inp["logit_bias"] is None else
                                 ctypes.c_void_p(inp["logit_bias"].data_ptr()),
                                 None if inp["sel_bias"] is None else
                                 ctypes.c_void_p(inp["sel_bias"].data_ptr()),
                                 ctypes.byref(got.c),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == moe.MOE_OK, moe.status_string(st)
        torch.cuda.synchronize()
        _compare(ref, got)
        # the routing left the scratch array's error word clear; a NULL
        # workspace reads (and clears) that word
        st, detail = moe.moe_read_error(None)
        assert st == moe.MOE_OK and detail == 0


def test_noalloc_refuses_configs_beyond_its_scratch():
    # 16384 tokens x 256 experts of expert choice need more than 4 MiB of
    # routing scratch (the dense [n, E] slot map alone is 32 MiB)
    w = wl.EC_BF16.replace(n=16384, E=256, d=128, h=128)
    cfg = moe.config(w)
    assert moe.sizes(cfg).route_ws > moe.MOE_ROUTE_NOALLOC_SCRATCH_BYTES
    rb = moe.RouteBuffers(cfg, DEV)
    X = torch.zeros((w.n, w.d), dtype=torch.bfloat16, device=DEV)
    Wg = torch.zeros((w.d, w.E), dtype=torch.float32, device=DEV)
    L = moe.lib()
    st = L.moe_route_noalloc(ctypes.byref(cfg), ctypes.c_void_p(X.data_ptr()),
                             ctypes.c_void_p(Wg.data_ptr()), None, None, ctypes.byref(rb.c),
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.MOE_ERR_WORKSPACE
