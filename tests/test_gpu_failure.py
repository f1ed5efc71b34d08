"""Failure detection on the GPU, without faulting the GPU.

Every device-side wait of the library is bounded: a wait that runs out
records a code in the workspace's error word and its kernel returns, so the
context stays usable and moe_read_error reports MOE_ERR_TIMEOUT. These tests
make such a wait run out on purpose, through the library's one-shot
failure-path hook (moe_debug_inject_fault): the grouped GEMM's producer
issues no loads, so nothing ever completes the stage its MMA warp waits on.
A second hook makes a launch fail on the host (MOE_ERR_CUDA). After either,
the next call on the same (re-initialised) workspace gives the same output,
bit for bit, as before the fault.
"""
import time

import pytest
import torch

from expert_dispatch_gemm_b200 import moe
from expert_dispatch_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"

# expert choice with a quota of 80 tokens (one 128-row block per expert): the
# single-CTA grouped GEMM
W = wl.SMALL[1]


@pytest.fixture(autouse=True)
def _disarm():
    yield
    moe.debug_inject_fault(moe.MOE_FAULT_NONE)
    torch.cuda.synchronize()


def _layer():
    assert W.dtype == "bf16" and W.mode == "ec" and W.n * W.c / W.E <= 128
    layer = moe.Layer(W, wl.make_inputs(W, DEV), DEV)
    ref = layer.forward().clone()
    st, detail = moe.moe_read_error(layer.ws)
    assert st == moe.MOE_OK, detail
    return layer, ref


def test_gemm_wait_runs_out_and_reports_timeout():
    layer, ref = _layer()
    moe.debug_inject_fault(moe.MOE_FAULT_GEMM_NO_LOADS)
    t0 = time.perf_counter()
    layer.forward()  # enqueues as usual: the host cannot know yet
    st, detail = moe.moe_read_error(layer.ws)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert st == moe.MOE_ERR_TIMEOUT, (st, hex(detail))
    assert detail & 0xF00 == 0x100  # a grouped-GEMM wait
    assert elapsed < 30.0  # the 2 s limit, not a hang
    # the context still works, the fault was one-shot, and the workspace
    # needs nothing but its error word cleared (moe_read_error cleared it)
    torch.cuda.synchronize()
    moe.lib().moe_workspace_init(moe._ptr(layer.ws), moe._stream(None))
    out = layer.forward()
    st, detail = moe.moe_read_error(layer.ws)
    assert st == moe.MOE_OK, hex(detail)
    assert torch.equal(out, ref)


def test_forced_launch_failure_returns_cuda_error():
    layer, ref = _layer()
    moe.debug_inject_fault(moe.MOE_FAULT_LAUNCH)
    with pytest.raises(moe.MoeError) as e:
        layer.forward()
    assert e.value.status == moe.MOE_ERR_CUDA
    torch.cuda.synchronize()  # the kernels enqueued before the failure finish
    moe.lib().moe_workspace_init(moe._ptr(layer.ws), moe._stream(None))
    out = layer.forward()
    st, detail = moe.moe_read_error(layer.ws)
    assert st == moe.MOE_OK, hex(detail)
    assert torch.equal(out, ref)
