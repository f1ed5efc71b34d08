"""Host-side checks of the C-ABI library (no GPU needed).

The library loads, exports every entry point include/moe.h declares, its
structs have the layout the header gives, and argument validation rejects
bad configs, missing pointers and short workspaces before any launch.
"""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

from expert_dispatch_gemm_b200 import build as build_mod
from expert_dispatch_gemm_b200 import moe
from expert_dispatch_gemm_b200 import workloads as wl
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    build_mod.build()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[^(]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported():
    syms = declared_symbols()
    assert len(syms) == 24
    assert sorted(moe.API_SYMBOLS) == syms
    L = ctypes.CDLL(moe.LIB_PATH)
    for s in syms:
        assert hasattr(L, s), s
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(m for m in re.findall(r" T (moe_\w+)", out))
    assert exported == syms  # nothing else leaks out of the library


def test_struct_layout_matches_header():
    src = r"""
    #include <stdio.h>
    #include <stddef.h>
    #include "moe.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu\n", sizeof(moe_config), offsetof(moe_config, capacity_factor),
             offsetof(moe_config, z_coef), sizeof(moe_route_out),
             offsetof(moe_route_out, ec_hist));
      return 0;
    }
    """
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        vals = [int(x) for x in subprocess.check_output([exe]).split()]
    assert vals == [ctypes.sizeof(moe.MoeConfig), moe.MoeConfig.capacity_factor.offset,
                    moe.MoeConfig.z_coef.offset, ctypes.sizeof(moe.MoeRouteOut),
                    moe.MoeRouteOut.ec_hist.offset]


def test_status_strings():
    for s in range(6):
        assert moe.status_string(s)
    assert moe.status_string(99) == "unknown status"


@pytest.mark.parametrize("w", wl.FULL + wl.SMALL, ids=lambda w: w.name)
def test_derived_sizes_match_the_pages(w):
    cfg = moe.config(w)
    assert moe.validate(cfg) == moe.MOE_OK
    sz = moe.sizes(cfg)
    spec = oracle.spec_of(w)
    if w.mode == "ec":
        assert sz.k == spec["k"]
        assert sz.slots == w.E
        assert sz.rows == w.E * ((sz.k + 127) // 128 * 128) + w.n_shared * ((w.n + 127) // 128 * 128)
    else:
        assert sz.k == w.K
        assert sz.capacity == spec["capacity"]
        assert sz.slots == w.K
    assert sz.route_ws > 0 and sz.layer_ws > sz.route_ws
    assert sz.rows % 128 == 0


def test_worked_quotas_through_the_library():
    # 4,096 tokens, 64 experts, c = 2 -> 128 per expert; 1024, 8, 2 -> 256
    for n, E, k in [(4096, 64, 128), (1024, 8, 256)]:
        cfg = moe.config(wl.EC_BF16.replace(n=n, E=E))
        assert moe.sizes(cfg).k == k
    cfg = moe.config(wl.TC_TOP2_CAP)
    assert moe.sizes(cfg).capacity == 1280


@pytest.mark.parametrize("field,value,status", [
    ("n", 0, moe.MOE_ERR_INVALID_ARG),
    ("E", 0, moe.MOE_ERR_INVALID_ARG),
    ("E", 257, moe.MOE_ERR_UNSUPPORTED),
    ("d", 100, moe.MOE_ERR_UNSUPPORTED),       # bf16 needs d % 64 == 0
    ("h", 96, moe.MOE_ERR_UNSUPPORTED),
    ("k", 0, moe.MOE_ERR_INVALID_ARG),         # token choice needs K >= 1
    ("k", 65, moe.MOE_ERR_INVALID_ARG),        # K > E
    ("mode", 7, moe.MOE_ERR_INVALID_ARG),
    ("act", 9, moe.MOE_ERR_INVALID_ARG),
    ("n_groups", 3, moe.MOE_ERR_INVALID_ARG),  # 64 % 3 != 0
    ("n_shared", 5, moe.MOE_ERR_INVALID_ARG),
])
def test_invalid_configs_rejected(field, value, status):
    base = wl.TC_DROPLESS if field != "n_groups" else wl.TC_DROPLESS.replace(
        n_groups=2, topk_groups=1, group_topn=2)
    cfg = moe.config(base)
    setattr(cfg, field, value)
    assert moe.validate(cfg) == status


def test_expert_choice_limits():
    cfg = moe.config(wl.EC_BF16.replace(n=20000))
    assert moe.validate(cfg) == moe.MOE_ERR_UNSUPPORTED  # one column must fit on chip
    cfg = moe.config(wl.EC_BF16)
    cfg.k = 5000  # more tokens per expert than tokens
    assert moe.validate(cfg) == moe.MOE_ERR_INVALID_ARG


def _fake(n):
    """Non-null, 256-aligned fake device addresses: never dereferenced,
    because validation fails before any launch."""
    return ctypes.c_void_p(0x10000000 + 256 * n)


def test_null_pointers_and_short_workspace_fail_before_launch():
    L = moe.lib()
    cfg = moe.config(wl.SMALL[2])
    sz = moe.sizes(cfg)
    out = moe.MoeRouteOut(*[0x20000000 + 4096 * i for i in range(14)])
    # X missing
    st = L.moe_route(ctypes.byref(cfg), None, _fake(1), None, None, ctypes.byref(out),
                     _fake(2), sz.route_ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # required output missing (drop is required for token choice)
    bad = moe.MoeRouteOut(*[0x20000000 + 4096 * i for i in range(14)])
    bad.drop = None
    st = L.moe_route(ctypes.byref(cfg), _fake(0), _fake(1), None, None, ctypes.byref(bad),
                     _fake(2), sz.route_ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # workspace too small / misaligned / missing
    st = L.moe_route(ctypes.byref(cfg), _fake(0), _fake(1), None, None, ctypes.byref(out),
                     _fake(2), sz.route_ws - 1, None)
    assert st == moe.MOE_ERR_WORKSPACE
    st = L.moe_route(ctypes.byref(cfg), _fake(0), _fake(1), None, None, ctypes.byref(out),
                     ctypes.c_void_p(0x10000010), sz.route_ws, None)
    assert st == moe.MOE_ERR_WORKSPACE
    st = L.moe_layer_forward(ctypes.byref(cfg), _fake(0), _fake(1), None, None, _fake(3),
                             _fake(4), _fake(5), None, None, None, _fake(6), ctypes.byref(out),
                             _fake(2), sz.route_ws, None)
    assert st == moe.MOE_ERR_WORKSPACE  # the layer needs the larger workspace
    # SwiGLU without W3
    st = L.moe_expert_ffn(ctypes.byref(cfg), _fake(0), _fake(1), _fake(2), None, _fake(3), None,
                          _fake(5), None, None, None, _fake(6), _fake(7), _fake(8), 4096, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # bias update is a token-choice operation
    ec = moe.config(wl.EC_FP32)
    st = L.moe_bias_update(ctypes.byref(ec), _fake(0), ctypes.c_float(0.001), _fake(1), None)
    assert st == moe.MOE_ERR_INVALID_ARG
    # host buffers: the host pointers are checked, then everything moe_layer_forward checks
    lw = sz.layer_ws
    st = L.moe_layer_forward_host(ctypes.byref(cfg), None, _fake(1), None, None, _fake(3),
                                  _fake(4), _fake(5), None, None, None, _fake(6), _fake(7),
                                  _fake(8), ctypes.byref(out), _fake(2), lw, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    st = L.moe_layer_forward_host(ctypes.byref(cfg), _fake(0), _fake(1), None, None, _fake(3),
                                  _fake(4), _fake(5), None, None, None, _fake(6), None,
                                  _fake(8), ctypes.byref(out), _fake(2), lw, None)
    assert st == moe.MOE_ERR_INVALID_ARG  # no device copy of X
    st = L.moe_layer_forward_host(ctypes.byref(cfg), _fake(0), _fake(1), None, None, _fake(3),
                                  _fake(4), _fake(5), None, None, None, _fake(6), _fake(7),
                                  _fake(8), ctypes.byref(out), _fake(2), lw - 1, None)
    assert st == moe.MOE_ERR_WORKSPACE
    if not torch.cuda.is_available():
        # no workspace: the no-alloc routing scratch's word, after a stream
        # synchronise that cannot succeed without a device
        assert L.moe_read_error(None, None, None) == moe.MOE_ERR_CUDA


def test_binding_refuses_to_run_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(moe, "_LIB", None)
    with pytest.raises(RuntimeError, match="missing"):
        moe.lib()


def test_launch_counts():
    """Kernels per call: the router (plus the split-k reduce that batches too
    small to fill the SMs take), the selection kernels, one gather, two GEMMs,
    one combine."""
    ec = moe.launch_counts(moe.config(wl.EC_BF16))
    assert ec == {"route": 3, "dispatch": 1, "ffn": 2, "combine": 1}
    tc = moe.launch_counts(moe.config(wl.TC_DROPLESS))
    assert tc == {"route": 4, "dispatch": 1, "ffn": 2, "combine": 1}
    decode = moe.launch_counts(moe.config(wl.DECODE))
    assert decode["route"] == 5
    assert moe.launch_counts(moe.config(wl.TC_SIGMOID_GROUPED))["ffn"] == 2


def test_fault_hook_arguments():
    """The failure-path hook takes the documented faults only, and
    MOE_FAULT_NONE disarms it (nothing is launched here)."""
    L = moe.lib()
    assert L.moe_debug_inject_fault(7) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_debug_inject_fault(-1) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_debug_inject_fault(moe.MOE_FAULT_LAUNCH) == moe.MOE_OK
    assert L.moe_debug_inject_fault(moe.MOE_FAULT_NONE) == moe.MOE_OK


def test_train_launch_counts():
    """The training forward enqueues the layer's kernels plus, for bf16, the
    clear of the dispatched rows' padding; the training backward one fewer
    than moe_layer_backward for bf16 (no recompute of the up projection)."""
    for w in (wl.EC_FP32, wl.EC_BF16, wl.TC_DROPLESS, wl.TC_SIGMOID_GROUPED):
        cfg = moe.config(w)
        f, b = moe.train_launch_counts(cfg)
        bf16 = int(w.dtype == "bf16")
        assert f == sum(moe.launch_counts(cfg).values()) + bf16, w.name
        assert b == _bwd_size(cfg)[2] - bf16, w.name


def _bwd_size(cfg):
    nbytes = ctypes.c_size_t()
    launches = ctypes.c_int()
    st = moe.lib().moe_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(nbytes),
                                               ctypes.byref(launches))
    return st, nbytes.value, launches.value


def test_backward_workspace_and_launches():
    """The backward enqueues the padding clear, the combine backward, five
    grouped GEMMs, the W_g transpose, the router's input gradient and its
    weight gradient (plus the ordered reduce of the weight gradient's token
    slices when there is more than one), for bf16 and fp32 layers alike."""
    for w in (wl.EC_FP32, wl.EC_BF16, wl.TC_TOP2_CAP, wl.TC_DROPLESS, wl.TC_SIGMOID_GROUPED,
              wl.DECODE):
        st, nbytes, launches = _bwd_size(moe.config(w))
        assert st == moe.MOE_OK, w.name
        sw = w.act == "swiglu"
        sz = moe.sizes(moe.config(w))
        elt = 4 if w.dtype == "f32" else 2
        # at least dY, U, (V), H, dU(,dV) and dX_perm over the dispatched rows
        assert nbytes >= sz.rows * elt * (w.d + w.h * (4 if sw else 2)), w.name
        assert launches in (10, 11), w.name


def test_backward_rejects_bad_arguments_before_launching():
    """Host-side validation: null required pointers fail without touching
    the (null) device pointers, for bf16 and fp32 configs."""
    cfg = moe.config(wl.TC_DROPLESS.replace(n=256, d=128, E=8, h=128))
    L = moe.lib()
    route = moe.MoeRouteOut()
    st = L.moe_layer_backward(ctypes.byref(cfg), *([None] * 8), ctypes.byref(route), None, 0,
                              *([None] * 10), None, 0, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    cfg32 = moe.config(wl.EC_FP32)
    st = L.moe_layer_backward(ctypes.byref(cfg32), *([None] * 8), ctypes.byref(route), None, 0,
                              *([None] * 10), None, 0, None)
    assert st == moe.MOE_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="hands fake device pointers to the library: host-only check")
def test_backward_host_validation_without_device_memory():
    """The backward entry points check workspaces and alignment on the host
    before any launch: fake (never dereferenced) 256-byte-aligned pointers
    with too-small workspaces, and a misaligned gradient pointer, are
    refused with the documented status."""
    cfg = moe.config(wl.TC_DROPLESS.replace(n=256, d=128, E=8, h=128))
    L = moe.lib()
    route = moe.MoeRouteOut(*[0x10000 + 0x1000 * i for i in range(14)])
    fake = [ctypes.c_void_p(0x100000 + 0x10000 * i) for i in range(24)]
    st, need, _ = _bwd_size(cfg)
    assert st == moe.MOE_OK and need > 0
    args = lambda fwd_bytes, ws_bytes, dX: (
        ctypes.byref(cfg), *fake[:8], ctypes.byref(route), fake[8], fwd_bytes, fake[9], dX,
        *fake[11:19], fake[19], ws_bytes, None)
    # forward workspace too small
    st = L.moe_layer_backward(*args(16, need, fake[10]))
    assert st == moe.MOE_ERR_WORKSPACE
    fwd_need = moe.sizes(cfg).layer_ws
    # backward workspace too small
    st = L.moe_layer_backward(*args(fwd_need, need - 1, fake[10]))
    assert st == moe.MOE_ERR_WORKSPACE
    st = L.moe_layer_backward_train(*args(fwd_need, need - 1, fake[10]))
    assert st == moe.MOE_ERR_WORKSPACE
    # dX not 16-byte aligned
    st = L.moe_layer_backward(*args(fwd_need, need, ctypes.c_void_p(0x200008)))
    assert st == moe.MOE_ERR_INVALID_ARG
    # the training forward checks its backward workspace too
    st = L.moe_layer_forward_train(ctypes.byref(cfg), *fake[:11], ctypes.byref(route), fake[11],
                                   fwd_need, fake[12], need - 1, None)
    assert st == moe.MOE_ERR_WORKSPACE
