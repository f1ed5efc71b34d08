"""Thin Python binding of libmoe (include/moe.h) over torch device tensors.

Argument marshalling only: every step of the layer runs in libmoe's CUDA
kernels. torch allocates the device memory and supplies the stream. The
library must have been built (``python -m expert_dispatch_gemm_b200.build``);
if ``libmoe.so`` is missing every call raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from .workloads import Workload

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")
# the checked build (every out-of-range routing index reported in the error
# word); MOE_LIBRARY=checked in the environment loads it instead, and
# MOE_LIBRARY=<path of a .so> loads another build of the same sources
CHECKED_LIB_PATH = os.path.join(_PKG, "libmoe_checked.so")
if os.environ.get("MOE_LIBRARY") == "checked":
    LIB_PATH = CHECKED_LIB_PATH
elif os.environ.get("MOE_LIBRARY"):
    LIB_PATH = os.path.abspath(os.environ["MOE_LIBRARY"])

# enums and limits of include/moe.h
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, \
    MOE_ERR_TIMEOUT = range(6)
MOE_EXPERT_CHOICE, MOE_TOKEN_CHOICE = 0, 1
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID, MOE_SCORE_SQRTSOFTPLUS = 0, 1, 2
MOE_W_RAW, MOE_W_NORMALIZED = 0, 1
MOE_ACT_RELU, MOE_ACT_GELU, MOE_ACT_SWIGLU = 0, 1, 2
MOE_F32, MOE_BF16 = 0, 1
MOE_ROW_ALIGN = 128
MOE_AUX_LEN = 8
AUX_NAMES = ["lb_loss", "z_loss", "maxvio", "dropped_assignments", "tokens_some_dropped",
             "tokens_all_dropped", "tokens_no_expert", "reserved"]

# every entry point include/moe.h declares
API_SYMBOLS = ["moe_status_string", "moe_validate", "moe_sizes", "moe_workspace_size",
               "moe_route", "moe_route_from_scores", "moe_dispatch", "moe_expert_ffn",
               "moe_combine", "moe_layer_forward", "moe_bias_update", "moe_workspace_init",
               "moe_read_error", "moe_route_noalloc", "moe_expert_ffn_gathered",
               "moe_launch_counts", "moe_backward_workspace_size", "moe_layer_backward",
               "moe_expert_ffn_combined", "moe_layer_forward_train", "moe_layer_backward_train",
               "moe_layer_forward_host", "moe_train_launch_counts", "moe_debug_inject_fault"]
MOE_FAULT_NONE, MOE_FAULT_GEMM_NO_LOADS, MOE_FAULT_LAUNCH = 0, 1, 2
MOE_ROUTE_NOALLOC_SCRATCH_BYTES = 4 << 20


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class MoeConfig(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("d", ctypes.c_int), ("E", ctypes.c_int),
                ("h", ctypes.c_int), ("mode", ctypes.c_int), ("score", ctypes.c_int),
                ("k", ctypes.c_int), ("capacity_factor", ctypes.c_float),
                ("capacity", ctypes.c_int), ("n_groups", ctypes.c_int),
                ("topk_groups", ctypes.c_int), ("group_topn", ctypes.c_int),
                ("weights", ctypes.c_int), ("act", ctypes.c_int), ("dtype", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("lb_coef", ctypes.c_float),
                ("z_coef", ctypes.c_float)]


class MoeRouteOut(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("idx", "gate", "load", "counts", "offsets", "row_token", "tok_row",
                 "tok_gate", "drop", "scores", "logits", "lse", "aux", "ec_hist")]


_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m expert_dispatch_gemm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        cfgp = ctypes.POINTER(MoeConfig)
        outp = ctypes.POINTER(MoeRouteOut)
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_validate.argtypes = [cfgp]
        ip = ctypes.POINTER(ctypes.c_int)
        L.moe_sizes.argtypes = [cfgp, ip, ip, ip, ip, ip]
        L.moe_workspace_size.argtypes = [cfgp, ctypes.POINTER(ctypes.c_size_t),
                                         ctypes.POINTER(ctypes.c_size_t)]
        L.moe_route.argtypes = [cfgp, P, P, P, P, outp, P, ctypes.c_size_t, P]
        L.moe_route_from_scores.argtypes = [cfgp, P, P, outp, P, ctypes.c_size_t, P]
        L.moe_dispatch.argtypes = [cfgp, P, outp, P, P]
        L.moe_expert_ffn.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                     ctypes.c_size_t, P]
        L.moe_combine.argtypes = [cfgp, P, outp, P, P]
        L.moe_layer_forward.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, outp, P,
                                        ctypes.c_size_t, P]
        L.moe_layer_forward_host.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P, outp,
                                             P, ctypes.c_size_t, P]
        L.moe_train_launch_counts.argtypes = [cfgp, ip, ip]
        L.moe_debug_inject_fault.argtypes = [ctypes.c_int]
        L.moe_bias_update.argtypes = [cfgp, P, ctypes.c_float, P, P]
        L.moe_workspace_init.argtypes = [P, P]
        L.moe_read_error.argtypes = [P, P, ip]
        L.moe_route_noalloc.argtypes = [cfgp, P, P, P, P, outp, P]
        L.moe_expert_ffn_gathered.argtypes = [cfgp, P, outp, P, P, P, P, P, P, P, P, P,
                                              ctypes.c_size_t, P]
        L.moe_expert_ffn_combined.argtypes = [cfgp, P, P, outp, P, P, P, P, P, P, P, P, P, P,
                                              P, ctypes.c_size_t, P]
        L.moe_layer_forward_train.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, outp, P,
                                              ctypes.c_size_t, P, ctypes.c_size_t, P]
        L.moe_layer_backward_train.argtypes = [cfgp, P, P, P, P, P, P, P, P, outp, P,
                                               ctypes.c_size_t, P, P, P, P, P, P, P, P, P, P, P,
                                               ctypes.c_size_t, P]
        L.moe_backward_workspace_size.argtypes = [cfgp, ctypes.POINTER(ctypes.c_size_t), ip]
        L.moe_layer_backward.argtypes = [cfgp, P, P, P, P, P, P, P, P, outp, P, ctypes.c_size_t,
                                         P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        for s in API_SYMBOLS[1:]:
            getattr(L, s).restype = ctypes.c_int
        _LIB = L
    return _LIB


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ---------------------------------------------------------------------------
# configs
# ---------------------------------------------------------------------------

def config(w: Workload, **override) -> MoeConfig:
    """The C config of a workload (k / capacity derived by the library)."""
    ec = w.mode == "ec"
    c = MoeConfig(
        n=w.n, d=w.d, E=w.E, h=w.h,
        mode=MOE_EXPERT_CHOICE if ec else MOE_TOKEN_CHOICE,
        score={"sigmoid": MOE_SCORE_SIGMOID,
               "sqrtsoftplus": MOE_SCORE_SQRTSOFTPLUS}.get(w.score, MOE_SCORE_SOFTMAX),
        k=0 if ec else w.K,
        capacity_factor=w.c if ec else w.capacity_factor,
        capacity=0 if (not ec and w.capacity_factor > 0) else -1,
        n_groups=w.n_groups, topk_groups=w.topk_groups, group_topn=w.group_topn,
        weights=MOE_W_NORMALIZED if w.weights == "normalized" else MOE_W_RAW,
        act={"relu": MOE_ACT_RELU, "gelu": MOE_ACT_GELU, "swiglu": MOE_ACT_SWIGLU}[w.act],
        dtype=MOE_F32 if w.dtype == "f32" else MOE_BF16,
        n_shared=w.n_shared, lb_coef=w.lb_coef, z_coef=w.z_coef)
    for k, v in override.items():
        setattr(c, k, v)
    return c


@dataclass
class Sizes:
    k: int
    capacity: int
    slots: int
    rows: int
    shared_row_base: int
    route_ws: int
    layer_ws: int


def sizes(cfg: MoeConfig) -> Sizes:
    L = lib()
    k, cap, slots, rows, sb = (ctypes.c_int() for _ in range(5))
    _check(L.moe_sizes(ctypes.byref(cfg), ctypes.byref(k), ctypes.byref(cap),
                       ctypes.byref(slots), ctypes.byref(rows), ctypes.byref(sb)), "moe_sizes")
    r, l = ctypes.c_size_t(), ctypes.c_size_t()
    _check(L.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(r), ctypes.byref(l)),
           "moe_workspace_size")
    return Sizes(k.value, cap.value, slots.value, rows.value, sb.value, r.value, l.value)


def launch_counts(cfg: MoeConfig) -> dict:
    """Kernels each call enqueues: route, dispatch, ffn, combine."""
    vals = [ctypes.c_int() for _ in range(4)]
    _check(lib().moe_launch_counts(ctypes.byref(cfg), *(ctypes.byref(v) for v in vals)),
           "moe_launch_counts")
    return dict(zip(("route", "dispatch", "ffn", "combine"), (v.value for v in vals)))


def train_launch_counts(cfg: MoeConfig) -> tuple:
    """Kernels of the training pair: (moe_layer_forward_train, moe_layer_backward_train)."""
    f, b = ctypes.c_int(), ctypes.c_int()
    _check(lib().moe_train_launch_counts(ctypes.byref(cfg), ctypes.byref(f), ctypes.byref(b)),
           "moe_train_launch_counts")
    return f.value, b.value


def validate(cfg: MoeConfig) -> int:
    return lib().moe_validate(ctypes.byref(cfg))


# ---------------------------------------------------------------------------
# buffers (torch allocates; the library only fills them)
# ---------------------------------------------------------------------------

class RouteBuffers:
    """Device tensors of one moe_route_out."""

    def __init__(self, cfg: MoeConfig, device, logits: bool = True):
        sz = sizes(cfg)
        n, E = cfg.n, cfg.E
        ec = cfg.mode == MOE_EXPERT_CHOICE
        i32, f32 = torch.int32, torch.float32
        shape = (E, sz.k) if ec else (n, sz.k)
        self.idx = torch.empty(shape, dtype=i32, device=device)
        self.gate = torch.empty(shape, dtype=f32, device=device)
        self.load = torch.empty(E, dtype=i32, device=device)
        self.counts = torch.empty(E, dtype=i32, device=device)
        self.offsets = torch.empty(E + 1, dtype=i32, device=device)
        self.row_token = torch.empty(max(sz.rows, 1), dtype=i32, device=device)
        self.tok_row = torch.empty((n, sz.slots), dtype=i32, device=device)
        self.tok_gate = torch.empty((n, sz.slots), dtype=f32, device=device)
        self.drop = None if ec else torch.empty((n, sz.k), dtype=torch.uint8, device=device)
        self.scores = torch.empty((n, E), dtype=f32, device=device)
        self.logits = torch.empty((n, E), dtype=f32, device=device) if logits else None
        self.lse = torch.empty(n, dtype=f32, device=device) if logits else None
        self.aux = torch.empty(MOE_AUX_LEN, dtype=f32, device=device)
        self.ec_hist = torch.empty(E + 1, dtype=i32, device=device) if ec else None
        self.sizes = sz
        self.c = MoeRouteOut(*[None if t is None else t.data_ptr() for t in (
            self.idx, self.gate, self.load, self.counts, self.offsets, self.row_token,
            self.tok_row, self.tok_gate, self.drop, self.scores, self.logits, self.lse,
            self.aux, self.ec_hist)])

    def aux_dict(self) -> dict:
        return dict(zip(AUX_NAMES, self.aux.tolist()))


def workspace(cfg: MoeConfig, device, layer: bool = True, stream=None) -> torch.Tensor:
    """A zero-initialised, 256-byte aligned workspace (torch caching allocator)."""
    sz = sizes(cfg)
    nbytes = sz.layer_ws if layer else sz.route_ws
    ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + nbytes]
    _check(lib().moe_workspace_init(_ptr(ws), _stream(stream)), "moe_workspace_init")
    return ws


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def moe_route(cfg, X, Wg, logit_bias, sel_bias, route: RouteBuffers, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(cfg), _ptr(X), _ptr(Wg), _ptr(logit_bias),
                           _ptr(sel_bias), ctypes.byref(route.c), _ptr(ws), ws.numel(),
                           _stream(stream)), "moe_route")


def moe_route_from_scores(cfg, S, sel_bias, route: RouteBuffers, ws, stream=None):
    _check(lib().moe_route_from_scores(ctypes.byref(cfg), _ptr(S), _ptr(sel_bias),
                                       ctypes.byref(route.c), _ptr(ws), ws.numel(),
                                       _stream(stream)), "moe_route_from_scores")


def moe_dispatch(cfg, X, route: RouteBuffers, X_perm, stream=None):
    _check(lib().moe_dispatch(ctypes.byref(cfg), _ptr(X), ctypes.byref(route.c),
                              _ptr(X_perm), _stream(stream)), "moe_dispatch")


def moe_expert_ffn(cfg, X, X_perm, offsets, W1, W3, W2, sW1, sW3, sW2, H, Y_perm, ws,
                   stream=None, counts=None):
    _check(lib().moe_expert_ffn(ctypes.byref(cfg), _ptr(X), _ptr(X_perm), _ptr(offsets),
                                _ptr(counts), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(sW1),
                                _ptr(sW3), _ptr(sW2), _ptr(H), _ptr(Y_perm), _ptr(ws),
                                ws.numel(), _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_gathered(cfg, X, route: RouteBuffers, W1, W3, W2, sW1, sW3, sW2, H, Y_perm,
                            ws, stream=None):
    _check(lib().moe_expert_ffn_gathered(ctypes.byref(cfg), _ptr(X), ctypes.byref(route.c),
                                         _ptr(W1), _ptr(W3), _ptr(W2), _ptr(sW1), _ptr(sW3),
                                         _ptr(sW2), _ptr(H), _ptr(Y_perm), _ptr(ws), ws.numel(),
                                         _stream(stream)), "moe_expert_ffn_gathered")


def moe_expert_ffn_combined(cfg, X, X_perm, route: RouteBuffers, W1, W3, W2, sW1, sW3, sW2, H,
                            acc, row_gate, out, ws, stream=None):
    _check(lib().moe_expert_ffn_combined(ctypes.byref(cfg), _ptr(X), _ptr(X_perm),
                                         ctypes.byref(route.c), _ptr(W1), _ptr(W3), _ptr(W2),
                                         _ptr(sW1), _ptr(sW3), _ptr(sW2), _ptr(H), _ptr(acc),
                                         _ptr(row_gate), _ptr(out), _ptr(ws), ws.numel(),
                                         _stream(stream)), "moe_expert_ffn_combined")


def moe_combine(cfg, Y_perm, route: RouteBuffers, out, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), _ptr(Y_perm), ctypes.byref(route.c),
                             _ptr(out), _stream(stream)), "moe_combine")


def moe_layer_forward(cfg, X, Wg, logit_bias, sel_bias, W1, W3, W2, sW1, sW3, sW2, out,
                      route: RouteBuffers, ws, stream=None):
    _check(lib().moe_layer_forward(ctypes.byref(cfg), _ptr(X), _ptr(Wg), _ptr(logit_bias),
                                   _ptr(sel_bias), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(sW1),
                                   _ptr(sW3), _ptr(sW2), _ptr(out), ctypes.byref(route.c),
                                   _ptr(ws), ws.numel(), _stream(stream)),
           "moe_layer_forward")


def moe_layer_forward_host(cfg, X_host, Wg, logit_bias, sel_bias, W1, W3, W2, sW1, sW3, sW2,
                           out_host, X_dev, out_dev, route: RouteBuffers, ws, stream=None):
    """moe_layer_forward on host X / out (CPU tensors, ideally pinned): the
    library copies X_host into X_dev, runs the layer and copies out_dev back
    into out_host, all on `stream`, without synchronising."""
    for t in (X_host, out_host):
        if t.is_cuda:
            raise ValueError("X_host and out_host must be host tensors")
    _check(lib().moe_layer_forward_host(ctypes.byref(cfg), _ptr(X_host), _ptr(Wg),
                                        _ptr(logit_bias), _ptr(sel_bias), _ptr(W1), _ptr(W3),
                                        _ptr(W2), _ptr(sW1), _ptr(sW3), _ptr(sW2),
                                        _ptr(out_host), _ptr(X_dev), _ptr(out_dev),
                                        ctypes.byref(route.c), _ptr(ws), ws.numel(),
                                        _stream(stream)), "moe_layer_forward_host")


def moe_bias_update(cfg, load, rate: float, bias, stream=None):
    _check(lib().moe_bias_update(ctypes.byref(cfg), _ptr(load), ctypes.c_float(rate),
                                 _ptr(bias), _stream(stream)), "moe_bias_update")


def moe_route_noalloc(cfg, X, Wg, logit_bias, sel_bias, route: RouteBuffers, stream=None):
    """moe_route with the library's built-in scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/moe.h)."""
    _check(lib().moe_route_noalloc(ctypes.byref(cfg), _ptr(X), _ptr(Wg), _ptr(logit_bias),
                                   _ptr(sel_bias), ctypes.byref(route.c), _stream(stream)),
           "moe_route_noalloc")


def backward_workspace(cfg: MoeConfig, device, stream=None):
    """(workspace tensor for moe_layer_backward, kernels it enqueues)."""
    nbytes = ctypes.c_size_t()
    launches = ctypes.c_int()
    _check(lib().moe_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(nbytes),
                                             ctypes.byref(launches)),
           "moe_backward_workspace_size")
    ws = torch.empty(nbytes.value + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + nbytes.value]
    _check(lib().moe_workspace_init(_ptr(ws), _stream(stream)), "moe_workspace_init")
    return ws, launches.value


def moe_layer_backward(cfg, X, Wg, W1, W3, W2, sW1, sW3, sW2, route: RouteBuffers, fwd_ws,
                       dout, dX, dWg, dW1, dW3, dW2, dsW1, dsW3, dsW2, dL, ws, stream=None):
    _check(lib().moe_layer_backward(ctypes.byref(cfg), _ptr(X), _ptr(Wg), _ptr(W1), _ptr(W3),
                                    _ptr(W2), _ptr(sW1), _ptr(sW3), _ptr(sW2),
                                    ctypes.byref(route.c), _ptr(fwd_ws), fwd_ws.numel(),
                                    _ptr(dout), _ptr(dX), _ptr(dWg), _ptr(dW1), _ptr(dW3),
                                    _ptr(dW2), _ptr(dsW1), _ptr(dsW3), _ptr(dsW2), _ptr(dL),
                                    _ptr(ws), ws.numel(), _stream(stream)),
           "moe_layer_backward")


def moe_layer_forward_train(cfg, X, Wg, logit_bias, sel_bias, W1, W3, W2, sW1, sW3, sW2, out,
                            route: RouteBuffers, ws, bwd_ws, stream=None):
    _check(lib().moe_layer_forward_train(ctypes.byref(cfg), _ptr(X), _ptr(Wg), _ptr(logit_bias),
                                         _ptr(sel_bias), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(sW1),
                                         _ptr(sW3), _ptr(sW2), _ptr(out), ctypes.byref(route.c),
                                         _ptr(ws), ws.numel(), _ptr(bwd_ws), bwd_ws.numel(),
                                         _stream(stream)), "moe_layer_forward_train")


def moe_layer_backward_train(cfg, X, Wg, W1, W3, W2, sW1, sW3, sW2, route: RouteBuffers, fwd_ws,
                             dout, dX, dWg, dW1, dW3, dW2, dsW1, dsW3, dsW2, dL, ws,
                             stream=None):
    _check(lib().moe_layer_backward_train(ctypes.byref(cfg), _ptr(X), _ptr(Wg), _ptr(W1),
                                          _ptr(W3), _ptr(W2), _ptr(sW1), _ptr(sW3), _ptr(sW2),
                                          ctypes.byref(route.c), _ptr(fwd_ws), fwd_ws.numel(),
                                          _ptr(dout), _ptr(dX), _ptr(dWg), _ptr(dW1), _ptr(dW3),
                                          _ptr(dW2), _ptr(dsW1), _ptr(dsW3), _ptr(dsW2),
                                          _ptr(dL), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_layer_backward_train")


def debug_inject_fault(fault: int):
    """Arms a one-shot failure-path test fault (moe_debug_inject_fault)."""
    _check(lib().moe_debug_inject_fault(fault), "moe_debug_inject_fault")


def moe_read_error(ws, stream=None):
    """(status, raw code) of the error word of `ws`; ws=None reads the word
    of moe_route_noalloc's built-in scratch on the current device."""
    detail = ctypes.c_int()
    st = lib().moe_read_error(_ptr(ws), _stream(stream), ctypes.byref(detail))
    return st, detail.value


# ---------------------------------------------------------------------------
# a whole layer with its buffers
# ---------------------------------------------------------------------------

class Layer:
    """Inputs, weights, buffers and workspace of one workload on one device."""

    def __init__(self, w: Workload, inputs: dict, device, **cfg_override):
        self.w = w
        self.cfg = config(w, **cfg_override)
        self.device = device
        self.inp = inputs
        self.route = RouteBuffers(self.cfg, device)
        self.ws = workspace(self.cfg, device, layer=True)
        self.out = torch.empty((w.n, w.d), dtype=w.torch_dtype, device=device)
        self.sizes = self.route.sizes

    def forward(self, X=None, stream=None):
        i = self.inp
        moe_layer_forward(self.cfg, i["X"] if X is None else X, i["Wg"], i.get("logit_bias"),
                          i.get("sel_bias"), i["W1"], i.get("W3"), i["W2"], i.get("sW1"),
                          i.get("sW3"), i.get("sW2"), self.out, self.route, self.ws, stream)
        return self.out

    def grads(self):
        """Gradient buffers of the layer's inputs and weights (allocated once)."""
        if not hasattr(self, "_grads"):
            i, dev = self.inp, self.device
            g = {"dX": torch.empty_like(i["X"]),
                 "dWg": torch.empty_like(i["Wg"]),
                 "dW1": torch.empty_like(i["W1"]), "dW2": torch.empty_like(i["W2"]),
                 "dW3": torch.empty_like(i["W3"]) if i.get("W3") is not None else None,
                 "dsW1": torch.empty_like(i["sW1"]) if i.get("sW1") is not None else None,
                 "dsW2": torch.empty_like(i["sW2"]) if i.get("sW2") is not None else None,
                 "dsW3": torch.empty_like(i["sW3"]) if i.get("sW3") is not None else None,
                 "dL": torch.empty((self.w.n, self.w.E), dtype=torch.float32, device=dev)}
            self._bws, self.bwd_launches = backward_workspace(self.cfg, dev)
            self._grads = g
        return self._grads

    def forward_train(self, X=None, stream=None):
        """forward() that also keeps the up projection's U, V and H for
        backward_train() (moe_layer_forward_train)."""
        i = self.inp
        self.grads()
        moe_layer_forward_train(self.cfg, i["X"] if X is None else X, i["Wg"],
                                i.get("logit_bias"), i.get("sel_bias"), i["W1"], i.get("W3"),
                                i["W2"], i.get("sW1"), i.get("sW3"), i.get("sW2"), self.out,
                                self.route, self.ws, self._bws, stream)
        return self.out

    def backward_train(self, dout, X=None, stream=None):
        """backward() after forward_train(): no recompute of the up projection."""
        i, g = self.inp, self.grads()
        moe_layer_backward_train(self.cfg, i["X"] if X is None else X, i["Wg"], i["W1"],
                                 i.get("W3"), i["W2"], i.get("sW1"), i.get("sW3"), i.get("sW2"),
                                 self.route, self.ws, dout, g["dX"], g["dWg"], g["dW1"],
                                 g["dW3"], g["dW2"], g["dsW1"], g["dsW3"], g["dsW2"], g["dL"],
                                 self._bws, stream)
        return g

    def backward(self, dout, X=None, stream=None):
        """Gradients of <dout, out> + the aux losses after forward() on the same
        inputs (the forward's workspace and routing are read)."""
        i, g = self.inp, self.grads()
        moe_layer_backward(self.cfg, i["X"] if X is None else X, i["Wg"], i["W1"], i.get("W3"),
                           i["W2"], i.get("sW1"), i.get("sW3"), i.get("sW2"), self.route,
                           self.ws, dout, g["dX"], g["dWg"], g["dW1"], g["dW3"], g["dW2"],
                           g["dsW1"], g["dsW3"], g["dsW2"], g["dL"], self._bws, stream)
        return g
