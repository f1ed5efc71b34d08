"""CPU oracle for the MoE routing-and-dispatch layer.

TEST INFRASTRUCTURE ONLY. Only tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. It
imports nothing from the CUDA package and the CUDA package imports nothing
from it; they share only the seeded input generators.

The arithmetic lives in ``moe_oracle.c`` (plain C, double accumulation,
single thread); this module marshals numpy arrays and composes the steps in
the order of the pages' statement of the problem ("Expert choice routing",
aicassindra.com, section "The math: a gating matrix and top-k over tokens"):
scores -> top-k -> gather -> per-expert FFN -> gate scale -> scatter_add.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, library special cases or the pages'
worked numbers, except the synthetic routing statistics (experts-per-token
histogram shape, overflow rates, MaxVio trajectory), which the pages measure
on trained models: those are reported, "parity unpinned".
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from .build import build as _build

SOFTMAX, SIGMOID, SQRTSOFTPLUS = 0, 1, 2
RELU, GELU, SWIGLU = 0, 1, 2
W_RAW, W_NORMALIZED = 0, 1
STORE_F32, STORE_BF16 = 0, 1

_LIB = None

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def _opt(ptype):
    """ndpointer that also accepts None (NULL)."""

    class _Opt(ptype):
        @classmethod
        def from_param(cls, obj):
            if obj is None:
                return None
            return ptype.from_param(obj)

    return _Opt


_LIB_PATH_OVERRIDE = None


def use_library(path):
    """Load the oracle from another build of moe_oracle.c (the mutation tests
    point this at a deliberately broken copy); None restores the default."""
    global _LIB, _LIB_PATH_OVERRIDE
    _LIB_PATH_OVERRIDE = path
    _LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _LIB_PATH_OVERRIDE or _build()
        L = ctypes.CDLL(path)
        c_int, c_float, c_double = ctypes.c_int, ctypes.c_float, ctypes.c_double
        L.orc_round_bf16.argtypes = [c_double]
        L.orc_round_bf16.restype = c_float
        L.orc_round_bf16_n.argtypes = [ctypes.c_longlong, _f64p, _f32p]
        L.orc_round_bf16_n.restype = None
        L.orc_router.argtypes = [c_int, c_int, c_int, _f32p, _f32p, _opt(_f32p), c_int,
                                 _f32p, _f32p, _f64p]
        L.orc_select_ec.argtypes = [c_int, c_int, c_int, _f32p, _i32p, _f32p]
        L.orc_select_tc.argtypes = [c_int, c_int, c_int, _f32p, _opt(_f32p), c_int, c_int,
                                    c_int, c_int, _i32p, _f32p]
        L.orc_weights_tc.argtypes = [c_int, c_int, c_int, _f32p, _i32p, c_int, _f32p]
        L.orc_capacity.argtypes = [c_int, c_int, c_int, _i32p, c_int, _u8p, _i32p, _i32p,
                                   _i32p]
        L.orc_expert_ffn.argtypes = [c_int, c_int, c_int, c_int, c_int, _f32p, _f32p,
                                     _opt(_f32p), _f32p, _f32p]
        L.orc_combine.argtypes = [c_int, c_int, c_int, _i32p, _f32p, _f32p, c_int, _f32p]
        L.orc_aux.argtypes = [c_int, c_int, c_int, _i32p, _f32p, _f64p, c_double, c_double,
                              ctypes.POINTER(c_double), ctypes.POINTER(c_double),
                              ctypes.POINTER(c_double)]
        L.orc_bias_update.argtypes = [c_int, c_int, c_int, _i32p, c_float, _f32p]
        L.orc_ec_histogram.argtypes = [c_int, c_int, c_int, _i32p, _i32p]
        L.orc_combine_backward.argtypes = [c_int, c_int, c_int, _i32p, _f32p, _f32p, _f32p,
                                           c_int, _f32p, _f32p]
        L.orc_expert_ffn_backward.argtypes = [c_int, c_int, c_int, c_int, c_int, _f32p, _f32p,
                                              _opt(_f32p), _f32p, _f32p, _f32p, _f32p,
                                              _opt(_f32p), _f32p, _opt(_f32p), _opt(_f32p),
                                              _opt(_f32p)]
        L.orc_gate_backward_tc.argtypes = [c_int, c_int, c_int, _f32p, _i32p, c_int, _f64p,
                                           _f64p]
        L.orc_score_backward.argtypes = [c_int, c_int, c_int, c_int, _f32p, _f32p, _f64p,
                                         _opt(_i32p), c_double, c_double, _f64p, _f64p]
        L.orc_router_backward.argtypes = [c_int, c_int, c_int, _f32p, _f32p, _f64p, _f32p,
                                          _f64p]
        for name in ("orc_router", "orc_select_ec", "orc_select_tc", "orc_weights_tc",
                     "orc_capacity",
                     "orc_expert_ffn", "orc_combine", "orc_aux", "orc_bias_update",
                     "orc_ec_histogram", "orc_combine_backward", "orc_expert_ffn_backward",
                     "orc_gate_backward_tc", "orc_score_backward", "orc_router_backward"):
            getattr(L, name).restype = None
        _LIB = L
    return _LIB


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


# --------------------------------------------------------------------------
# single steps
# --------------------------------------------------------------------------

def round_bf16(a) -> np.ndarray:
    """Round each value to the nearest bf16 (ties to even); float32 result."""
    flat = np.ascontiguousarray(np.asarray(a, dtype=np.float64).ravel())
    out = np.empty(flat.shape, np.float32)
    lib().orc_round_bf16_n(flat.size, flat, out)
    return out.reshape(np.shape(a))


def router(X, Wg, logit_bias=None, score=SOFTMAX):
    """logits = X.W_g (+ logit bias), S = softmax / sigmoid / sqrt(softplus) of
    the logits, lse per row."""
    X = _f32(X)
    Wg = _f32(Wg)
    n, d = X.shape
    d2, E = Wg.shape
    assert d == d2
    logits = np.empty((n, E), np.float32)
    S = np.empty((n, E), np.float32)
    lse = np.empty((n,), np.float64)
    lib().orc_router(n, d, E, X, Wg, None if logit_bias is None else _f32(logit_bias),
                     score, logits, S, lse)
    return logits, S, lse


def ec_quota(n: int, E: int, c: float) -> int:
    """Expert-choice tokens per expert, k = n c / E ("Token choice vs expert
    choice routing in MoE", section "Who picks whom"); floor when inexact."""
    return int(math.floor(n * c / E + 1e-9))


def capacity_of(n: int, E: int, cf: float) -> int:
    """Per-expert buffer = tokens per batch / experts x capacity factor
    ("MoE routing strategies explained", section "2. Top-1 switch routing
    with a capacity factor"); floor when inexact."""
    return int(math.floor(n / E * cf + 1e-9))


def select_ec(S, k: int):
    S = _f32(S)
    n, E = S.shape
    assert 1 <= k <= n
    I = np.empty((E, k), np.int32)
    G = np.empty((E, k), np.float32)
    lib().orc_select_ec(n, E, k, S, I, G)
    return I, G


def select_tc(S, K: int, sel_bias=None, n_groups: int = 1, topk_groups: int = 1,
              group_topn: int = 1, weights: int = W_RAW):
    S = _f32(S)
    n, E = S.shape
    if n_groups > 1:
        assert E % n_groups == 0 and 1 <= topk_groups <= n_groups
        assert 1 <= group_topn <= E // n_groups
        assert K <= topk_groups * (E // n_groups)
    assert 1 <= K <= E
    idx = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float32)
    lib().orc_select_tc(n, E, K, S, None if sel_bias is None else _f32(sel_bias),
                        n_groups, topk_groups, group_topn, weights, idx, w)
    return idx, w


def weights_tc(S, idx, weights: int = W_RAW):
    """Mixing weights [n,K] of the given selection idx [n,K] from the scores S
    (the weights select_tc returns along with its own selection)."""
    S = _f32(S)
    idx = _i32(idx)
    n, E = S.shape
    K = idx.shape[1]
    assert idx.shape[0] == n and ((idx >= 0) & (idx < E)).all()
    w = np.empty((n, K), np.float32)
    lib().orc_weights_tc(n, E, K, S, idx, weights, w)
    return w


def apply_capacity(idx, E: int, cap: int):
    """Returns drop [n,K] u8, load [E], kept [E], pos [n,K] (-1 when dropped)."""
    idx = _i32(idx)
    n, K = idx.shape
    drop = np.empty((n, K), np.uint8)
    load = np.empty((E,), np.int32)
    kept = np.empty((E,), np.int32)
    pos = np.empty((n, K), np.int32)
    lib().orc_capacity(n, E, K, idx, int(cap), drop, load, kept, pos)
    return drop, load, kept, pos


def expert_ffn(X, W1, W3, W2, act: int, store: int):
    X = _f32(X)
    m, d = X.shape
    h = W1.shape[0]
    Y = np.empty((m, d), np.float32)
    if m:
        lib().orc_expert_ffn(m, d, h, act, store, X, _f32(W1),
                             None if W3 is None else _f32(W3), _f32(W2), Y)
    return Y


def combine(n: int, pair_token, pair_gate, Y, store: int):
    Y = _f32(Y)
    P = len(pair_token)
    d = Y.shape[1]
    out = np.empty((n, d), np.float32)
    lib().orc_combine(n, d, P, _i32(pair_token), _f32(pair_gate), Y, store, out)
    return out


def aux(load, S, lse, K: int, lb_coef: float = 0.01, z_coef: float = 0.001):
    S = _f32(S)
    n, E = S.shape
    lb, z, mv = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    lib().orc_aux(n, E, K, _i32(load), S, np.ascontiguousarray(lse, np.float64),
                  lb_coef, z_coef, ctypes.byref(lb), ctypes.byref(z), ctypes.byref(mv))
    return lb.value, z.value, mv.value


def bias_update(load, n: int, K: int, rate: float, bias):
    b = np.array(bias, dtype=np.float32, copy=True)
    lib().orc_bias_update(n, len(b), K, _i32(load), rate, b)
    return b


def ec_histogram(I, n: int):
    I = _i32(I)
    E, k = I.shape
    hist = np.empty((E + 1,), np.int32)
    lib().orc_ec_histogram(n, E, k, I, hist)
    return hist


# --------------------------------------------------------------------------
# the whole layer
# --------------------------------------------------------------------------

def spec_of(w) -> dict:
    """Oracle spec of a workload description (any object with the fields
    mode, n, E, c, K, capacity_factor, n_groups, topk_groups, group_topn,
    weights, act, dtype, n_shared, score, lb_coef, z_coef). The quota and
    the capacity are derived here, from the pages' formulas."""
    if w.mode == "ec":
        spec = dict(mode="ec", k=ec_quota(w.n, w.E, w.c))
    else:
        cap = capacity_of(w.n, w.E, w.capacity_factor) if w.capacity_factor > 0 else -1
        spec = dict(mode="tc", K=w.K, capacity=cap, n_groups=w.n_groups,
                    topk_groups=w.topk_groups, group_topn=w.group_topn,
                    weights=W_NORMALIZED if w.weights == "normalized" else W_RAW)
    spec.update(act={"relu": RELU, "gelu": GELU, "swiglu": SWIGLU}[w.act],
                store=STORE_F32 if w.dtype == "f32" else STORE_BF16,
                n_shared=w.n_shared,
                score={"sigmoid": SIGMOID, "sqrtsoftplus": SQRTSOFTPLUS}.get(w.score, SOFTMAX),
                lb_coef=w.lb_coef, z_coef=w.z_coef)
    return spec


def route(spec: dict, S, lse=None, sel_bias=None):
    """Selection + capacity + aux from a score matrix, per ``spec``:

    mode 'ec' | 'tc'; k (EC tokens per expert) or K (TC experts per token);
    capacity (-1 dropless); n_groups/topk_groups/group_topn; weights.
    Returns a dict of the routing tensors."""
    S = _f32(S)
    n, E = S.shape
    r = {"S": S}
    if spec["mode"] == "ec":
        I, G = select_ec(S, spec["k"])
        r.update(I=I, G=G, hist=ec_histogram(I, n),
                 load=np.full((E,), spec["k"], np.int32))
        r["kept"] = r["load"].copy()
    else:
        K = spec["K"]
        idx, w = select_tc(S, K, sel_bias, spec.get("n_groups", 1), spec.get("topk_groups", 1),
                           spec.get("group_topn", 1), spec.get("weights", W_RAW))
        drop, load, kept, pos = apply_capacity(idx, E, spec.get("capacity", -1))
        r.update(idx=idx, w=w, drop=drop, load=load, kept=kept, pos=pos)
        if lse is not None:
            r["lb"], r["z"], r["maxvio"] = aux(load, S, lse, K, spec.get("lb_coef", 0.01),
                                               spec.get("z_coef", 0.001))
    return r


def token_pairs(spec: dict, routing: dict, n: int, tokens=None):
    """The (token, expert, gate) pairs whose FFN output reaches `tokens`
    (all tokens when None), ordered by token then expert."""
    want = None if tokens is None else set(int(t) for t in tokens)
    pairs = []
    if spec["mode"] == "ec":
        I, G = routing["I"], routing["G"]
        E, k = I.shape
        for e in range(E):
            for j in range(k):
                t = int(I[e, j])
                if want is None or t in want:
                    pairs.append((t, e, float(G[e, j])))
    else:
        idx, w, drop = routing["idx"], routing["w"], routing["drop"]
        nK = idx.shape[1]
        rows = range(n) if want is None else sorted(want)
        for t in rows:
            for j in range(nK):
                if not drop[t, j]:
                    pairs.append((t, int(idx[t, j]), float(w[t, j])))
    pairs.sort(key=lambda p: (p[0], p[1]))
    return pairs


def layer_forward(spec: dict, X, routing: dict, expert_weights, shared_weights=None,
                  tokens=None, absum: bool = False):
    """out rows for `tokens` (all when None) of the MoE layer given a routing.

    expert_weights(e) -> (W1 [h,d], W3 [h,d] or None, W2 [d,h]) as float32;
    shared_weights(s) -> same for always-on shared expert s (weight 1,
    "MoE routing strategies explained", section "3. Shared plus routed
    experts"). The residual is not added: the layer returns scatter_add only.
    With absum=True, returns (out, A) where A is the same combine taken over
    |gate| * |Y| (fp32, unrounded): the scale of each output element's terms,
    which the tests use to bound rounding differences."""
    X = _f32(X)
    n, d = X.shape
    store, act = spec["store"], spec["act"]
    pairs = token_pairs(spec, routing, n, tokens)
    rows = list(range(n)) if tokens is None else [int(t) for t in tokens]
    pos_of = {t: i for i, t in enumerate(rows)}
    Ys, ptok, pgate = [], [], []
    by_e = {}
    for t, e, g in pairs:
        by_e.setdefault(e, []).append((t, g))
    for e in sorted(by_e):
        W1, W3, W2 = expert_weights(e)
        ts = [t for t, _ in by_e[e]]
        Y = expert_ffn(X[ts], W1, W3, W2, act, store)
        Ys.append(Y)
        ptok += [pos_of[t] for t in ts]
        pgate += [g for _, g in by_e[e]]
    for s in range(spec.get("n_shared", 0)):
        W1, W3, W2 = shared_weights(s)
        Ys.append(expert_ffn(X[rows], W1, W3, W2, act, store))
        ptok += list(range(len(rows)))
        pgate += [1.0] * len(rows)
    Yall = np.concatenate(Ys, 0) if Ys else np.zeros((0, d), np.float32)
    order = np.argsort(np.asarray(ptok, np.int64), kind="stable")
    tok_o = np.asarray(ptok, np.int32)[order]
    gate_o = np.asarray(pgate, np.float32)[order]
    out = combine(len(rows), tok_o, gate_o, Yall[order], store)
    if not absum:
        return out
    return out, combine(len(rows), tok_o, np.abs(gate_o), np.abs(Yall[order]), STORE_F32)


# --------------------------------------------------------------------------
# backward pass: the chain rule through the steps above
# --------------------------------------------------------------------------

def combine_backward(pair_token, pair_gate, Y, dout, store: int):
    """dY[p] = gate[p] dout[token[p]] (stored), dgate[p] = <dout[token[p]], Y[p]>."""
    Y = _f32(Y)
    dout = _f32(dout)
    P, d = Y.shape
    dY = np.empty((P, d), np.float32)
    dgate = np.empty((P,), np.float32)
    if P:
        lib().orc_combine_backward(dout.shape[0], d, P, _i32(pair_token), _f32(pair_gate), Y,
                                   dout, store, dY, dgate)
    return dY, dgate


def expert_ffn_backward(X, W1, W3, W2, dY, act: int, store: int, absum: bool = False):
    """One expert's backward over its rows: (dX [m,d], dW1 [h,d], dW3 [h,d] or
    None, dW2 [d,h]). With absum=True, also (aW1, aW3, aW2): the weight
    gradients' sums taken over the absolute values of their terms
    (sum_r |dU_rj| |x_ri|, ...), a bound helper for comparing gradients whose
    factors were stored in bf16."""
    X = _f32(X)
    m, d = X.shape
    h = W1.shape[0]
    dX = np.empty((m, d), np.float32)
    dW1 = np.zeros((h, d), np.float32)
    dW3 = np.zeros((h, d), np.float32) if act == SWIGLU else None
    dW2 = np.zeros((d, h), np.float32)
    aW1 = np.zeros((h, d), np.float32) if absum else None
    aW3 = np.zeros((h, d), np.float32) if absum and act == SWIGLU else None
    aW2 = np.zeros((d, h), np.float32) if absum else None
    if m:
        lib().orc_expert_ffn_backward(m, d, h, act, store, X, _f32(W1),
                                      None if W3 is None else _f32(W3), _f32(W2), _f32(dY),
                                      dX, dW1, dW3, dW2, aW1, aW3, aW2)
    if absum:
        return dX, dW1, dW3, dW2, aW1, aW3, aW2
    return dX, dW1, dW3, dW2


def gate_backward_tc(S, idx, weights: int, dw):
    """dS [n,E] (double) from the gradients dw [n,K] of the mixing weights."""
    S = _f32(S)
    n, E = S.shape
    K = idx.shape[1]
    dS = np.zeros((n, E), np.float64)
    lib().orc_gate_backward_tc(n, E, K, S, _i32(idx), weights,
                               np.ascontiguousarray(dw, np.float64), dS)
    return dS


def score_backward(logits, S, lse, dS, score: int, load=None, K: int = 1,
                   lb_coef: float = 0.0, z_coef: float = 0.0):
    """dL [n,E] (double) from dS, with the balance- and z-loss terms."""
    S = _f32(S)
    n, E = S.shape
    dL = np.empty((n, E), np.float64)
    lib().orc_score_backward(n, E, K, score, _f32(logits), S,
                             np.ascontiguousarray(lse, np.float64),
                             None if load is None else _i32(load), lb_coef, z_coef,
                             np.ascontiguousarray(dS, np.float64), dL)
    return dL


def router_backward(X, Wg, dL):
    """(dWg [d,E] fp32, dXr [n,d] double)."""
    X = _f32(X)
    Wg = _f32(Wg)
    n, d = X.shape
    E = Wg.shape[1]
    dWg = np.empty((d, E), np.float32)
    dXr = np.empty((n, d), np.float64)
    lib().orc_router_backward(n, d, E, X, Wg, np.ascontiguousarray(dL, np.float64), dWg, dXr)
    return dWg, dXr


def layer_backward(spec: dict, X, Wg, dout, expert_weights, shared_weights=None,
                   logit_bias=None, sel_bias=None, tokens=None, pre=None,
                   absum: bool = False):
    """Gradients of <dout, out> + lb_coef L_lb + z_coef L_z (token choice) for
    the layer of ``layer_forward``, by the chain rule through the same steps:
    combine -> expert FFN -> dispatch (a sum over each token's pairs), and
    mixing weights -> scores -> router. Selections, drops and counts are
    piecewise constant and carry no gradient.

    Returns a dict: dX [n,d] (rounded to the layer's store), dL [n,E]
    (double, the logits' gradient), dWg [d,E], dW1/dW3/dW2 {expert: array},
    dsW1/dsW3/dsW2 {shared expert: array}, dgate {(t, e): value}.
    With ``tokens`` only those rows of dX and dL are computed (each needs only
    its own pairs), and no weight gradient is returned. ``pre`` = (logits, S,
    lse, routing) from an earlier ``router`` + ``route`` of the same inputs
    skips recomputing them. With ``absum`` (and no ``tokens``) the dict also
    holds aW1/aW3/aW2 and asW1/asW3/asW2: each weight gradient's sum over the
    absolute values of its terms (see ``expert_ffn_backward``)."""
    X = _f32(X)
    dout = _f32(dout)
    n, d = X.shape
    store, act = spec["store"], spec["act"]
    score = spec.get("score", SOFTMAX)
    if pre is None:
        logits, S, lse = router(X, Wg, logit_bias, score)
        r = route(spec, S, lse, sel_bias)
    else:
        logits, S, lse, r = pre
    E = S.shape[1]
    rows = list(range(n)) if tokens is None else sorted(int(t) for t in tokens)
    pairs = token_pairs(spec, r, n, rows if tokens is not None else None)
    by_e = {}
    for t, e, g in pairs:
        by_e.setdefault(e, []).append((t, g))
    dXacc = np.zeros((n, d), np.float64)
    dgate = {}
    grads = {"dW1": {}, "dW3": {}, "dW2": {}, "dsW1": {}, "dsW3": {}, "dsW2": {}}
    want_abs = absum and tokens is None
    if want_abs:
        grads.update({"aW1": {}, "aW3": {}, "aW2": {}, "asW1": {}, "asW3": {}, "asW2": {}})
    for e in sorted(by_e):
        W1, W3, W2 = expert_weights(e)
        ts = [t for t, _ in by_e[e]]
        gs = [g for _, g in by_e[e]]
        Y = expert_ffn(X[ts], W1, W3, W2, act, store)
        dY, dg = combine_backward(np.asarray(ts, np.int32), np.asarray(gs, np.float32), Y,
                                  dout, store)
        for t, v in zip(ts, dg):
            dgate[(t, e)] = float(v)
        res = expert_ffn_backward(X[ts], W1, W3, W2, dY, act, store, absum=want_abs)
        dXp, dW1, dW3, dW2 = res[:4]
        if want_abs:
            grads["aW1"][e], grads["aW2"][e] = res[4], res[6]
            if res[5] is not None:
                grads["aW3"][e] = res[5]
        np.add.at(dXacc, np.asarray(ts), dXp.astype(np.float64))
        if tokens is None:
            grads["dW1"][e], grads["dW2"][e] = dW1, dW2
            if dW3 is not None:
                grads["dW3"][e] = dW3
    for s_ in range(spec.get("n_shared", 0)):
        W1, W3, W2 = shared_weights(s_)
        dY, _ = combine_backward(np.asarray(rows, np.int32), np.ones(len(rows), np.float32),
                                 np.zeros((len(rows), d), np.float32), dout, store)
        res = expert_ffn_backward(X[rows], W1, W3, W2, dY, act, store, absum=want_abs)
        dXp, dW1, dW3, dW2 = res[:4]
        if want_abs:
            grads["asW1"][s_], grads["asW2"][s_] = res[4], res[6]
            if res[5] is not None:
                grads["asW3"][s_] = res[5]
        dXacc[rows] += dXp.astype(np.float64)
        if tokens is None:
            grads["dsW1"][s_], grads["dsW2"][s_] = dW1, dW2
            if dW3 is not None:
                grads["dsW3"][s_] = dW3
    dS = np.zeros((n, E), np.float64)
    if spec["mode"] == "ec":
        I = r["I"]
        for e in range(E):
            for t in I[e]:
                t = int(t)
                if (t, e) in dgate:
                    dS[t, e] += dgate[(t, e)]
        lb_coef = z_coef = 0.0
        K = 1
    else:
        idx, drop = r["idx"], r["drop"]
        K = idx.shape[1]
        dw = np.zeros(idx.shape, np.float64)
        for t in rows:
            for j in range(K):
                if not drop[t, j]:
                    dw[t, j] = dgate[(t, int(idx[t, j]))]
        dS = gate_backward_tc(S, idx, spec.get("weights", W_RAW), dw)
        lb_coef, z_coef = spec.get("lb_coef", 0.0), spec.get("z_coef", 0.0)
    dL = score_backward(logits, S, lse, dS, score, r.get("load"), K, lb_coef, z_coef)
    out = {"dgate": dgate, "routing": r, "logits": logits, "S": S, "lse": lse}
    if tokens is None:
        dWg, dXr = router_backward(X, Wg, dL)
        out["dWg"] = dWg
        dXacc += dXr
        rws = slice(None)
    else:
        sub = np.asarray(rows)
        _, dXr = router_backward(X[sub], Wg, dL[sub])
        dXacc[sub] += dXr
        rws = sub
    dXs = dXacc[rws]
    out["dX"] = round_bf16(dXs) if store == STORE_BF16 else dXs.astype(np.float32)
    out["dL"] = dL[rws]
    out.update(grads)
    return out
