"""GPU parity of the layer's backward pass (moe_layer_backward through the C
ABI) against the oracle's chain-rule backward on the same seeded inputs.

Every gradient the library writes is compared: the logits' gradient dL and
the router weight gradient dWg (fp32) to a relative Frobenius error of 5e-3,
the input gradient dX and every expert's and shared expert's weight
gradients (bf16) to 2e-2, the same bar as the layer's bf16 outputs. Experts
that received no rows must get exactly zero weight gradients.
"""
import numpy as np
import pytest
import torch

import oracle
from expert_dispatch_gemm_b200 import moe
from expert_dispatch_gemm_b200 import workloads as wl
from tests.gpu_common import bf16_ulp, expert_weights_from, explained_routing_diff, host

pytestmark = pytest.mark.gpu
DEV = "cuda"

F32_GRAD_TOL = 5e-3
BF16_GRAD_TOL = 2e-2
FP32_LAYER_TOL = 1e-4  # every gradient of an fp32 layer (FFMA, no rounding to bf16)

BWD_SMALL = wl.SMALL + [
    # fp32 end to end: token choice, SwiGLU, a shared expert, capacity drops
    wl.TC_TOP2_CAP.replace(name="bwd-f32-top2of8-cap-shared1-n500-d128-h192", n=500, d=128,
                           h=192, dtype="f32", n_shared=1),
    # ReLU experts, strong aux-loss coefficients (their gradient terms matter)
    wl.TC_DROPLESS.replace(name="bwd-top4of16-relu-aux0.5-n1000-d192-h192", n=1000, d=192, E=16,
                           K=4, h=192, act="relu", lb_coef=0.5, z_coef=0.5),
    # sqrt(softplus) scores, shared expert, group-limited
    wl.TC_SIGMOID_GROUPED.replace(name="bwd-sqrtsoftplus-grouped-shared-n300-d128-e64-h128",
                                  n=300, d=128, E=64, h=128, score="sqrtsoftplus", bias_steps=0,
                                  z_coef=0.2),
    # 64 tokens over 64 experts, top-1: most experts get no rows (zero
    # gradients) and the rest one or two
    wl.TC_DROPLESS.replace(name="bwd-top1of64-sparse-n64-d128-h128", n=64, d=128, E=64, K=1,
                           h=128),
    # expert choice, GELU, the capacity of several 128-row blocks per expert
    wl.EC_BF16.replace(name="bwd-ec-gelu-n768-d128-e8-c4-h256", n=768, d=128, E=8, h=256, c=4.0),
    # the decoding regime: 16 tokens over 64 grouped sigmoid experts plus a
    # shared expert of fewer than 128 rows
    wl.TC_SIGMOID_GROUPED.replace(name="bwd-decode-n16-top8of64-shared1-d256-h128", n=16, d=256,
                                  E=64, h=128, bias_steps=0),
    # about 256 rows per expert: dX with the weights as the M side (W1 read
    # MN-major), with a shared expert; GELU (one weight matrix) and SwiGLU
    # (W3 from K = h on, the forward's weights-as-M up projection too)
    wl.TC_DROPLESS.replace(name="bwd-swap-top4of16-shared1-gelu-n1024-d256-h256", n=1024, d=256,
                           E=16, K=4, h=256, act="gelu", n_shared=1),
    wl.TC_SIGMOID_GROUPED.replace(name="bwd-swap-grouped-top8of32-shared1-n1024-d256-h256",
                                  n=1024, d=256, E=32, h=256, bias_steps=0),
]


@pytest.fixture(autouse=True)
def _cleanup():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _dout(w, seed=17):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((w.n, w.d), generator=g).to(w.torch_dtype).to(DEV)


def _rel(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return np.linalg.norm(got - ref) / den if den > 0 else np.linalg.norm(got)


def _close(got, ref, tol, bf16, what="", absum=None):
    """A gradient against the oracle's, row by row (rows = tokens, or hidden
    units of a weight gradient): the whole block and every row within `tol`
    relative Frobenius error (a row the oracle leaves at zero must be zero),
    and, for values stored in bf16, every element within two bf16 spacings of
    the oracle's value plus 2% of its row's rms (the two sides' roundings of
    a stored value may land one spacing apart, and a weight gradient sums an
    expert's few rows of bf16 products, where one flipped input moves an
    element by up to a few percent of the row's rms). A weight gradient also
    passes the oracle's sum of its terms' magnitudes (`absum`, the same
    shape): each of its two factors per term (dU or dV and x; dY and H) is
    stored in bf16, and a rounding that lands one spacing away moves that
    term by at most 2^-7 of its size per factor, so the element may be off by
    2^-6 of the sum of |terms| (when an expert's rows cancel, that sum is far
    above the row's rms)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    g2 = got.reshape(got.shape[0], -1)
    r2 = ref.reshape(ref.shape[0], -1)
    rel = _rel(g2, r2)
    assert rel < tol, f"{what}: relative error {rel:.4g}"
    norms = np.linalg.norm(r2, axis=1)
    zero = norms == 0
    assert not g2[zero].any(), f"{what}: rows the oracle leaves at zero are not zero"
    rows = np.linalg.norm(g2 - r2, axis=1)[~zero] / norms[~zero]
    assert rows.size == 0 or rows.max() < tol, f"{what}: worst row error {rows.max():.4g}"
    if bf16:
        rms = norms / np.sqrt(r2.shape[1])
        bound = 2.0 * bf16_ulp(r2) + 2e-2 * rms[:, None]
        if absum is not None:
            bound = bound + 2.0 ** -6 * np.asarray(absum, np.float64).reshape(r2.shape)
        over = np.abs(g2 - r2) > bound
        assert not over.any(), (f"{what}: {int(over.sum())} elements beyond two bf16 "
                                f"spacings + 2% of the row rms; worst excess "
                                f"{float((np.abs(g2 - r2) - bound).max()):.4g}")
    return rel


def _close_dl(got, ref, tol, what="dL"):
    """Sampled rows of the logit gradient: the block within `tol` relative
    Frobenius error, and each row within `tol` of the larger of its own norm
    and the block's rms row norm. A row's expert terms go through the
    mixing-weight gradient dgate = <dout, Y>, a sum over d products whose
    factors Y are stored in bf16 on both sides; when that sum nearly cancels
    (a token whose dgate is small against its d terms) the two sides'
    rounding of Y moves it by a few per cent of itself, and the row is small
    too, so a row's own norm is no scale for it (the layers of
    `test_backward_small` keep the all-rows check)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = _rel(got, ref)
    assert rel < tol, f"{what}: relative error {rel:.4g}"
    norms = np.linalg.norm(ref, axis=1)
    err = np.linalg.norm(got - ref, axis=1)
    den = np.maximum(norms, np.sqrt(np.mean(norms ** 2)))
    bad = err > tol * den
    assert not bad.any(), (f"{what}: rows {np.nonzero(bad)[0].tolist()} beyond {tol}; worst "
                           f"{float((err / den).max()):.4g}")


def _close_dwg(got, ref, X, dL_ref, tol=F32_GRAD_TOL, what="dWg"):
    """dW_g = X^T dL against the oracle's: the block within `tol` relative
    Frobenius error, and every element within tol * sum_t |X[t, i]| *
    ||dL_ref[t]||: what the per-token bound ||dL_t - dL_ref_t|| <= tol
    ||dL_ref_t|| allows for a sum over tokens (a per-expert bound would not
    hold where the tokens' terms cancel)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = _rel(got, ref)
    assert rel < tol, f"{what}: relative error {rel:.4g}"
    scale = np.abs(np.asarray(X, np.float64)).T @ np.linalg.norm(
        np.asarray(dL_ref, np.float64), axis=1)
    bound = tol * scale[:, None] + 1e-7
    over = np.abs(got - ref) > bound
    assert not over.any(), f"{what}: {int(over.sum())} elements beyond the token-sum bound"
    return rel


def _ws_ok(ws):
    st, detail = moe.moe_read_error(ws)
    assert st == moe.MOE_OK, f"device error word {detail:#x}"


def _oracle_route(w, inp):
    spec = oracle.spec_of(w)
    logits, S, lse = oracle.router(host(inp["X"]), host(inp["Wg"]), host(inp.get("logit_bias")),
                                   spec["score"])
    r = oracle.route(spec, S, lse, host(inp.get("sel_bias")))
    return spec, S, r


@pytest.mark.parametrize("w", BWD_SMALL, ids=lambda w: w.name)
def test_backward_small(w):
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    layer.forward()
    dout = _dout(w)
    g = layer.backward(dout)
    torch.cuda.synchronize()
    _ws_ok(layer.ws)
    _ws_ok(layer._bws)
    spec, S, r = _oracle_route(w, inp)
    bad = explained_routing_diff(spec, r, layer.route, S, host(inp.get("sel_bias")))
    assert not bad, f"routing differs from the oracle's on {len(bad)} tokens"
    ref = oracle.layer_backward(spec, host(inp["X"]), host(inp["Wg"]), host(dout),
                                expert_weights_from(inp),
                                expert_weights_from(inp, "s") if w.n_shared else None,
                                host(inp.get("logit_bias")), host(inp.get("sel_bias")),
                                absum=True)
    f32 = w.dtype == "f32"
    tol_f32 = FP32_LAYER_TOL if f32 else F32_GRAD_TOL
    tol = FP32_LAYER_TOL if f32 else BF16_GRAD_TOL
    bf16 = not f32
    _close(host(g["dL"]), ref["dL"], tol_f32, False, "dL")
    _close_dwg(host(g["dWg"]), ref["dWg"], host(inp["X"]), ref["dL"], tol_f32)
    _close(host(g["dX"]), ref["dX"], tol, bf16, "dX")
    names = ["dW1", "dW2"] + (["dW3"] if w.act == "swiglu" else [])
    for e in range(w.E):
        for nm in names:
            got = host(g[nm][e])
            if e in ref[nm]:
                _close(got, ref[nm][e], tol, bf16, f"{nm}[{e}]", ref["a" + nm[1:]][e])
            else:
                assert not got.any(), (nm, e, "expert without rows")
    for s in range(w.n_shared):
        for nm in names:
            _close(host(g["ds" + nm[1:]][s]), ref["ds" + nm[1:]][s], tol, bf16, f"s{nm}[{s}]",
                   ref["as" + nm[1:]][s])


def test_backward_repeatable_and_forward_unchanged():
    """Two backward calls give bit-identical gradients (no atomics anywhere),
    and the forward output is the same before and after (the backward only
    clears padding rows of the forward's workspace)."""
    w = wl.SMALL[3]
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    out0 = layer.forward().clone()
    dout = _dout(w, seed=3)
    g1 = {k: v.clone() for k, v in layer.backward(dout).items() if v is not None}
    g2 = layer.backward(dout)
    torch.cuda.synchronize()
    for k, v in g1.items():
        assert torch.equal(v, g2[k]), k
    out1 = layer.forward()
    torch.cuda.synchronize()
    assert torch.equal(out0, out1)
    _ws_ok(layer._bws)


def test_backward_zero_dout_gives_only_aux_gradients():
    """dout = 0: every expert gradient and the experts' share of dX vanish;
    what remains is the aux losses' gradient (token choice), so dL has the
    closed form of the balance- and z-loss terms alone, which the oracle's
    backward also gives."""
    w = wl.SMALL[3].replace(lb_coef=0.3, z_coef=0.2)
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    layer.forward()
    dout = torch.zeros((w.n, w.d), dtype=w.torch_dtype, device=DEV)
    g = layer.backward(dout)
    torch.cuda.synchronize()
    for nm in ("dW1", "dW2", "dW3"):
        assert not g[nm].any(), nm
    spec, S, r = _oracle_route(w, inp)
    ref = oracle.layer_backward(spec, host(inp["X"]), host(inp["Wg"]), host(dout),
                                expert_weights_from(inp), None, None, None)
    _close(host(g["dL"]), ref["dL"], F32_GRAD_TOL, False, "dL")
    _close(host(g["dX"]), ref["dX"], BF16_GRAD_TOL, True, "dX")


def _flip_free_experts(spec, r, rb, bad):
    """Experts whose rows are the same on both sides (no selection flip
    touches them)."""
    if not bad:
        return None
    if spec["mode"] == "ec":
        I_g = rb.idx.cpu().numpy()
        return {e for e in range(I_g.shape[0]) if set(I_g[e].tolist()) == set(r["I"][e].tolist())}
    idx_g = rb.idx.cpu().numpy()
    touched = set()
    for t in bad:
        touched |= set(idx_g[t].tolist()) | set(r["idx"][t].tolist())
    return {e for e in range(rb.counts.numel()) if e not in touched}


@pytest.mark.parametrize("w", [wl.EC_BF16, wl.TC_TOP2_CAP, wl.TC_DROPLESS, wl.TC_SIGMOID_GROUPED],
                         ids=lambda w: w.name)
def test_backward_full_size_sampled(w):
    """The benchmark's workloads at full size: dX and dL on sampled tokens
    (each needs only its own pairs), sampled hidden units of the weight
    gradients of five experts and of the shared expert (a hidden unit's
    weight gradients depend on that unit alone, so the oracle runs the
    expert's backward restricted to the sampled units), and the whole dWg of
    a backward whose dout is zero outside the sampled tokens, against the
    oracle's. The experts are the one with the most rows, the one with the
    fewest and three between (so tiles of one and of two token chunks, odd
    and even 128-row block counts); the tokens include each such expert's
    first and last row (the first and the last tile of its dX); the hidden
    units include both ends of the first 256-unit tile and the last unit
    (both CTAs of a paired weight-gradient tile, first and last tiles)."""
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    layer.forward()
    dout = _dout(w, seed=5)
    g = layer.backward(dout)
    torch.cuda.synchronize()
    _ws_ok(layer.ws)
    _ws_ok(layer._bws)
    spec = oracle.spec_of(w)
    X = host(inp["X"])
    logits, S, lse = oracle.router(X, host(inp["Wg"]), host(inp.get("logit_bias")),
                                   spec["score"])
    r = oracle.route(spec, S, lse, host(inp.get("sel_bias")))
    bad = explained_routing_diff(spec, r, layer.route, S, host(inp.get("sel_bias")))
    rng = np.random.default_rng(3)
    pairs = oracle.token_pairs(spec, r, w.n)
    by_e = {}
    for t, e, gate in pairs:
        by_e.setdefault(e, []).append((t, gate))
    ok = _flip_free_experts(spec, r, layer.route, bad)
    cands = sorted((e for e in by_e if ok is None or e in ok), key=lambda e: (len(by_e[e]), e))
    experts = sorted({cands[0], cands[-1]} | {cands[len(cands) * q // 4] for q in (1, 2, 3)})
    # the oracle's per-token backward costs about 8 K d h FLOPs (K pairs per
    # token): at most ~8 GFLOP of it, 4 to 16 tokens; the experts' last rows
    # first, then their first rows, then random ones
    k_eff = w.K if spec["mode"] == "tc" else max(1, round(w.c))  # EC: c pairs per token
    most = int(min(16, max(4, 8e9 / (8.0 * k_eff * w.d * w.h))))
    order = ([by_e[e][-1][0] for e in experts] + [by_e[e][0][0] for e in experts] +
             [int(t) for t in rng.choice(w.n, size=16, replace=False)])
    toks = []
    for t in order:
        if t not in bad and t not in toks and len(toks) < most:
            toks.append(t)
    toks = sorted(toks)
    ref = oracle.layer_backward(spec, X, host(inp["Wg"]), host(dout), expert_weights_from(inp),
                                expert_weights_from(inp, "s") if w.n_shared else None,
                                host(inp.get("logit_bias")), host(inp.get("sel_bias")),
                                tokens=toks, pre=(logits, S, lse, r))
    tt = torch.as_tensor(toks, device=DEV)
    _close(host(g["dX"][tt]), ref["dX"], BF16_GRAD_TOL, True, "dX")
    _close_dl(host(g["dL"][tt]), ref["dL"], F32_GRAD_TOL)
    # weight gradients: sampled hidden units of the five experts (and the
    # shared one)
    J = np.unique(np.concatenate([[0, 127, 128, min(255, w.h - 1), w.h - 1],
                                  rng.choice(w.h, size=3, replace=False)]))
    W1, W3, W2 = inp["W1"], inp.get("W3"), inp["W2"]
    swiglu = W3 is not None
    checks = [(e, False) for e in experts] + [(s, True) for s in range(w.n_shared)]
    for e, shared in checks:
        p = "s" if shared else ""
        if shared:
            ts, gs = list(range(w.n)), [1.0] * w.n
        else:
            ts, gs = [t for t, _ in by_e[e]], [gt for _, gt in by_e[e]]
        dY, _ = oracle.combine_backward(np.asarray(ts, np.int32), np.asarray(gs, np.float32),
                                        np.zeros((len(ts), w.d), np.float32), host(dout),
                                        spec["store"])
        w1 = host(inp[p + "W1"][e])[J]
        w3 = host(inp[p + "W3"][e])[J] if swiglu else None
        w2 = host(inp[p + "W2"][e])[:, J]
        _, r1, r3, r2, a1, a3, a2 = oracle.expert_ffn_backward(X[ts], w1, w3, w2, dY,
                                                               spec["act"], spec["store"],
                                                               absum=True)
        jt = torch.as_tensor(J, device=DEV)
        _close(host(g["d" + p + "W1"][e][jt]), r1, BF16_GRAD_TOL, True, f"d{p}W1[{e}]", a1)
        _close(host(g["d" + p + "W2"][e][:, jt]).T, r2.T, BF16_GRAD_TOL, True, f"d{p}W2[{e}]",
               a2.T)
        if swiglu:
            _close(host(g["d" + p + "W3"][e][jt]), r3, BF16_GRAD_TOL, True, f"d{p}W3[{e}]", a3)
    # the router weight gradient dWg = X^T dL sums over every token. A second
    # backward, with dout zero outside `toks`, leaves the other tokens' dL at
    # the aux losses' terms alone, which the oracle's score backward gives for
    # every row at once (dS = 0); the oracle's router backward then gives the
    # whole dWg. (Last: this backward reuses the gradient buffers.)
    mask = torch.zeros((w.n, 1), dtype=dout.dtype, device=DEV)
    mask[tt] = 1
    dout_t = dout * mask
    layer.forward()
    g_t = layer.backward(dout_t)
    torch.cuda.synchronize()
    # a token's dL depends on its own dout row and on the aux terms alone, so
    # the sampled rows are the first oracle call's
    ref_t = ref
    tc = spec["mode"] == "tc"
    dL_all = oracle.score_backward(logits, S, lse, np.zeros(S.shape), spec["score"],
                                   r.get("load"), spec.get("K", 1),
                                   w.lb_coef if tc else 0.0, w.z_coef if tc else 0.0)
    dL_all[toks] = ref_t["dL"]
    dWg_ref, _ = oracle.router_backward(X, host(inp["Wg"]), dL_all)
    _close_dl(host(g_t["dL"][tt]), ref_t["dL"], F32_GRAD_TOL, "dL (masked dout)")
    _close_dwg(host(g_t["dWg"]), dWg_ref, X, dL_all, what="dWg (masked dout)")


@pytest.mark.parametrize("w", wl.SMALL + [wl.TC_SIGMOID_GROUPED.replace(
    name="bwd-train-pair-swap-top8of64-shared1-n2048-d256-h128", n=2048, d=256, E=64, h=128,
    bias_steps=0)], ids=lambda w: w.name)
def test_training_pair_matches_recompute(w):
    """moe_layer_forward_train + moe_layer_backward_train (U, V and H kept by
    the forward) against moe_layer_forward + moe_layer_backward (recomputed):
    the same kernels compute U, V and H from the same fp32 accumulators, so
    every output and gradient agrees to rounding."""
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    out0 = layer.forward().clone()
    dout = _dout(w, seed=23)
    g0 = {k: v.clone() for k, v in layer.backward(dout).items() if v is not None}
    out1 = layer.forward_train()
    g1 = layer.backward_train(dout)
    torch.cuda.synchronize()
    _ws_ok(layer.ws)
    _ws_ok(layer._bws)
    assert _rel(host(out1), host(out0)) < 1e-6
    for k, v in g0.items():
        assert _rel(host(g1[k]), host(v)) < (1e-6 if w.dtype == "f32" else 2e-3), k
