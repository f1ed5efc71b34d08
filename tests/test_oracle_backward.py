"""Pins of the oracle's backward pass.

The backward pass is the gradient of the forward layer, so it is pinned
against central finite differences of the (already pinned) forward oracle:
the loss <dout, out> + L_lb + L_z is evaluated at perturbed inputs and
weights, and the difference quotient must match the analytic gradient the
oracle returns. A dropped term, a wrong sign or a transposed operand anywhere
in the chain (combine, expert FFN, dispatch, mixing weights, scores, aux
losses, router) moves some coordinate far outside the tolerance. Every
perturbation is checked to leave the selection unchanged (the loss is only
piecewise smooth); coordinates that would flip it are skipped.

A second group checks the backward against torch.autograd on the special
cases where the layer reduces to a dense differentiable computation.
"""
import numpy as np
import pytest
import torch

import oracle

F32 = oracle.STORE_F32


def _case(name):
    """Tiny layers covering every score, weight mode, activation, capacity,
    group limit, selection bias, logit bias and shared expert."""
    base = dict(store=F32, n_shared=0, score=oracle.SOFTMAX, lb_coef=0.0, z_coef=0.0)
    if name == "ec-softmax-relu":
        return dict(base, mode="ec", k=8, act=oracle.RELU), dict(n=16, d=8, E=4, h=6)
    if name == "ec-softmax-gelu":
        return dict(base, mode="ec", k=5, act=oracle.GELU), dict(n=10, d=6, E=4, h=5)
    if name == "tc-top2-cap-swiglu-normalized":
        return (dict(base, mode="tc", K=2, capacity=5, n_groups=1, topk_groups=1, group_topn=1,
                     weights=oracle.W_NORMALIZED, act=oracle.SWIGLU, lb_coef=0.5, z_coef=0.3),
                dict(n=14, d=8, E=4, h=6, logit_bias=True))
    if name == "tc-top2-dropless-raw-relu-aux":
        return (dict(base, mode="tc", K=2, capacity=-1, n_groups=1, topk_groups=1, group_topn=1,
                     weights=oracle.W_RAW, act=oracle.RELU, lb_coef=0.7, z_coef=0.4),
                dict(n=12, d=6, E=5, h=4))
    if name == "tc-sigmoid-grouped-shared-swiglu":
        return (dict(base, mode="tc", K=2, capacity=-1, n_groups=4, topk_groups=2, group_topn=1,
                     weights=oracle.W_NORMALIZED, act=oracle.SWIGLU, n_shared=1,
                     score=oracle.SIGMOID, lb_coef=0.2, z_coef=0.2),
                dict(n=10, d=6, E=8, h=4, sel_bias=True))
    if name == "tc-sqrtsoftplus-raw-gelu":
        return (dict(base, mode="tc", K=2, capacity=-1, n_groups=1, topk_groups=1, group_topn=1,
                     weights=oracle.W_RAW, act=oracle.GELU, score=oracle.SQRTSOFTPLUS,
                     lb_coef=0.3, z_coef=0.3),
                dict(n=10, d=6, E=4, h=5))
    raise KeyError(name)


CASES = ["ec-softmax-relu", "ec-softmax-gelu", "tc-top2-cap-swiglu-normalized",
         "tc-top2-dropless-raw-relu-aux", "tc-sigmoid-grouped-shared-swiglu",
         "tc-sqrtsoftplus-raw-gelu"]


def _tensors(spec, shp, seed):
    rng = np.random.default_rng(seed)
    n, d, E, h = shp["n"], shp["d"], shp["E"], shp["h"]
    swiglu = spec["act"] == oracle.SWIGLU
    t = {
        "X": rng.standard_normal((n, d)).astype(np.float32),
        "Wg": (rng.standard_normal((d, E)) * 0.8).astype(np.float32),
        "W1": (rng.standard_normal((E, h, d)) / np.sqrt(d)).astype(np.float32),
        "W3": (rng.standard_normal((E, h, d)) / np.sqrt(d)).astype(np.float32) if swiglu else None,
        "W2": (rng.standard_normal((E, d, h)) / np.sqrt(h)).astype(np.float32),
        "dout": rng.standard_normal((n, d)).astype(np.float32),
        "logit_bias": (rng.standard_normal(E) * 0.5).astype(np.float32)
        if shp.get("logit_bias") else None,
        "sel_bias": (rng.standard_normal(E) * 0.05).astype(np.float32)
        if shp.get("sel_bias") else None,
    }
    ns = spec.get("n_shared", 0)
    t["sW1"] = (rng.standard_normal((max(ns, 1), h, d)) / np.sqrt(d)).astype(np.float32)
    t["sW3"] = (rng.standard_normal((max(ns, 1), h, d)) / np.sqrt(d)).astype(np.float32)
    t["sW2"] = (rng.standard_normal((max(ns, 1), d, h)) / np.sqrt(h)).astype(np.float32)
    return t


def _ew(t, pre=""):
    def f(e):
        return (t[pre + "W1"][e], None if t[pre + "W3"] is None else t[pre + "W3"][e],
                t[pre + "W2"][e])
    return f


def _loss(spec, t):
    """<dout, out> + L_lb + L_z, and a signature of the selection."""
    logits, S, lse = oracle.router(t["X"], t["Wg"], t["logit_bias"], spec["score"])
    r = oracle.route(spec, S, lse, t["sel_bias"])
    out = oracle.layer_forward(spec, t["X"], r, _ew(t),
                               _ew(t, "s") if spec.get("n_shared") else None)
    val = float((t["dout"].astype(np.float64) * out.astype(np.float64)).sum())
    if spec["mode"] == "tc":
        val += r["lb"] + r["z"]
        sig = (r["idx"].tobytes(), r["drop"].tobytes())
    else:
        sig = (r["I"].tobytes(),)
    return val, sig


def _analytic(spec, t):
    return oracle.layer_backward(spec, t["X"], t["Wg"], t["dout"], _ew(t),
                                 _ew(t, "s") if spec.get("n_shared") else None,
                                 t["logit_bias"], t["sel_bias"])


def _fd(spec, t, name, index, eps):
    arr = t[name]
    old = arr[index]
    arr[index] = np.float32(old + eps)
    hi = float(arr[index])
    lp, sp = _loss(spec, t)
    arr[index] = np.float32(old - eps)
    lo = float(arr[index])
    lm, sm = _loss(spec, t)
    arr[index] = old
    return (lp - lm) / (hi - lo), sp, sm


def _coords(rng, shape, count):
    return [tuple(int(rng.integers(0, s)) for s in shape) for _ in range(count)]


@pytest.mark.parametrize("name", CASES)
def test_backward_matches_finite_differences(name):
    spec, shp = _case(name)
    t = _tensors(spec, shp, seed=11)
    g = _analytic(spec, t)
    _, sig0 = _loss(spec, t)
    rng = np.random.default_rng(5)
    E = shp["E"]
    checks = [("X", g["dX"], None), ("Wg", g["dWg"], None)]
    for e in sorted(g["dW1"]):
        checks += [("W1", g["dW1"][e], e), ("W2", g["dW2"][e], e)]
        if spec["act"] == oracle.SWIGLU:
            checks.append(("W3", g["dW3"][e], e))
    for s_ in range(spec.get("n_shared", 0)):
        checks += [("sW1", g["dsW1"][s_], s_), ("sW2", g["dsW2"][s_], s_),
                   ("sW3", g["dsW3"][s_], s_)]
    n_checked = 0
    for pname, grad, e in checks:
        shape = grad.shape
        for c in _coords(rng, shape, 4):
            index = c if e is None else (e,) + c
            fd, sp, sm = _fd(spec, t, pname, index, 1e-3)
            if sp != sig0 or sm != sig0:
                continue  # the perturbation moved a selection boundary
            an = float(grad[c])
            assert abs(fd - an) <= 2e-3 * max(abs(an), 0.05) + 3e-4, (pname, e, c, fd, an)
            n_checked += 1
    # every gradient family was exercised
    assert n_checked >= 0.8 * 4 * len(checks), n_checked
    assert E == t["Wg"].shape[1]


def test_logit_gradient_matches_finite_differences():
    """dL itself: perturb one logit through the logit bias (a per-expert shift
    of every token's logit) and compare with the column sum of dL."""
    spec, shp = _case("tc-top2-cap-swiglu-normalized")
    t = _tensors(spec, shp, seed=3)
    g = _analytic(spec, t)
    _, sig0 = _loss(spec, t)
    for e in range(shp["E"]):
        fd, sp, sm = _fd(spec, t, "logit_bias", (e,), 1e-3)
        if sp != sig0 or sm != sig0:
            continue
        an = float(g["dL"][:, e].sum())
        assert abs(fd - an) <= 2e-3 * max(abs(an), 0.05) + 3e-4, (e, fd, an)


@pytest.mark.parametrize("act", [oracle.RELU, oracle.GELU, oracle.SWIGLU])
def test_expert_backward_against_autograd(act):
    """One expert in double precision: the oracle's rows, weight gradients and
    input gradient against torch.autograd of the same MLP (fp32 storage, so
    the comparison is at fp32 rounding)."""
    rng = np.random.default_rng(7)
    m, d, h = 9, 12, 10
    X = rng.standard_normal((m, d)).astype(np.float32)
    W1 = (rng.standard_normal((h, d)) / 3).astype(np.float32)
    W3 = (rng.standard_normal((h, d)) / 3).astype(np.float32)
    W2 = (rng.standard_normal((d, h)) / 3).astype(np.float32)
    dY = rng.standard_normal((m, d)).astype(np.float32)
    dX, dW1, dW3, dW2 = oracle.expert_ffn_backward(X, W1, W3 if act == oracle.SWIGLU else None,
                                                   W2, dY, act, F32)
    tX, t1, t3, t2 = (torch.tensor(a, dtype=torch.float64, requires_grad=True)
                      for a in (X, W1, W3, W2))
    u = tX @ t1.T
    if act == oracle.SWIGLU:
        hdn = torch.nn.functional.silu(u) * (tX @ t3.T)
    elif act == oracle.GELU:
        hdn = torch.nn.functional.gelu(u)
    else:
        hdn = torch.relu(u)
    y = hdn @ t2.T
    y.backward(torch.tensor(dY, dtype=torch.float64))
    np.testing.assert_allclose(dX, tX.grad.numpy(), rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(dW1, t1.grad.numpy(), rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(dW2, t2.grad.numpy(), rtol=1e-5, atol=1e-5)
    if act == oracle.SWIGLU:
        np.testing.assert_allclose(dW3, t3.grad.numpy(), rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("act", [oracle.SWIGLU, oracle.GELU])
def test_expert_backward_term_magnitudes(act):
    """The weight gradients' sums over |terms| (the comparison bound's input):
    sum_r |dU_rj| |x_ri| (and dV, and sum_r |dY_ri| |H_rj|) against the same
    sums of autograd's pre-activation gradients and hidden rows; each sum is
    at least |gradient|, and with one row it is |gradient| itself."""
    rng = np.random.default_rng(11)
    m, d, h = 9, 12, 10
    X = rng.standard_normal((m, d)).astype(np.float32)
    W1 = (rng.standard_normal((h, d)) / 3).astype(np.float32)
    W3 = (rng.standard_normal((h, d)) / 3).astype(np.float32)
    W2 = (rng.standard_normal((d, h)) / 3).astype(np.float32)
    dY = rng.standard_normal((m, d)).astype(np.float32)
    sw = act == oracle.SWIGLU
    _, dW1, dW3, dW2, a1, a3, a2 = oracle.expert_ffn_backward(
        X, W1, W3 if sw else None, W2, dY, act, F32, absum=True)
    tX = torch.tensor(X, dtype=torch.float64)
    u = (tX @ torch.tensor(W1, dtype=torch.float64).T).requires_grad_(True)
    v = (tX @ torch.tensor(W3, dtype=torch.float64).T).requires_grad_(True)
    hdn = torch.nn.functional.silu(u) * v if sw else torch.nn.functional.gelu(u)
    y = hdn @ torch.tensor(W2, dtype=torch.float64).T
    y.backward(torch.tensor(dY, dtype=torch.float64))
    ax = tX.abs()
    np.testing.assert_allclose(a1, (u.grad.abs().T @ ax).numpy(), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(a2, (torch.tensor(dY, dtype=torch.float64).abs().T
                                    @ hdn.detach().abs()).numpy(), rtol=1e-5, atol=1e-6)
    if sw:
        np.testing.assert_allclose(a3, (v.grad.abs().T @ ax).numpy(), rtol=1e-5, atol=1e-6)
    else:
        assert a3 is None
    for g, a in ((dW1, a1), (dW2, a2)) + (((dW3, a3),) if sw else ()):
        assert (a >= np.abs(g) * (1 - 1e-6)).all()
    # one row: every sum has a single term
    _, g1, g3, g2, b1, b3, b2 = oracle.expert_ffn_backward(
        X[:1], W1, W3 if sw else None, W2, dY[:1], act, F32, absum=True)
    for g, a in ((g1, b1), (g2, b2)) + (((g3, b3),) if sw else ()):
        np.testing.assert_allclose(a, np.abs(g), rtol=1e-6, atol=0)


@pytest.mark.parametrize("score", [oracle.SOFTMAX, oracle.SIGMOID, oracle.SQRTSOFTPLUS])
def test_score_and_router_backward_against_autograd(score):
    """With every expert selected and raw weights, the router's gradient is
    that of the dense differentiable map X -> scores, which autograd gives;
    the z-loss and balance-loss terms are added as their closed forms."""
    rng = np.random.default_rng(9)
    n, d, E = 7, 5, 4
    X = rng.standard_normal((n, d)).astype(np.float32)
    Wg = rng.standard_normal((d, E)).astype(np.float32)
    dS = rng.standard_normal((n, E))
    load = np.array([3, 9, 5, 7], np.int32)
    K, lb, z = 3, 0.4, 0.25
    logits, S, lse = oracle.router(X, Wg, None, score)
    dL = oracle.score_backward(logits, S, lse, dS, score, load, K, lb, z)
    dWg, dXr = oracle.router_backward(X, Wg, dL)
    tX = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    tW = torch.tensor(Wg, dtype=torch.float64, requires_grad=True)
    L = tX @ tW
    if score == oracle.SOFTMAX:
        s = torch.softmax(L, -1)
    elif score == oracle.SIGMOID:
        s = torch.sigmoid(L)
    else:
        s = torch.sqrt(torch.nn.functional.softplus(L))
    f = torch.tensor(load / (n * K), dtype=torch.float64)
    loss = (s * torch.tensor(dS)).sum() + lb * E * (f * s.mean(0)).sum() + \
        z * (torch.logsumexp(L, -1) ** 2).mean()
    loss.backward()
    # the oracle reads the fp32-rounded scores, so agreement is at fp32 level
    np.testing.assert_allclose(dWg, tW.grad.numpy(), rtol=2e-5, atol=2e-5)
    np.testing.assert_allclose(dXr, tX.grad.numpy(), rtol=2e-5, atol=2e-5)


def test_normalized_gate_backward_closed_form():
    """w = s / sum(s) over the selected experts: scaling every selected score
    by the same factor leaves w unchanged, so dS is orthogonal to the
    selected scores; and with dw = w (the gradient of sum w^2 / 2 is w) the
    closed form gives dS_k = (w_k - sum w^2) / sum s."""
    rng = np.random.default_rng(2)
    n, E, K = 5, 6, 3
    S = rng.uniform(0.1, 1.0, (n, E)).astype(np.float32)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(n)]).astype(np.int32)
    dw = rng.standard_normal((n, K))
    dS = oracle.gate_backward_tc(S, idx, oracle.W_NORMALIZED, dw)
    for t in range(n):
        s = S[t, idx[t]].astype(np.float64)
        assert abs(float(np.dot(dS[t, idx[t]], s))) < 1e-12
        others = np.setdiff1d(np.arange(E), idx[t])
        assert np.all(dS[t, others] == 0)
    w = S[np.arange(n)[:, None], idx].astype(np.float64)
    w = w / w.sum(1, keepdims=True)
    dS2 = oracle.gate_backward_tc(S, idx, oracle.W_NORMALIZED, w)
    for t in range(n):
        s = S[t, idx[t]].astype(np.float64)
        want = (w[t] - (w[t] ** 2).sum()) / s.sum()
        np.testing.assert_allclose(dS2[t, idx[t]], want, rtol=1e-12, atol=1e-15)
    raw = oracle.gate_backward_tc(S, idx, oracle.W_RAW, dw)
    for t in range(n):
        np.testing.assert_array_equal(raw[t, idx[t]], dw[t])
