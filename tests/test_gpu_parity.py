"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

  * identical score matrices -> routing bit-exact (indices, counts, offsets,
    dispatched-row order, drop masks, slot lists);
  * end to end from X -> logits/scores within fp32 rounding, selections equal
    except where the oracle's boundary gap is below 1e-5, layer outputs within
    max-abs 1e-4 (fp32) or relative error 2e-2 (bf16);
  * full-size workloads in the benchmark's launch configuration, checked on
    sampled tokens the oracle computes one by one;
  * edge cases: ties, a single expert, all experts, k = n, capacity 1, one
    token, ragged tails.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from expert_dispatch_gemm_b200 import moe
from expert_dispatch_gemm_b200 import workloads as wl
from tests.gpu_common import (check_routing_exact, compare_out, covering_tokens,
                              expert_weights_from, explained_routing_diff, host,
                              routing_on_gpu_selection, weights_rtol)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _cleanup():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# "7 MoE routing strategies": 2. top-1 switch with a capacity factor, plus a
# shared expert (Llama 4 Maverick); 5. grouping dropped (n_group = 1, Kimi
# K2); 4. sqrt(softplus) scores with bias balancing (DeepSeek-V4)
ROUTE_VARIANTS = [
    wl.TC_TOP2_CAP.replace(name="tc-switch-top1-cap1.25-shared1", n=384, d=128, E=8, K=1, h=128,
                           n_shared=1, logit_skew_var=0.0),
    wl.TC_SIGMOID_GROUPED.replace(name="tc-sigmoid-ngroup1-top8of64", n=260, d=128, E=64, h=64,
                                  n_groups=1, topk_groups=1, bias_steps=2),
    wl.TC_SIGMOID_GROUPED.replace(name="tc-sqrtsoftplus-grouped8keep4-top8of64", n=300, d=192,
                                  E=64, h=64, score="sqrtsoftplus", bias_steps=2),
    # 256 experts over 4,096 tokens: the router's 16-column register tiles
    # (32 rows per CTA), as the full DeepSeek-V3-shaped layer uses (56 rows)
    wl.TC_SIGMOID_GROUPED.replace(name="tc-router16-grouped8keep4-top8of256-n4096-d512", n=4096,
                                  d=512, E=256, h=64, bias_steps=2),
]


def _sel_bias(w, seed, scale=0.05):
    if w.score not in ("sigmoid", "sqrtsoftplus"):
        return None
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(w.E, generator=g) * scale).float()


def _ws_ok(ws):
    st, detail = moe.moe_read_error(ws)
    assert st == moe.MOE_OK, f"device error word {detail:#x}"


# --------------------------------------------------------------------------
# identical scores -> bit-exact routing
# --------------------------------------------------------------------------

# the largest expert-choice batch: 1024-thread selection CTAs, k > 1024 picks
EC_MAX = wl.EC_BF16.replace(name="ec-max-tokens-n16384-k2048", n=16384, d=64, E=16, h=64, c=2.0)


@pytest.mark.parametrize("kind", ["random", "ties"])
@pytest.mark.parametrize("w", wl.SMALL + wl.FULL + ROUTE_VARIANTS + [EC_MAX],
                         ids=lambda w: w.name)
def test_route_from_scores_bit_exact(w, kind):
    S = (wl.tie_heavy_scores(w.n, w.E, 5, seed=11) if kind == "ties"
         else wl.random_scores(w.n, w.E, seed=12))
    bias = _sel_bias(w, 13)
    cfg = moe.config(w)
    rb = moe.RouteBuffers(cfg, DEV, logits=False)
    ws = moe.workspace(cfg, DEV, layer=False)
    moe.moe_route_from_scores(cfg, S.to(DEV), None if bias is None else bias.to(DEV), rb, ws)
    torch.cuda.synchronize()
    spec = oracle.spec_of(w)
    Sn = S.numpy()
    bn = None if bias is None else bias.numpy()
    r = oracle.route(spec, Sn, None, bn)
    check_routing_exact(spec, r, rb, w.n, w.E, weights_rtol(spec))
    np.testing.assert_array_equal(host(rb.scores), Sn)
    aux = rb.aux.cpu().numpy()
    if spec["mode"] == "tc":
        lb, _, mv = oracle.aux(r["load"], Sn, np.zeros(w.n), spec["K"], w.lb_coef, w.z_coef)
        np.testing.assert_allclose(aux[moe.AUX_NAMES.index("lb_loss")], lb, rtol=1e-5)
        np.testing.assert_allclose(aux[2], mv, rtol=1e-6, atol=1e-7)
        assert aux[3] == int((r["load"] - r["kept"]).sum())
        assert aux[4] == int((r["drop"].sum(1) > 0).sum())
        assert aux[5] == int((r["drop"].sum(1) == spec["K"]).sum())
    else:
        assert aux[6] == r["hist"][0]
    _ws_ok(ws)


# --------------------------------------------------------------------------
# end to end from X (small sizes)
# --------------------------------------------------------------------------

def _oracle_from_x(w, inp):
    spec = oracle.spec_of(w)
    lb = inp.get("logit_bias")
    logits, S, lse = oracle.router(host(inp["X"]), host(inp["Wg"]), host(lb), spec["score"])
    sb = inp.get("sel_bias")
    r = oracle.route(spec, S, lse, host(sb))
    return spec, logits, S, lse, r


# the DeepSeek-V3-shaped layer's routing at full size (8,192 tokens, d 7168,
# 256 experts): the router launch the benchmark times, without the experts'
# weights (routing only)
ROUTE_FULL = [wl.TC_SIGMOID_GROUPED.replace(
    name="route-only-sigmoid-grouped8keep4-top8of256-n8192-d7168", bias_steps=0)]


@pytest.mark.parametrize("w", wl.SMALL + ROUTE_VARIANTS + ROUTE_FULL, ids=lambda w: w.name)
def test_route_from_x(w):
    inp = wl.make_inputs(w, DEV, experts=False)
    cfg = moe.config(w)
    rb = moe.RouteBuffers(cfg, DEV)
    ws = moe.workspace(cfg, DEV, layer=False)
    moe.moe_route(cfg, inp["X"], inp["Wg"], inp["logit_bias"], inp["sel_bias"], rb, ws)
    torch.cuda.synchronize()
    spec, logits, S, lse, r = _oracle_from_x(w, inp)
    np.testing.assert_allclose(host(rb.logits), logits, rtol=1e-5, atol=2e-5)
    np.testing.assert_allclose(host(rb.scores), S, rtol=2e-5, atol=1e-7)
    np.testing.assert_allclose(host(rb.lse), lse, rtol=1e-5, atol=2e-5)
    bad = explained_routing_diff(spec, r, rb, S, host(inp.get("sel_bias")))
    if not bad:
        check_routing_exact(spec, r, rb, w.n, w.E, weights_rtol=5e-5)
    aux = rb.aux.cpu().numpy()
    z = w.z_coef * float(np.mean(lse ** 2))
    np.testing.assert_allclose(aux[1], z, rtol=1e-4)
    if spec["mode"] == "tc":
        np.testing.assert_allclose(aux[0], r["lb"], rtol=1e-4)
    _ws_ok(ws)


def check_layer_rows(w, inp, out, rb, spec, S, r, tokens=None):
    """The layer's output rows of `tokens` (all when None) against the
    oracle, element by element. Tokens whose routing agrees with the oracle's
    are compared with the oracle's layer; tokens where a selection flipped at
    a boundary gap below 1e-5 (and, under a capacity, the drops that flip
    moved) are compared with the oracle's layer on the GPU's selection, the
    weights from the oracle's own scores."""
    bad = explained_routing_diff(spec, r, rb, S, host(inp.get("sel_bias")))
    assert len(bad) <= max(4, w.n // 100), f"{len(bad)} tokens route differently"
    toks = list(range(w.n)) if tokens is None else sorted(set(tokens) | bad)
    good = [t for t in toks if t not in bad]
    flipped = [t for t in toks if t in bad]
    ew = expert_weights_from(inp)
    sw = expert_weights_from(inp, "s") if w.n_shared else None
    X = host(inp["X"])
    got = host(out)
    worst = 0.0
    if good:
        ref, terms = oracle.layer_forward(spec, X, r, ew, sw, tokens=good, absum=True)
        worst = compare_out(spec["store"], got[good], ref, w.name, absum=terms)
    if flipped:
        rg = routing_on_gpu_selection(spec, S, rb)
        ref, terms = oracle.layer_forward(spec, X, rg, ew, sw, tokens=flipped, absum=True)
        worst = max(worst, compare_out(spec["store"], got[flipped], ref,
                                       w.name + " (flipped tokens, GPU selection)",
                                       absum=terms))
    return good, flipped, worst


@pytest.mark.parametrize("w", wl.SMALL, ids=lambda w: w.name)
def test_layer_small(w):
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    out = layer.forward()
    torch.cuda.synchronize()
    spec, logits, S, lse, r = _oracle_from_x(w, inp)
    check_layer_rows(w, inp, out, layer.route, spec, S, r)
    _ws_ok(layer.ws)


def test_stepwise_calls_equal_layer_forward():
    w = wl.SMALL[3]
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    ref = layer.forward().clone()
    cfg = layer.cfg
    sz = moe.sizes(cfg)
    rb = moe.RouteBuffers(cfg, DEV)
    ws = moe.workspace(cfg, DEV, layer=False)
    dt = w.torch_dtype
    X_perm = torch.empty((sz.rows, w.d), dtype=dt, device=DEV)
    H = torch.empty((sz.rows, w.h), dtype=dt, device=DEV)
    Y = torch.empty((sz.rows, w.d), dtype=dt, device=DEV)
    out = torch.empty((w.n, w.d), dtype=dt, device=DEV)
    moe.moe_route(cfg, inp["X"], inp["Wg"], None, None, rb, ws)
    moe.moe_dispatch(cfg, inp["X"], rb, X_perm)
    moe.moe_expert_ffn(cfg, inp["X"], X_perm, rb.offsets, inp["W1"], inp["W3"], inp["W2"],
                       None, None, None, H, Y, ws, counts=rb.counts)
    moe.moe_combine(cfg, Y, rb, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    used = int(rb.offsets[-1])
    rt = rb.row_token[:used]
    real = rt >= 0
    # the gather is an exact copy of the source rows
    assert torch.equal(X_perm[:used][real], inp["X"][rt[real].long()])
    _ws_ok(ws)


def _gathered_vs_unfused(w):
    """moe_expert_ffn_gathered (rows read from X through row_token) against
    moe_dispatch + moe_expert_ffn: same rows in, same arithmetic, so H and Y
    must agree bit for bit on every real (non-padding) row."""
    inp = wl.make_inputs(w, DEV)
    cfg = moe.config(w)
    sz = moe.sizes(cfg)
    rb = moe.RouteBuffers(cfg, DEV)
    ws = moe.workspace(cfg, DEV, layer=False)
    dt = w.torch_dtype
    X_perm = torch.empty((sz.rows, w.d), dtype=dt, device=DEV)
    H1, H2 = (torch.empty((sz.rows, w.h), dtype=dt, device=DEV) for _ in range(2))
    Y1, Y2 = (torch.empty((sz.rows, w.d), dtype=dt, device=DEV) for _ in range(2))
    moe.moe_route(cfg, inp["X"], inp["Wg"], inp["logit_bias"], inp["sel_bias"], rb, ws)
    moe.moe_dispatch(cfg, inp["X"], rb, X_perm)
    args = (inp["W1"], inp.get("W3"), inp["W2"], inp.get("sW1"), inp.get("sW3"), inp.get("sW2"))
    moe.moe_expert_ffn(cfg, inp["X"], X_perm, rb.offsets, *args, H1, Y1, ws)
    moe.moe_expert_ffn_gathered(cfg, inp["X"], rb, *args, H2, Y2, ws)
    torch.cuda.synchronize()
    used = int(rb.offsets[-1])
    real = torch.nonzero(rb.row_token[:used] >= 0).flatten()
    if w.n_shared:
        for s in range(w.n_shared):
            base = sz.shared_row_base + s * ((w.n + 127) // 128 * 128)
            real = torch.cat([real, torch.arange(base, base + w.n, device=DEV)])
    assert real.numel() > 0
    assert torch.equal(H1[real], H2[real])
    assert torch.equal(Y1[real], Y2[real])
    _ws_ok(ws)


@pytest.mark.parametrize("w", wl.SMALL, ids=lambda w: w.name)
def test_gathered_ffn_equals_dispatch_then_ffn(w):
    _gathered_vs_unfused(w)


# --------------------------------------------------------------------------
# selection-bias steps ("4. Sigmoid gating with aux-loss-free bias")
# --------------------------------------------------------------------------

def test_bias_steps_bit_exact_on_identical_scores():
    w = wl.SMALL[4]
    cfg = moe.config(w)
    spec = oracle.spec_of(w)
    rb = moe.RouteBuffers(cfg, DEV, logits=False)
    ws = moe.workspace(cfg, DEV, layer=False)
    bias_g = torch.zeros(w.E, dtype=torch.float32, device=DEV)
    bias_o = np.zeros(w.E, np.float32)
    for step in range(6):
        S = wl.random_scores(w.n, w.E, seed=100 + step) * 0.02 + 0.5  # narrow, bias matters
        moe.moe_route_from_scores(cfg, S.to(DEV), bias_g, rb, ws)
        r = oracle.route(spec, S.numpy(), None, bias_o)
        moe.moe_bias_update(cfg, rb.load, w.bias_rate, bias_g)
        bias_o = oracle.bias_update(r["load"], w.n, w.K, w.bias_rate, bias_o)
        torch.cuda.synchronize()
        check_routing_exact(spec, r, rb, w.n, w.E, weights_rtol(spec))
        np.testing.assert_array_equal(bias_g.cpu().numpy(), bias_o)
    assert np.abs(bias_o).max() > 0
    _ws_ok(ws)


# --------------------------------------------------------------------------
# full-size workloads, sampled tokens
# --------------------------------------------------------------------------

@pytest.mark.parametrize("w", wl.FULL, ids=lambda w: w.name)
def test_full_size_sampled(w):
    """The five workloads at full size in the benchmark's launch
    configuration (one moe_layer_forward call). Compared rows: for every
    expert, the token in its last kept row (its last 128-row block, which a
    CTA pair repeats when the expert's block count is odd, and the tail of
    its last weights-as-M chunk); tokens until every expert with rows is
    covered; seeded random tokens; dropped and expert-less tokens; and every
    token whose selection flipped (on the GPU's selection)."""
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    out = layer.forward()
    torch.cuda.synchronize()
    spec, logits, S, lse, r = _oracle_from_x(w, inp)
    np.testing.assert_allclose(host(layer.route.logits), logits, rtol=1e-5, atol=5e-5)
    tokens = covering_tokens(spec, r, w.n, w.E, seed=5)
    good, flipped, _ = check_layer_rows(w, inp, out, layer.route, spec, S, r, tokens)
    # every expert with kept rows feeds at least one compared token
    compared = set(good)
    if spec["mode"] == "ec":
        hit = {e for e in range(w.E) if compared & set(r["I"][e].tolist())}
        assert hit == set(range(w.E))
    else:
        kept = r["idx"][good][r["drop"][good] == 0]
        assert set(kept.tolist()) >= {e for e in range(w.E) if r["kept"][e] > 0} - \
            {int(e) for t in flipped for e in r["idx"][t]}
    if spec["mode"] == "tc" and spec.get("capacity", -1) >= 0:
        got = host(out)
        dropped_all = [t for t in good if r["drop"][t].all()]
        assert dropped_all and all((got[t] == 0).all() for t in dropped_all)  # residual only
    _ws_ok(layer.ws)


# --------------------------------------------------------------------------
# edge cases
# --------------------------------------------------------------------------

EDGE = ROUTE_VARIANTS + [
    EC_MAX,
    # 128 to 512 rows per expert on average: the weights-as-M projections
    # (exact token counts, chunks of at most 256 tokens per tile; the SwiGLU
    # up projection with two MMA issuers when h is a multiple of 256, the
    # down projection on two tile streams)
    wl.TC_DROPLESS.replace(name="tc-swap-swiglu-top4of16", n=1024, d=256, E=16, K=4, h=256),
    wl.TC_DROPLESS.replace(name="tc-swap-gelu-shared-top2of8", n=600, d=256, E=8, K=2, h=256,
                           act="gelu", n_shared=1),
    wl.TC_DROPLESS.replace(name="tc-swap-chunks-top1of4", n=2048, d=256, E=4, K=1, h=128),
    wl.TC_SIGMOID_GROUPED.replace(name="tc-swap-sigmoid-grouped-shared-top8of64", n=2048,
                                  d=256, E=64, h=128, bias_steps=0),
    # the weights-as-M down projection over two 256-unit hidden tiles of the
    # up projection, the DeepSeek-V3 routing, a shared expert
    wl.TC_SIGMOID_GROUPED.replace(name="tc-swap-grouped-shared-top8of64-h512", n=2048,
                                  d=256, E=64, h=512, bias_steps=0),
    # ~500 tokens per expert: two token chunks each in the down projection, a
    # ragged batch, a shared expert over 1000 tokens (four chunks)
    wl.TC_DROPLESS.replace(name="tc-swap-chunks-top4of8-shared1-n1000", n=1000, d=256, E=8,
                           K=4, h=256, n_shared=1),
    # a quota of three 128-row blocks per expert: CTA pairs, the second CTA of
    # an expert's last pair repeats its block and stores nothing
    wl.EC_BF16.replace(name="ec-k384-odd-blocks", n=768, d=128, E=8, h=128, c=4.0),
    # about 275 rows per expert, ragged: CTA pairs, with odd 128-row blocks
    wl.TC_DROPLESS.replace(name="tc-pair-ragged-top2of8", n=1100, d=128, E=8, K=2, h=192),
    # decoding: a handful of tokens, most experts idle, a shared expert over
    # fewer rows than one 128-row tile
    wl.TC_SIGMOID_GROUPED.replace(name="tc-decode-n16-top8of256-shared1", n=16, d=256, E=256,
                                  h=128, bias_steps=0),
    wl.TC_DROPLESS.replace(name="tc-all-experts-k8of8", n=200, d=128, E=8, K=8, h=128),
    wl.TC_DROPLESS.replace(name="tc-single-expert", n=130, d=64, E=1, K=1, h=64),
    wl.TC_DROPLESS.replace(name="tc-one-token", n=1, d=128, E=16, K=2, h=192),
    wl.TC_TOP2_CAP.replace(name="tc-capacity-1", n=64, d=64, E=8, h=64,
                           capacity_factor=0.125, logit_skew_var=0.0),
    wl.EC_BF16.replace(name="ec-k-equals-n", n=256, d=128, E=4, h=128, c=4.0),
    wl.EC_BF16.replace(name="ec-k1", n=300, d=64, E=16, h=64, c=0.06),
    wl.EC_FP32.replace(name="ec-fp32-ragged", n=200, d=40, E=5, h=24, c=1.5),
    wl.TC_SIGMOID_GROUPED.replace(name="tc-grouped-keep-all", n=260, d=128, E=32, h=64,
                                  topk_groups=8, bias_steps=0),
    wl.TC_SIGMOID_GROUPED.replace(name="tc-grouped-f32-relu", n=150, d=64, E=64, h=32,
                                  dtype="f32", act="relu", n_shared=2, bias_steps=0),
]


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
def test_edge_cases(w):
    test_layer_small(w)
    _gathered_vs_unfused(w)


# rows longer than one 16 KB staging unit: the staged gather (K >= 4) copies
# them in two segments
LONG_ROWS = wl.TC_DROPLESS.replace(name="tc-top4of16-long-rows-d12352", n=300, d=12352, E=16,
                                   K=4, h=64)


@pytest.mark.parametrize("w", wl.SMALL + EDGE + [LONG_ROWS] + wl.FULL, ids=lambda w: w.name)
def test_dispatch_exact_copy(w):
    """The gather copies each token's row, byte for byte, to exactly the rows
    row_token names, and leaves every other row of X_perm untouched."""
    inp = wl.make_inputs(w, DEV, experts=False)
    cfg = moe.config(w)
    sz = moe.sizes(cfg)
    rb = moe.RouteBuffers(cfg, DEV, logits=False)
    ws = moe.workspace(cfg, DEV, layer=False)
    moe.moe_route(cfg, inp["X"], inp["Wg"], inp["logit_bias"], inp["sel_bias"], rb, ws)
    X_perm = torch.full((sz.rows, w.d), 12352.0, dtype=w.torch_dtype, device=DEV)
    moe.moe_dispatch(cfg, inp["X"], rb, X_perm)
    torch.cuda.synchronize()
    used = int(rb.offsets[-1])
    rt = rb.row_token[:used]
    real = rt >= 0
    assert torch.equal(X_perm[:used][real], inp["X"][rt[real].long()])
    assert bool((X_perm[:used][~real] == 12352.0).all())
    assert bool((X_perm[used:] == 12352.0).all())
    _ws_ok(ws)


def test_dispatch_rejects_misaligned_rows():
    w = wl.SMALL[1]
    inp = wl.make_inputs(w, DEV, experts=False)
    cfg = moe.config(w)
    sz = moe.sizes(cfg)
    rb = moe.RouteBuffers(cfg, DEV, logits=False)
    ws = moe.workspace(cfg, DEV, layer=False)
    moe.moe_route(cfg, inp["X"], inp["Wg"], None, None, rb, ws)
    buf = torch.empty(sz.rows * w.d + 8, dtype=w.torch_dtype, device=DEV)
    X_perm = buf[1:1 + sz.rows * w.d].view(sz.rows, w.d)  # 2 bytes off a 16-byte boundary
    with pytest.raises(moe.MoeError) as e:
        moe.moe_dispatch(cfg, inp["X"], rb, X_perm)
    assert e.value.status == moe.MOE_ERR_INVALID_ARG
    _ws_ok(ws)


def test_capacity_one_all_equal_scores():
    w = next(x for x in EDGE if x.name == "tc-capacity-1")
    cfg = moe.config(w)
    assert moe.sizes(cfg).capacity == 1
    S = torch.full((w.n, w.E), 0.125)
    rb = moe.RouteBuffers(cfg, DEV, logits=False)
    ws = moe.workspace(cfg, DEV, layer=False)
    moe.moe_route_from_scores(cfg, S.to(DEV), None, rb, ws)
    torch.cuda.synchronize()
    # ties -> experts 0 and 1 for every token; only token 0 fits
    assert (rb.idx.cpu()[:, 0] == 0).all() and (rb.idx.cpu()[:, 1] == 1).all()
    assert rb.counts.cpu().tolist() == [1, 1, 0, 0, 0, 0, 0, 0]
    drop = rb.drop.cpu()
    assert drop[0].sum() == 0 and (drop[1:] == 1).all()
    spec = oracle.spec_of(w)
    check_routing_exact(spec, oracle.route(spec, S.numpy()), rb, w.n, w.E, weights_rtol(spec))


# --------------------------------------------------------------------------
# the combine fused into the down projection (moe_expert_ffn_combined)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("w", wl.SMALL[1:] + [wl.TC_DROPLESS], ids=lambda w: w.name)
@pytest.mark.parametrize("gathered", [False, True], ids=["x_perm", "gathered"])
def test_fused_combine(w, gathered):
    """out from the gate-scaled scatter-add in the down projection's epilogue
    against the oracle (bf16 bar on the tokens whose routing agrees) and
    against the unfused layer: the only differences are the fp32 reduction
    order and Y not being rounded to bf16 first."""
    inp = wl.make_inputs(w, DEV)
    layer = moe.Layer(w, inp, DEV)
    ref_out = layer.forward().clone()
    cfg, rb = layer.cfg, layer.route
    sz = moe.sizes(cfg)
    X_perm = None
    if not gathered:
        X_perm = torch.empty((sz.rows, w.d), dtype=w.torch_dtype, device=DEV)
        moe.moe_dispatch(cfg, inp["X"], rb, X_perm)
    H = torch.empty((sz.rows, w.h), dtype=w.torch_dtype, device=DEV)
    acc = torch.empty((w.n, w.d), dtype=torch.float32, device=DEV)
    row_gate = torch.empty(max(sz.rows, 1), dtype=torch.float32, device=DEV)
    out = torch.empty((w.n, w.d), dtype=w.torch_dtype, device=DEV)
    moe.moe_expert_ffn_combined(cfg, inp["X"], X_perm, rb, inp["W1"], inp.get("W3"), inp["W2"],
                                inp.get("sW1"), inp.get("sW3"), inp.get("sW2"), H, acc, row_gate,
                                out, layer.ws)
    torch.cuda.synchronize()
    _ws_ok(layer.ws)
    got = host(out).astype(np.float64)
    unfused = host(ref_out).astype(np.float64)
    rel = np.linalg.norm(got - unfused) / np.linalg.norm(unfused)
    assert rel < 5e-3, rel
    if w.n <= 2048:
        spec, logits, S, lse, r = _oracle_from_x(w, inp)
        bad = explained_routing_diff(spec, r, layer.route, S, host(inp.get("sel_bias")))
        ref, terms = oracle.layer_forward(spec, host(inp["X"]), r, expert_weights_from(inp),
                                          expert_weights_from(inp, "s") if w.n_shared else None,
                                          absum=True)
        keep = np.array([t not in bad for t in range(w.n)])
        # the fused epilogue adds each gate-scaled row unrounded (no bf16 Y)
        # in a varying order: one bf16 rounding fewer than the oracle's
        compare_out(spec["store"], got[keep], ref[keep], w.name, absum=terms[keep])
