"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test names the passage it checks. None of these re-types an oracle
formula and compares it with itself: they use the pages' worked numbers,
brute-force enumeration, closed forms, invariants and library special cases.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy import special

import oracle
from expert_dispatch_gemm_b200 import workloads as wl
from tests.conftest import GOLDEN


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# expert-choice quota ("Who picks whom"; "A worked example")
# --------------------------------------------------------------------------

def test_ec_quota_worked_examples():
    for case in _load("ec_quota_worked_examples.json")["cases"]:
        k = oracle.ec_quota(case["n"], case["E"], case["c"])
        assert k == case["k"]
        assert case["E"] * k == case["total"] == case["c"] * case["n"]


@pytest.mark.parametrize("n,E,c", [(1024, 8, 2), (512, 8, 2), (640, 16, 2)])
def test_ec_every_expert_holds_exactly_k_distinct(n, E, c):
    S = wl.random_scores(n, E, seed=3).numpy()
    k = oracle.ec_quota(n, E, c)
    I, G = oracle.select_ec(S, k)
    assert I.shape == (E, k)
    for e in range(E):
        assert len(set(I[e].tolist())) == k
        np.testing.assert_array_equal(G[e], S[I[e], e])
    hist = oracle.ec_histogram(I, n)
    assert hist.sum() == n
    assert int((np.arange(E + 1) * hist).sum()) == E * k == int(c * n)


# --------------------------------------------------------------------------
# top-k: brute force on tiny inputs, with ties (strict order: key desc,
# index asc)
# --------------------------------------------------------------------------

def _brute_topk(keys, k):
    """Lexicographically smallest index set among the optimal k-subsets."""
    m = len(keys)
    best = None
    for A in itertools.combinations(range(m), k):
        inside = min(keys[i] for i in A)
        outside = [keys[j] for j in range(m) if j not in A]
        if outside and inside < max(outside):
            continue
        if best is None or A < best:
            best = A
    return best


def _check_sorted(keys, order):
    for a, b in zip(order, order[1:]):
        assert keys[a] > keys[b] or (keys[a] == keys[b] and a < b)


@pytest.mark.parametrize("seed", range(12))
def test_tc_topk_matches_brute_force(seed):
    levels = 3 if seed % 2 else 1000
    n, E = 7, 6
    S = wl.tie_heavy_scores(n, E, levels, seed).numpy()
    for K in (1, 2, 3, 6):
        idx, _ = oracle.select_tc(S, K)
        for t in range(n):
            keys = S[t].tolist()
            assert tuple(sorted(idx[t].tolist())) == _brute_topk(keys, K)
            _check_sorted(keys, idx[t].tolist())
            assert len(set(idx[t].tolist())) == K  # exactly K distinct experts


@pytest.mark.parametrize("seed", range(8))
def test_ec_topk_matches_brute_force(seed):
    levels = 2 if seed % 2 else 1000
    n, E = 9, 4
    S = wl.tie_heavy_scores(n, E, levels, seed).numpy()
    for k in (1, 3, 5, 9):
        I, _ = oracle.select_ec(S, k)
        for e in range(E):
            keys = S[:, e].tolist()
            assert tuple(sorted(I[e].tolist())) == _brute_topk(keys, k)
            _check_sorted(keys, I[e].tolist())


def test_all_equal_keys_pick_lowest_indices():
    S = np.full((5, 8), 0.125, np.float32)
    idx, _ = oracle.select_tc(S, 3)
    assert (idx == np.array([0, 1, 2])).all()
    I, _ = oracle.select_ec(S, 2)
    assert (I == np.array([0, 1])).all()


def test_negative_zero_ties_with_positive_zero():
    S = np.array([[-0.0, 0.0, 0.0, -1.0]], np.float32)
    idx, _ = oracle.select_tc(S, 2)
    assert idx.tolist() == [[0, 1]]


# --------------------------------------------------------------------------
# group-limited selection ("5. Group-limited and node-limited routing")
# --------------------------------------------------------------------------

def test_group_limited_by_construction():
    # 8 groups of 4; the single largest key sits in group 0, whose second key
    # is tiny, so group 0 loses to four groups with two medium keys each.
    E, G = 32, 8
    keys = np.full((1, E), 0.01, np.float32)
    keys[0, 0] = 0.9            # group 0: 0.9 + 0.01 = 0.91
    for g in (1, 3, 5, 7):      # each: 0.5 + 0.5 = 1.0
        keys[0, 4 * g] = 0.5
        keys[0, 4 * g + 1] = 0.5
    idx, _ = oracle.select_tc(keys, 8, n_groups=G, topk_groups=4, group_topn=2)
    assert 0 not in idx[0].tolist()
    assert sorted(idx[0].tolist()) == [4, 5, 12, 13, 20, 21, 28, 29]
    # without grouping the largest key wins
    idx1, _ = oracle.select_tc(keys, 8)
    assert idx1[0, 0] == 0


def _brute_group_limited(keys, K, n_groups, keep, topn):
    E = len(keys)
    gs = E // n_groups
    scores = []
    for g in range(n_groups):
        top = sorted(keys[g * gs:(g + 1) * gs], reverse=True)[:topn]
        acc = np.float32(0.0)
        for v in top:
            acc = np.float32(acc + np.float32(v))
        scores.append(float(acc))
    groups = _brute_topk(scores, keep)
    allowed = [e for g in groups for e in range(g * gs, (g + 1) * gs)]
    sub = _brute_topk([keys[e] for e in allowed], K)
    return tuple(sorted(allowed[i] for i in sub))


@pytest.mark.parametrize("seed", range(10))
def test_group_limited_matches_brute_force(seed):
    levels = 3 if seed % 2 else 1000
    n, E = 6, 8
    S = wl.tie_heavy_scores(n, E, levels, seed).numpy()
    for (G, keep, topn, K) in [(4, 2, 2, 3), (4, 2, 1, 2), (2, 1, 2, 4), (4, 3, 2, 5)]:
        idx, _ = oracle.select_tc(S, K, n_groups=G, topk_groups=keep, group_topn=topn)
        for t in range(n):
            assert tuple(sorted(idx[t].tolist())) == _brute_group_limited(
                S[t].tolist(), K, G, keep, topn)
            _check_sorted(S[t].tolist(), idx[t].tolist())


def test_one_group_or_all_groups_reduce_to_plain_topk():
    S = wl.random_scores(50, 32, seed=4).numpy()
    plain, _ = oracle.select_tc(S, 8)
    one, _ = oracle.select_tc(S, 8, n_groups=1)
    allg, _ = oracle.select_tc(S, 8, n_groups=8, topk_groups=8, group_topn=2)
    np.testing.assert_array_equal(plain, one)
    np.testing.assert_array_equal(plain, allg)


def test_groups_larger_than_1024_experts():
    """Groups of 1,280 experts (no fixed-size buffer in the C entry): keeping
    both groups reduces to plain top-K, and keeping one group takes every
    pick from the group whose two largest keys sum highest."""
    E, G, K = 2560, 2, 8
    S = wl.random_scores(4, E, seed=9).numpy()
    plain, _ = oracle.select_tc(S, K)
    both, _ = oracle.select_tc(S, K, n_groups=G, topk_groups=2, group_topn=2)
    np.testing.assert_array_equal(plain, both)
    S[:, 1280 + 7] = 2.0       # group 1: the two largest keys sum above 2
    S[:, 1280 + 1000] = 1.5
    S[:, 3] = 2.5              # group 0 holds the largest key, but its two sum below 3.5
    one, _ = oracle.select_tc(S, K, n_groups=G, topk_groups=1, group_topn=2)
    assert (one >= 1280).all()
    assert (one[:, 0] == 1280 + 7).all() and (one[:, 1] == 1280 + 1000).all()


# --------------------------------------------------------------------------
# capacity and overflow ("Dropped tokens flow in opposite directions";
# "2. Top-1 switch routing with a capacity factor")
# --------------------------------------------------------------------------

def test_capacity_values():
    for case in _load("capacity_buffer.json")["cases"]:
        assert oracle.capacity_of(case["n"], case["E"], case["capacity_factor"]) == \
            case["capacity"]


def _brute_positions(idx, E):
    n, K = idx.shape
    pos = np.zeros_like(idx)
    for t in range(n):
        for j in range(K):
            e = idx[t, j]
            pos[t, j] = int((idx[:t] == e).sum())
    return pos


@pytest.mark.parametrize("cap", [-1, 0, 3, 10, 1000])
def test_capacity_closed_forms(cap):
    n, E, K = 60, 6, 2
    S = wl.random_scores(n, E, seed=9).numpy() ** 3  # lumpy preferences
    idx, _ = oracle.select_tc(S, K)
    drop, load, kept, pos = oracle.apply_capacity(idx, E, cap)
    arrival = _brute_positions(idx, E)  # tokens before t that picked e
    np.testing.assert_array_equal(load, np.bincount(idx.ravel(), minlength=E))
    eff = n * K if cap < 0 else cap
    np.testing.assert_array_equal(kept, np.minimum(load, eff))
    assert kept.sum() <= E * eff
    np.testing.assert_array_equal(drop.astype(bool), arrival >= eff)
    np.testing.assert_array_equal(pos, np.where(arrival < eff, arrival, -1))
    if cap < 0:
        assert drop.sum() == 0 and load.sum() == n * K


def test_capacity_all_equal_scores_worked_shape():
    # n = 8192, E = 8, capacity factor 1.25 -> 1280; with all scores equal the
    # strict order sends every token to experts 0 and 1, which keep tokens
    # 0..1279 and drop the rest.
    n, E, K = 8192, 8, 2
    cap = oracle.capacity_of(n, E, 1.25)
    assert cap == 1280
    S = np.full((n, E), 1.0 / E, np.float32)
    idx, _ = oracle.select_tc(S, K)
    drop, load, kept, pos = oracle.apply_capacity(idx, E, cap)
    assert (idx[:, 0] == 0).all() and (idx[:, 1] == 1).all()
    assert kept.tolist() == [1280, 1280, 0, 0, 0, 0, 0, 0]
    assert (drop[:1280] == 0).all() and (drop[1280:] == 1).all()


# --------------------------------------------------------------------------
# mixing weights ("1. Softmax top-k token choice"; "4. Sigmoid gating with
# aux-loss-free bias")
# --------------------------------------------------------------------------

def test_softmax_over_kept_logits_identity():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((40, 16)).astype(np.float32)
    Wg = (rng.standard_normal((16, 8)) / 4).astype(np.float32)
    logits, S, _ = oracle.router(X, Wg)
    idx, w = oracle.select_tc(S, 2, weights=oracle.W_NORMALIZED)
    kept = np.take_along_axis(logits.astype(np.float64), idx, 1)
    ref = special.softmax(kept, axis=1)
    np.testing.assert_allclose(w, ref, rtol=2e-6, atol=0)


def test_weights_of_a_given_selection():
    """weights_tc on select_tc's own selection returns select_tc's weights
    bit for bit (raw and normalised, with a selection bias and groups), and
    on any other selection the softmax-over-kept identity holds: normalised
    weights of softmax scores equal a softmax over the chosen logits."""
    rng = np.random.default_rng(5)
    X = rng.standard_normal((50, 24)).astype(np.float32)
    Wg = (rng.standard_normal((24, 32)) / 5).astype(np.float32)
    logits, S, _ = oracle.router(X, Wg)
    _, s, _ = oracle.router(X, Wg, score=oracle.SIGMOID)
    bias = (rng.standard_normal(32) * 0.1).astype(np.float32)
    for scores, b, G in ((S, None, 1), (s, bias, 4), (s, None, 8)):
        for mode in (oracle.W_RAW, oracle.W_NORMALIZED):
            idx, w = oracle.select_tc(scores, 4, b, n_groups=G, topk_groups=min(2, G),
                                      group_topn=2 if G > 1 else 1, weights=mode)
            np.testing.assert_array_equal(oracle.weights_tc(scores, idx, mode), w)
    other = np.stack([rng.permutation(32)[:3] for _ in range(50)]).astype(np.int32)
    w = oracle.weights_tc(S, other, oracle.W_NORMALIZED)
    ref = special.softmax(np.take_along_axis(logits.astype(np.float64), other, 1), axis=1)
    np.testing.assert_allclose(w, ref, rtol=2e-6, atol=0)
    raw = oracle.weights_tc(S, other, oracle.W_RAW)
    np.testing.assert_array_equal(raw, np.take_along_axis(S, other, 1))


def test_selection_only_bias():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((64, 32)).astype(np.float32)
    Wg = (rng.standard_normal((32, 16)) / np.sqrt(32)).astype(np.float32)
    _, s, _ = oracle.router(X, Wg, score=oracle.SIGMOID)
    K = 4
    plain_idx, plain_w = oracle.select_tc(s, K, weights=oracle.W_NORMALIZED)
    zero_idx, zero_w = oracle.select_tc(s, K, np.zeros(16, np.float32),
                                        weights=oracle.W_NORMALIZED)
    np.testing.assert_array_equal(plain_idx, zero_idx)
    np.testing.assert_array_equal(plain_w, zero_w)
    bias = np.zeros(16, np.float32)
    bias[5] = 10.0
    b_idx, b_w = oracle.select_tc(s, K, bias, weights=oracle.W_NORMALIZED)
    assert (b_idx[:, 0] == 5).all()  # the bias forces expert 5 into every row
    # the weights come from the raw sigmoid scores, never from score + bias
    for t in range(64):
        sel = b_idx[t]
        raw = s[t, sel].astype(np.float64)
        np.testing.assert_allclose(b_w[t], raw / raw.sum(), rtol=2e-7)
        # ratios of weights are ratios of raw scores
        assert abs(b_w[t, 0] / b_w[t, 1] - raw[0] / raw[1]) < 1e-5 * raw[0] / raw[1]
        if set(sel.tolist()) == set(plain_idx[t].tolist()):
            m = {e: w for e, w in zip(plain_idx[t].tolist(), plain_w[t].tolist())}
            for e, w in zip(sel.tolist(), b_w[t].tolist()):
                assert w == m[e]
    assert np.allclose(b_w.sum(1), 1.0, atol=1e-6)


# --------------------------------------------------------------------------
# router ("The transposed selection": S = softmax(X W_g), W_g: [d, E];
# sigmoid scores; logsumexp for the z-loss)
# --------------------------------------------------------------------------

def test_router_against_library():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((33, 48)).astype(np.float32)
    Wg = (rng.standard_normal((48, 12)) / np.sqrt(48)).astype(np.float32)
    b = rng.standard_normal(12).astype(np.float32)
    logits, S, lse = oracle.router(X, Wg, b)
    ref = X.astype(np.float64) @ Wg.astype(np.float64) + b
    np.testing.assert_allclose(logits, ref, rtol=1e-6, atol=1e-6)
    L64 = logits.astype(np.float64)
    np.testing.assert_allclose(S, special.softmax(L64, axis=1), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(lse, special.logsumexp(L64, axis=1), rtol=1e-12)
    np.testing.assert_allclose(S.sum(1), 1.0, atol=1e-6)
    _, s, _ = oracle.router(X, Wg, b, score=oracle.SIGMOID)
    np.testing.assert_allclose(s, special.expit(L64), rtol=1e-6, atol=1e-9)


def test_sqrtsoftplus_closed_forms():
    """sqrt(softplus(l)) on logits fixed through the bias (X = 0): l = 0 gives
    sqrt(ln 2); l = 100 gives 10 (ln(1 + e^-100) is below double precision at
    100); l = -30 gives e^-15 to first order; l = 2 gives sqrt(2 + ln(1 +
    e^-2)) = sqrt(ln(1 + e^2)); the score grows with l."""
    b = np.array([0.0, 100.0, -30.0, 2.0, -1.0, 1.0], np.float32)
    X = np.zeros((3, 4), np.float32)
    Wg = np.ones((4, b.size), np.float32)
    _, s, _ = oracle.router(X, Wg, b, score=oracle.SQRTSOFTPLUS)
    assert np.allclose(s[:, 0], np.sqrt(np.log(2.0)), rtol=1e-7)
    assert np.all(s[:, 1] == np.float32(10.0))
    assert np.allclose(s[:, 2], np.exp(-15.0), rtol=1e-6)
    assert np.allclose(s[:, 3], np.sqrt(np.log1p(np.exp(2.0))), rtol=1e-7)
    order = np.argsort(b)
    assert np.all(np.diff(s[0, order].astype(np.float64)) > 0)


def test_monotone_scores_select_the_same_experts():
    """Without a selection bias or groups, top-K of any score that grows with
    the logit picks the same experts in the same order: softmax, sigmoid and
    sqrt(softplus) agree on every token (distinct random logits)."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((64, 32)).astype(np.float32)
    Wg = (rng.standard_normal((32, 16)) / np.sqrt(32)).astype(np.float32)
    picks = []
    for score in (oracle.SOFTMAX, oracle.SIGMOID, oracle.SQRTSOFTPLUS):
        _, s, _ = oracle.router(X, Wg, score=score)
        idx, _ = oracle.select_tc(s, 4)
        picks.append(idx)
    np.testing.assert_array_equal(picks[0], picks[1])
    np.testing.assert_array_equal(picks[0], picks[2])


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------

def test_round_bf16_against_torch_and_ties():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(v.astype(np.float64)), ref)
    one = 1.0
    assert oracle.round_bf16([one + 2 ** -8])[0] == 1.0              # tie -> even
    assert oracle.round_bf16([one + 3 * 2 ** -8])[0] == 1.0 + 2 ** -6  # tie -> even
    # just above a tie: direct rounding goes up, rounding via fp32 would not
    assert oracle.round_bf16([one + 2 ** -8 + 2 ** -30])[0] == 1.0 + 2 ** -7
    assert oracle.round_bf16([3.5e38])[0] == np.inf


# --------------------------------------------------------------------------
# expert FFN against torch float64 (library special case)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("act", [oracle.RELU, oracle.GELU, oracle.SWIGLU])
def test_expert_ffn_against_torch(act):
    g = torch.Generator().manual_seed(5)
    m, d, h = 7, 24, 40
    X = torch.randn(m, d, generator=g, dtype=torch.float64)
    W1 = torch.randn(h, d, generator=g, dtype=torch.float64) / 5
    W3 = torch.randn(h, d, generator=g, dtype=torch.float64) / 5
    W2 = torch.randn(d, h, generator=g, dtype=torch.float64) / 6
    X, W1, W3, W2 = (t.float().double() for t in (X, W1, W3, W2))
    u = X @ W1.T
    if act == oracle.RELU:
        H = torch.relu(u)
    elif act == oracle.GELU:
        H = torch.nn.functional.gelu(u, approximate="none")
    else:
        H = torch.nn.functional.silu(u) * (X @ W3.T)
    # fp32 storage
    Hs = H.float().double()
    ref = (Hs @ W2.T).float().numpy()
    got = oracle.expert_ffn(X.float().numpy(), W1.float().numpy(),
                            W3.float().numpy() if act == oracle.SWIGLU else None,
                            W2.float().numpy(), act, oracle.STORE_F32)
    np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-7)
    # bf16 storage of the hidden activations and of Y
    Hb = torch.from_numpy(oracle.round_bf16(H.numpy())).double()
    refb = oracle.round_bf16((Hb @ W2.T).numpy())
    gotb = oracle.expert_ffn(X.float().numpy(), W1.float().numpy(),
                             W3.float().numpy() if act == oracle.SWIGLU else None,
                             W2.float().numpy(), act, oracle.STORE_BF16)
    np.testing.assert_allclose(gotb, refb, rtol=2 ** -7, atol=1e-30)


# --------------------------------------------------------------------------
# the whole layer: the pages' one-hot formulation, closed forms, invariants
# --------------------------------------------------------------------------

def _dense_experts(E, h, d, seed, identical=False, swiglu=False):
    g = torch.Generator().manual_seed(seed)
    W1 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).numpy()
    W3 = (torch.randn(E, h, d, generator=g) / math.sqrt(d)).numpy() if swiglu else None
    W2 = (torch.randn(E, d, h, generator=g) / math.sqrt(h)).numpy()
    if identical:
        W1 = np.repeat(W1[:1], E, 0)
        W2 = np.repeat(W2[:1], E, 0)
        W3 = None if W3 is None else np.repeat(W3[:1], E, 0)
    return W1, W3, W2


def test_ec_layer_matches_onehot_formulation():
    # X_in[e] = P[e] X with P = onehot(I) [E,k,n]; Y[e] = G[e] * FFN_e(X_in[e]);
    # out = scatter_add(Y, I) ("The math: a gating matrix and top-k over tokens")
    n, d, E, h, c = 40, 16, 4, 24, 2
    rng = np.random.default_rng(6)
    X = rng.standard_normal((n, d)).astype(np.float32)
    Wg = (rng.standard_normal((d, E)) / 4).astype(np.float32)
    W1, _, W2 = _dense_experts(E, h, d, 7)
    _, S, lse = oracle.router(X, Wg)
    k = oracle.ec_quota(n, E, c)
    spec = dict(mode="ec", k=k, act=oracle.RELU, store=oracle.STORE_F32)
    r = oracle.route(spec, S, lse)
    got = oracle.layer_forward(spec, X, r, lambda e: (W1[e], None, W2[e]))
    I, G = r["I"], r["G"]
    P = np.zeros((E, k, n))
    for e in range(E):
        P[e, np.arange(k), I[e]] = 1.0
    X_in = P @ X.astype(np.float64)                       # [E,k,d]
    Y = np.stack([G[e][:, None] * (np.maximum(X_in[e] @ W1[e].T.astype(np.float64), 0)
                                   @ W2[e].T.astype(np.float64)) for e in range(E)])
    ref = np.einsum("ekn,ekd->nd", P, Y)                  # scatter_add back to [n, d]
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)
    # a token picked by no expert gets nothing ("Variable tokens-per-token")
    unpicked = np.setdiff1d(np.arange(n), I.ravel())
    assert (got[unpicked] == 0).all()


def test_ec_every_expert_takes_every_token_identity():
    # k = n (c = E): every expert takes every token; with identical experts
    # out = FFN(x) * sum_e S[t,e] = FFN(x)
    n, d, E, h = 24, 16, 4, 20
    rng = np.random.default_rng(8)
    X = rng.standard_normal((n, d)).astype(np.float32)
    Wg = (rng.standard_normal((d, E)) / 4).astype(np.float32)
    W1, _, W2 = _dense_experts(E, h, d, 9, identical=True)
    _, S, lse = oracle.router(X, Wg)
    spec = dict(mode="ec", k=oracle.ec_quota(n, E, E), act=oracle.GELU,
                store=oracle.STORE_F32)
    r = oracle.route(spec, S, lse)
    got = oracle.layer_forward(spec, X, r, lambda e: (W1[e], None, W2[e]))
    ffn = oracle.expert_ffn(X, W1[0], None, W2[0], oracle.GELU, oracle.STORE_F32)
    np.testing.assert_allclose(got, ffn, rtol=3e-6, atol=3e-7)


def test_tc_identical_experts_normalised_weights_identity():
    n, d, E, h, K = 30, 16, 8, 20, 3
    rng = np.random.default_rng(10)
    X = rng.standard_normal((n, d)).astype(np.float32)
    Wg = (rng.standard_normal((d, E)) / 4).astype(np.float32)
    W1, W3, W2 = _dense_experts(E, h, d, 11, identical=True, swiglu=True)
    _, s, lse = oracle.router(X, Wg, score=oracle.SIGMOID)
    spec = dict(mode="tc", K=K, capacity=-1, weights=oracle.W_NORMALIZED,
                act=oracle.SWIGLU, store=oracle.STORE_F32)
    r = oracle.route(spec, s, lse)
    got = oracle.layer_forward(spec, X, r, lambda e: (W1[e], W3[e], W2[e]))
    ffn = oracle.expert_ffn(X, W1[0], W3[0], W2[0], oracle.SWIGLU, oracle.STORE_F32)
    np.testing.assert_allclose(got, ffn, rtol=3e-6, atol=3e-7)


def test_shared_expert_adds_weight_one_term():
    n, d, E, h, K = 20, 16, 8, 12, 2
    rng = np.random.default_rng(12)
    X = rng.standard_normal((n, d)).astype(np.float32)
    Wg = (rng.standard_normal((d, E)) / 4).astype(np.float32)
    W1, W3, W2 = _dense_experts(E, h, d, 13, swiglu=True)
    sW1, sW3, sW2 = _dense_experts(1, h, d, 14, swiglu=True)
    _, s, lse = oracle.router(X, Wg, score=oracle.SIGMOID)
    spec = dict(mode="tc", K=K, capacity=-1, weights=oracle.W_NORMALIZED,
                act=oracle.SWIGLU, store=oracle.STORE_F32, n_shared=1)
    r = oracle.route(spec, s, lse)
    ew = lambda e: (W1[e], W3[e], W2[e])  # noqa: E731
    with_sh = oracle.layer_forward(spec, X, r, ew, lambda i: (sW1[0], sW3[0], sW2[0]))
    without = oracle.layer_forward(dict(spec, n_shared=0), X, r, ew)
    shared = oracle.expert_ffn(X, sW1[0], sW3[0], sW2[0], oracle.SWIGLU, oracle.STORE_F32)
    np.testing.assert_allclose(with_sh, without + shared, rtol=1e-5, atol=1e-6)


def test_tc_dropless_is_per_token():
    # "Token-choice: the token picks experts": no other token's hidden state
    # enters a token's routing, so permuting the batch permutes the output
    n, d, E, h, K = 36, 16, 8, 12, 2
    rng = np.random.default_rng(15)
    X = rng.standard_normal((n, d)).astype(np.float32)
    Wg = (rng.standard_normal((d, E)) / 4).astype(np.float32)
    W1, W3, W2 = _dense_experts(E, h, d, 16, swiglu=True)
    spec = dict(mode="tc", K=K, capacity=-1, weights=oracle.W_RAW, act=oracle.SWIGLU,
                store=oracle.STORE_BF16)
    ew = lambda e: (W1[e], W3[e], W2[e])  # noqa: E731

    def run(Xp):
        _, S, lse = oracle.router(Xp, Wg)
        return oracle.layer_forward(spec, Xp, oracle.route(spec, S, lse), ew)

    perm = rng.permutation(n)
    np.testing.assert_array_equal(run(X)[perm], run(X[perm]))
    # splitting the batch does not change any token either
    np.testing.assert_array_equal(run(X)[: n // 2], run(X[: n // 2]))


def test_ec_equivariant_without_ties():
    n, E = 50, 5
    S = wl.random_scores(n, E, seed=17).numpy()
    k = 10
    I, G = oracle.select_ec(S, k)
    perm = np.random.default_rng(18).permutation(n)
    I2, G2 = oracle.select_ec(S[perm], k)
    np.testing.assert_array_equal(perm[I2], I)
    np.testing.assert_array_equal(G2, G)


# --------------------------------------------------------------------------
# aux values ("What each direction guarantees"; MaxVio in the TL;DR of
# "MoE routing strategies explained"; bias update in "4. Sigmoid gating with
# aux-loss-free bias")
# --------------------------------------------------------------------------

def test_balanced_targets_from_pages():
    g = _load("balance_targets.json")
    for case in g["cases"]:
        n, E, K = case["n"], case["E"], case["K"]
        assert n * K // E == case["target_per_expert"]
        assert case["target_per_expert"] / n == case["fraction_of_batch"]


def test_lb_loss_is_coefficient_at_perfect_balance():
    n, E, K = 64, 8, 2
    S = np.full((n, E), 1.0 / E, np.float32)
    load = np.full(E, n * K // E, np.int32)
    lse = np.zeros(n)
    lb, z, mv = oracle.aux(load, S, lse, K, lb_coef=0.01, z_coef=0.001)
    assert abs(lb - 0.01) < 1e-12
    assert mv == 0.0
    # all load on one expert while S still uniform: f = (1,0,..), lb = coef
    load2 = np.zeros(E, np.int32)
    load2[0] = n * K
    lb2, _, mv2 = oracle.aux(load2, S, lse, K)
    assert abs(lb2 - 0.01) < 1e-12 and mv2 == E - 1
    # concentrated scores and loads: the loss grows to coef * E
    S3 = np.zeros((n, E), np.float32)
    S3[:, 0] = 1.0
    lb3, _, _ = oracle.aux(load2, S3, lse, K)
    assert abs(lb3 - 0.01 * E) < 1e-12


def test_z_loss_of_zero_logits():
    n, d, E = 10, 8, 64
    _, S, lse = oracle.router(np.zeros((n, d), np.float32), np.ones((d, E), np.float32))
    np.testing.assert_allclose(lse, math.log(64), rtol=1e-15)
    _, z, _ = oracle.aux(np.full(E, 1, np.int32), S, lse, 8, z_coef=0.001)
    assert abs(z - 0.001 * math.log(64) ** 2) < 1e-15


def test_bias_update_two_expert_example():
    n, K, E = 2, 2, 2  # mean load = 2
    b = oracle.bias_update(np.array([3, 1], np.int32), n, K, 0.001, np.zeros(2, np.float32))
    assert b.tolist() == [np.float32(-0.001), np.float32(0.001)]
    b2 = oracle.bias_update(np.array([2, 2], np.int32), n, K, 0.001, b)
    np.testing.assert_array_equal(b2, b)  # sign(0) = 0
    b3 = oracle.bias_update(np.array([1, 3], np.int32), n, K, 0.001, b2)
    assert b3.tolist() == [np.float32(np.float32(-0.001) + np.float32(0.001)),
                           np.float32(np.float32(0.001) - np.float32(0.001))]


def test_ec_histogram_counts():
    I = np.array([[0, 1, 2], [1, 2, 3], [2, 3, 4]], np.int32)  # E=3, k=3, n=6
    hist = oracle.ec_histogram(I, 6)
    # token 0:1, 1:2, 2:3, 3:2, 4:1, 5:0
    assert hist.tolist() == [1, 2, 2, 1]
