"""Shared checks for the GPU parity tests: run the CUDA path through the C
ABI, run the oracle on the same seeded inputs, compare.

Nothing computed by the CUDA path is ever fed to the oracle: both sides
start from the seeded inputs (X, W_g, weights, or a seeded score matrix).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from expert_dispatch_gemm_b200 import moe

GAP_TOL = 1e-5        # a selection may differ only where the oracle's gap is below this
BF16_REL_TOL = 2e-2   # relative Frobenius error of bf16 layer outputs
F32_ABS_TOL = 1e-4    # max-abs error of fp32 layer outputs


def host(t):
    return None if t is None else t.detach().float().cpu().numpy()


def round128(x):
    return (np.asarray(x, np.int64) + 127) // 128 * 128


# --------------------------------------------------------------------------
# exact comparison of routing tensors (identical scores on both sides)
# --------------------------------------------------------------------------

def expected_layout(spec, r, n, E):
    """Offsets / row_token / per-token slot lists implied by the oracle's
    routing and the library's documented dispatched-row layout."""
    if spec["mode"] == "ec":
        k = spec["k"]
        kpad = int(round128(k))
        offsets = np.arange(E + 1, dtype=np.int64) * kpad
        row_token = np.full(E * kpad, -1, np.int64)
        lists = [[] for _ in range(n)]
        for e in range(E):
            for j in range(k):
                t = int(r["I"][e, j])
                row_token[e * kpad + j] = t
                lists[t].append((e, e * kpad + j, float(r["G"][e, j])))
        tok = [[(row, g) for (_, row, g) in sorted(l)] for l in lists]
        return offsets, row_token, tok
    idx, drop, pos, kept = r["idx"], r["drop"], r["pos"], r["kept"]
    offsets = np.concatenate([[0], np.cumsum(round128(kept))])
    row_token = np.full(int(offsets[-1]), -1, np.int64)
    tok = []
    for t in range(n):
        l = []
        for j in range(idx.shape[1]):
            if not drop[t, j]:
                e = int(idx[t, j])
                row = int(offsets[e] + pos[t, j])
                row_token[row] = t
                l.append((row, float(r["w"][t, j])))
        tok.append(l)
    return offsets, row_token, tok


def check_routing_exact(spec, r, rb: moe.RouteBuffers, n, E, weights_rtol=0.0):
    """Integer routing outputs bit-exact; gates exact (raw) or to rtol."""
    offsets, row_token, tok = expected_layout(spec, r, n, E)
    got_off = rb.offsets.cpu().numpy()
    np.testing.assert_array_equal(got_off, offsets)
    used = int(offsets[-1])
    np.testing.assert_array_equal(rb.row_token[:used].cpu().numpy(), row_token)
    tok_row = rb.tok_row.cpu().numpy()
    tok_gate = rb.tok_gate.cpu().numpy()
    for t in range(n):
        l = tok[t]
        m = len(l)
        np.testing.assert_array_equal(tok_row[t, :m], [x[0] for x in l])
        assert (tok_row[t, m:] == -1).all()
        if weights_rtol == 0.0:
            np.testing.assert_array_equal(tok_gate[t, :m], np.float32([x[1] for x in l]))
        else:
            np.testing.assert_allclose(tok_gate[t, :m], [x[1] for x in l], rtol=weights_rtol)
    if spec["mode"] == "ec":
        np.testing.assert_array_equal(rb.idx.cpu().numpy(), r["I"])
        if weights_rtol == 0.0:
            np.testing.assert_array_equal(rb.gate.cpu().numpy(), r["G"])
        else:
            np.testing.assert_allclose(rb.gate.cpu().numpy(), r["G"], rtol=weights_rtol)
        np.testing.assert_array_equal(rb.load.cpu().numpy(), r["load"])
        np.testing.assert_array_equal(rb.counts.cpu().numpy(), r["kept"])
        np.testing.assert_array_equal(rb.ec_hist.cpu().numpy(), r["hist"])
    else:
        np.testing.assert_array_equal(rb.idx.cpu().numpy(), r["idx"])
        if weights_rtol == 0.0:
            np.testing.assert_array_equal(rb.gate.cpu().numpy(), r["w"])
        else:
            np.testing.assert_allclose(rb.gate.cpu().numpy(), r["w"], rtol=weights_rtol)
        np.testing.assert_array_equal(rb.drop.cpu().numpy(), r["drop"])
        np.testing.assert_array_equal(rb.load.cpu().numpy(), r["load"])
        np.testing.assert_array_equal(rb.counts.cpu().numpy(), r["kept"])


def weights_rtol(spec):
    # normalised weights: fp32 sum and divide on the GPU vs one rounding of
    # the double quotient in the oracle -> a few ulp
    return 1e-6 if spec.get("weights") == oracle.W_NORMALIZED and spec["mode"] == "tc" else 0.0


# --------------------------------------------------------------------------
# boundary gaps (selection flips are allowed only where these are tiny)
# --------------------------------------------------------------------------

def tc_row_gap(spec, s_row, bias=None):
    keys = s_row.astype(np.float32) + (bias if bias is not None else np.float32(0))
    keys = keys.astype(np.float32)
    E = len(keys)
    K = spec["K"]
    gaps = []
    allowed = np.arange(E)
    G = spec.get("n_groups", 1)
    if G > 1:
        gs = E // G
        scores = []
        for g in range(G):
            top = np.sort(keys[g * gs:(g + 1) * gs])[::-1][:spec["group_topn"]]
            acc = np.float32(0)
            for v in top:
                acc = np.float32(acc + v)
            scores.append(float(acc))
        order = sorted(range(G), key=lambda g: (-scores[g], g))
        kg = spec["topk_groups"]
        if kg < G:
            gaps.append(scores[order[kg - 1]] - scores[order[kg]])
        allowed = np.concatenate([np.arange(g * gs, (g + 1) * gs) for g in order[:kg]])
    sub = np.sort(keys[allowed].astype(np.float64))[::-1]
    if K < len(sub):
        gaps.append(sub[K - 1] - sub[K])
    return min(gaps) if gaps else np.inf


def ec_col_gap(k, col):
    s = np.sort(col.astype(np.float64))[::-1]
    return s[k - 1] - s[k] if k < len(s) else np.inf


def explained_routing_diff(spec, r_or, rb, S_or, sel_bias=None):
    """Tokens whose routing differs between the GPU and the oracle run from
    X. Asserts every difference is a flip at a boundary gap < GAP_TOL (or,
    under a capacity, a drop caused by such a flip on the same expert)."""
    n, E = S_or.shape
    bad = set()
    if spec["mode"] == "ec":
        I_g = rb.idx.cpu().numpy()
        for e in range(E):
            a, b = set(I_g[e].tolist()), set(r_or["I"][e].tolist())
            if a != b:
                gap = ec_col_gap(spec["k"], S_or[:, e])
                assert gap < GAP_TOL, f"expert {e}: selection differs with gap {gap}"
                bad |= a ^ b
            # same set: order and gates may still differ only if scores tie
        return bad
    idx_g = rb.idx.cpu().numpy()
    flip_experts = set()
    for t in np.nonzero((idx_g != r_or["idx"]).any(1))[0]:
        if set(idx_g[t].tolist()) == set(r_or["idx"][t].tolist()):
            # order differs: only possible at exact-ish ties inside the top K
            pass
        gap = tc_row_gap(spec, S_or[t], sel_bias)
        if set(idx_g[t].tolist()) != set(r_or["idx"][t].tolist()):
            assert gap < GAP_TOL, f"token {t}: selection differs with gap {gap}"
        bad.add(int(t))
        flip_experts |= set(idx_g[t].tolist()) ^ set(r_or["idx"][t].tolist())
    if spec.get("capacity", -1) >= 0:
        drop_g = rb.drop.cpu().numpy()
        for t in np.nonzero((drop_g != r_or["drop"]).any(1))[0]:
            if int(t) in bad:
                continue
            es = set(idx_g[t][drop_g[t] != r_or["drop"][t]].tolist())
            assert es <= flip_experts, f"token {t}: drop differs without a flip"
            bad.add(int(t))
    return bad


# --------------------------------------------------------------------------
# layer outputs
# --------------------------------------------------------------------------

def expert_weights_from(inputs, prefix=""):
    W1, W3, W2 = inputs[prefix + "W1"], inputs.get(prefix + "W3"), inputs[prefix + "W2"]

    def get(e):
        return (host(W1[e]), None if W3 is None else host(W3[e]), host(W2[e]))
    return get


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (8 significant bits): 2^(e - 7) for
    |x| in [2^e, 2^(e+1)); the smallest normal spacing below that range."""
    a = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


# element-wise bound of bf16 layer outputs. Each side rounds every expert
# output Y to bf16 and then the result (R22); where the two sides' unrounded
# values straddle a rounding boundary the stored values differ by one bf16
# spacing. A flipped Y element moves the output by its gate times one spacing
# of Y (at most 2^-7 |Y|), so the bound is: two spacings of the result, plus
# 2^-7 of the sum of |gate| |Y| over the element's terms (absum, from the
# oracle), plus 0.5% of the row's rms for the fp32 / fp64 accumulation orders.
# Without absum the bound falls back to two spacings + 2% of the row's rms.
BF16_ULPS = 2.0
BF16_TERM_REL = 2.0 ** -7
BF16_ROW_RMS_TOL = 5e-3
BF16_ROW_RMS_TOL_NO_TERMS = 2e-2


def compare_out(store, got, ref, what="", absum=None, row_tol=BF16_REL_TOL):
    """Layer outputs (rows = tokens) against the oracle's, element by element.

    fp32: max-abs error <= 1e-4. bf16, three checks that must all hold:
      * every row: ||got_t - ref_t|| / ||ref_t|| <= 2e-2 (a row the oracle
        leaves at zero, a token with no kept expert, must be exactly zero);
      * every element: |got - ref| <= 2 bf16 spacings of ref + 2^-7 absum +
        0.5% rms(ref_t) (absum: the oracle's sum of |gate| |Y| per element),
        or 2 spacings + 2% rms(ref_t) without absum;
      * the whole block: ||got - ref||_F / ||ref||_F <= 2e-2.
    Returns the worst per-row relative error."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if store == oracle.STORE_F32:
        err = np.abs(got - ref).max() if got.size else 0.0
        assert err <= F32_ABS_TOL, f"{what} max-abs error {err}"
        return err
    if got.size == 0:
        return 0.0
    g2 = got.reshape(got.shape[0], -1)
    r2 = ref.reshape(ref.shape[0], -1)
    diff = np.abs(g2 - r2)
    norms = np.linalg.norm(r2, axis=1)
    zero = norms == 0
    assert not diff[zero].any(), f"{what}: rows the oracle leaves at zero are not zero"
    rel_rows = np.linalg.norm(g2 - r2, axis=1)[~zero] / norms[~zero]
    worst = float(rel_rows.max()) if rel_rows.size else 0.0
    assert worst <= row_tol, (f"{what}: row {int(np.nonzero(~zero)[0][rel_rows.argmax()])} "
                              f"relative error {worst:.4g}")
    rms = norms / np.sqrt(r2.shape[1])
    if absum is None:
        bound = BF16_ULPS * bf16_ulp(r2) + BF16_ROW_RMS_TOL_NO_TERMS * rms[:, None]
    else:
        a2 = np.asarray(absum, np.float64).reshape(r2.shape)
        bound = BF16_ULPS * bf16_ulp(r2) + BF16_TERM_REL * a2 + BF16_ROW_RMS_TOL * rms[:, None]
    over = diff > bound
    if over.any():
        i, j = np.argwhere(over)[0]
        raise AssertionError(
            f"{what}: {int(over.sum())} elements beyond the element-wise bound; first at "
            f"[{i}, {j}]: got {g2[i, j]:.6g} ref {r2[i, j]:.6g} (row rms {rms[i]:.4g}, "
            f"bound {bound[i, j]:.4g})")
    den = np.linalg.norm(r2)
    err = np.linalg.norm(g2 - r2) / (den if den > 0 else 1.0)
    assert err <= BF16_REL_TOL, f"{what} relative error {err}"
    return worst


# --------------------------------------------------------------------------
# sampling at full size, and the oracle on the GPU's selection
# --------------------------------------------------------------------------

def covering_tokens(spec, r, n, E, seed, extra=8):
    """Tokens whose outputs, together, exercise every expert's GEMM tiles:
      * for every expert, the token in its last kept row (the expert's last
        128-row block, which a CTA pair repeats when the block count is odd,
        and the tail of its last weights-as-M token chunk);
      * greedily, tokens until every expert with a kept row is covered;
      * `extra` seeded random tokens; under a capacity, tokens with a drop
        and with every choice dropped; under expert choice, tokens with no
        expert and the token with the most.
    Returns a sorted list of token ids."""
    rng = np.random.default_rng(seed)
    rows = {e: [] for e in range(E)}        # kept tokens of each expert, row order
    if spec["mode"] == "ec":
        for e in range(E):
            rows[e] = [int(t) for t in r["I"][e]]
    else:
        idx, drop = r["idx"], r["drop"]
        for t in range(n):
            for j in range(idx.shape[1]):
                if not drop[t, j]:
                    rows[int(idx[t, j])].append(t)
    picks = {l[-1] for l in rows.values() if l}
    experts_of = {}
    for e, l in rows.items():
        for t in l:
            experts_of.setdefault(t, set()).add(e)
    covered = set()
    for t in picks:
        covered |= experts_of.get(t, set())
    need = {e for e, l in rows.items() if l} - covered
    while need:
        t = max(experts_of, key=lambda u: (len(experts_of[u] & need), -u))
        picks.add(t)
        need -= experts_of[t]
    picks |= set(rng.choice(n, size=min(extra, n), replace=False).tolist())
    if spec["mode"] == "tc" and spec.get("capacity", -1) >= 0:
        picks |= set(np.nonzero(r["drop"].any(1))[0][:2].tolist())
        picks |= set(np.nonzero(r["drop"].all(1))[0][:1].tolist())
    if spec["mode"] == "ec":
        per_token = np.bincount(r["I"].ravel(), minlength=n)
        picks |= set(np.nonzero(per_token == 0)[0][:2].tolist())
        picks |= set(np.argsort(-per_token, kind="stable")[:1].tolist())
    return sorted(int(t) for t in picks)


def routing_on_gpu_selection(spec, S_or, rb: moe.RouteBuffers):
    """The oracle's routing dict with the GPU's selection (and, under a
    capacity, its drops) in place of the oracle's own, the weights computed
    by the oracle from its own scores (R24: where a boundary gap below
    GAP_TOL lets the two sides select differently, the outputs are compared
    on the GPU's selection)."""
    if spec["mode"] == "ec":
        I = rb.idx.cpu().numpy().astype(np.int32)
        E = I.shape[0]
        G = np.stack([S_or[I[e], e] for e in range(E)]).astype(np.float32)
        return {"I": I, "G": G}
    idx = rb.idx.cpu().numpy().astype(np.int32)
    w = oracle.weights_tc(S_or, idx, spec.get("weights", oracle.W_RAW))
    return {"idx": idx, "w": w, "drop": rb.drop.cpu().numpy()}
