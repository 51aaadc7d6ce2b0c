"""Pins for the oracle's re-selection rules.

OEA ("Opportunistic Expert Activation: Batch-Aware Expert Routing for
Faster Decode Without Retraining", abstract and lay summary): checked
against a declarative characterisation that determines the result
uniquely (kept prefix, fills drawn from the union of kept sets, maximal
fill count, and every skipped candidate ranked below every fill), plus the
closed forms k0 = k (standard top-k) and B = 1 (only the kept experts).

XShare ("XShare: Collaborative in-Batch Expert Sharing for Faster MoE
Inference", AI summary and abstract): the chosen expert set is compared
with an exhaustive search over all subsets of the batch union for the
modular objective, plus the closed form budget >= |union| (standard top-k).

XShare's hierarchical selection for speculative batches (same page,
abstract): the closed forms group = 1 (plain XShare) and one request for the
whole batch (plain XShare with budget k), an exhaustive search over the
subsets at both levels on tiny batches, and a hand-worked case where the
request level changes the batch set.

Hand-derived cases (worked out in the comments) pin the fill order and the
tie rules.
"""
import itertools

import numpy as np
import pytest

import moe_synth as ms

NONE, OEA, XSHARE, XSHARE_HIER = 0, 1, 2, 4


def _rank_order(logits):
    B, E = logits.shape
    idx = np.arange(E)
    return np.stack([np.lexsort((idx, -logits[b].astype(np.float64))) for b in range(B)])


def _random_router(rng, B, E, scale=1.5, skew=2.0):
    logits = (rng.standard_normal((B, E)) * scale - skew * np.log1p(rng.permutation(E))).astype(np.float32)
    p = np.exp(logits.astype(np.float64) - logits.max(1, keepdims=True))
    probs = (p / p.sum(1, keepdims=True)).astype(np.float32)
    return logits, probs


def _check_weights(probs, sel, w):
    for b in range(sel.shape[0]):
        m = sel[b] >= 0
        assert np.all(w[b, ~m] == 0)
        pk = probs[b, sel[b, m]].astype(np.float64)
        assert np.allclose(w[b, m], pk / pk.sum(), rtol=3e-7, atol=0)
        assert abs(float(w[b, m].astype(np.float64).sum()) - 1.0) <= 1e-6


def check_oea(logits, probs, sel, w, k, k0):
    order = _rank_order(logits)
    B = logits.shape[0]
    kept = order[:, :k0]
    u_kept = set(kept.ravel().tolist())
    u_base = set(order[:, :k].ravel().tolist())
    assert u_kept <= u_base
    for b in range(B):
        row = sel[b].tolist()
        n = sum(1 for e in row if e >= 0)
        assert all(e >= 0 for e in row[:n]) and all(e == -1 for e in row[n:])
        chosen = row[:n]
        assert len(set(chosen)) == n
        assert chosen[:k0] == kept[b].tolist()                 # keeps its top-k0
        fills = chosen[k0:]
        cand = u_kept - set(kept[b].tolist())
        assert set(fills) <= cand                              # only experts already loaded
        assert len(fills) == min(k - k0, len(cand))            # as many as fit
        rank = {e: r for r, e in enumerate(order[b].tolist())}
        assert [rank[e] for e in fills] == sorted(rank[e] for e in fills)
        rest = cand - set(fills)
        if fills and rest:                                     # highest-ranked candidates
            assert max(rank[e] for e in fills) < min(rank[e] for e in rest)
    active = set(e for e in sel.ravel().tolist() if e >= 0)
    assert active == u_kept
    _check_weights(probs, sel, w)


def _xshare_scores64(probs, order, k):
    B, E = probs.shape
    s = np.zeros(E)
    for b in range(B):
        for e in order[b, :k]:
            s[e] += float(probs[b, e])
    return s


def check_xshare(logits, probs, sel, w, k, budget, brute=False):
    order = _rank_order(logits)
    B, E = logits.shape
    u_base = sorted(set(order[:, :k].ravel().tolist()))
    mp = min(budget, len(u_base))
    S = sorted(set(e for e in sel.ravel().tolist() if e >= 0))
    assert len(S) == mp and set(S) <= set(u_base)
    for b in range(B):
        row = sel[b].tolist()
        assert all(e >= 0 for e in row) and len(set(row)) == k
        want = [e for e in order[b].tolist() if e in set(S)][:k]
        assert row == want
    _check_weights(probs, sel, w)
    if brute:
        s = _xshare_scores64(probs, order, k)
        got = s[S].sum()
        best = max(s[list(c)].sum() for c in itertools.combinations(u_base, mp))
        assert got >= best - 1e-6 * max(1.0, best)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("k,k0", [(4, 1), (4, 2), (4, 3), (8, 2), (8, 4), (8, 6)])
def test_oea_characterisation_random(oracle_lib, seed, k, k0):
    rng = np.random.default_rng(100 * seed + 10 * k + k0)
    B = int(rng.integers(1, 40))
    E = int(rng.choice([16, 64, 128, 256]))
    logits, probs = _random_router(rng, B, E)
    sel, w = oracle_lib.reselect(logits, probs, k, OEA, k0=k0)
    check_oea(logits, probs, sel, w, k, k0)


@pytest.mark.parametrize("shape,B,k0", [("tiny", 4, 2), ("e64", 16, 4), ("q30b", 16, 2),
                                        ("q30b", 16, 4), ("q30b", 64, 6), ("q235b", 16, 4)])
def test_oea_characterisation_layers(oracle_lib, shape, B, k0):
    S = ms.SHAPES[shape]
    L = ms.make_weights(S, 0, experts=False)
    x = ms.make_tokens(S, B, 0)
    logits, probs, ti, tw = oracle_lib.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle_lib.reselect(logits, probs, S.k, OEA, k0=k0)
    check_oea(logits, probs, sel, w, S.k, k0)
    base = len(set(ti.ravel().tolist()))
    n_act = len(set(e for e in sel.ravel().tolist() if e >= 0))
    assert n_act <= base


@pytest.mark.parametrize("seed", range(4))
def test_oea_k0_equals_k_is_standard_topk(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    logits, probs = _random_router(rng, 17, 128)
    s_none, w_none = oracle_lib.reselect(logits, probs, 8, NONE)
    s_oea, w_oea = oracle_lib.reselect(logits, probs, 8, OEA, k0=8)
    assert np.array_equal(s_none, s_oea)
    assert np.array_equal(w_none.view(np.uint32), w_oea.view(np.uint32))
    assert np.array_equal(s_none, _rank_order(logits)[:, :8])


def test_oea_batch_of_one_keeps_only_k0(oracle_lib):
    rng = np.random.default_rng(3)
    logits, probs = _random_router(rng, 1, 128)
    for k0 in range(1, 9):
        sel, w = oracle_lib.reselect(logits, probs, 8, OEA, k0=k0)
        assert (sel >= 0).sum() == k0
        assert sel[0, :k0].tolist() == _rank_order(logits)[0, :k0].tolist()


def test_oea_hand_worked_example(oracle_lib):
    # B=3, E=6, k=3, k0=1.  Rank orders:
    #   token 0: 0 3 1 2 4 5   kept {0}
    #   token 1: 1 0 5 2 3 4   kept {1}
    #   token 2: 2 4 3 0 1 5   kept {2}
    # U_kept = {0,1,2}.  Fills walk each order and take members of U_kept:
    #   token 0: 3 no, 1 yes, 2 yes      -> [0, 1, 2]
    #   token 1: 0 yes, 5 no, 2 yes      -> [1, 0, 2]
    #   token 2: 4 no, 3 no, 0 yes, 1 yes -> [2, 0, 1]
    # Standard top-3 would activate all 6 experts; OEA activates 3.
    orders = [[0, 3, 1, 2, 4, 5], [1, 0, 5, 2, 3, 4], [2, 4, 3, 0, 1, 5]]
    logits = np.zeros((3, 6), np.float32)
    for b, o in enumerate(orders):
        for r, e in enumerate(o):
            logits[b, e] = 5.0 - r
    p = np.exp(logits - logits.max(1, keepdims=True))
    probs = (p / p.sum(1, keepdims=True)).astype(np.float32)
    sel, w = oracle_lib.reselect(logits, probs, 3, OEA, k0=1)
    assert sel.tolist() == [[0, 1, 2], [1, 0, 2], [2, 0, 1]]
    sel_n, _ = oracle_lib.reselect(logits, probs, 3, NONE)
    assert sel_n.tolist() == [[0, 3, 1], [1, 0, 5], [2, 4, 3]]


def test_oea_short_sets_are_padded(oracle_lib):
    # both tokens keep expert 0 (k0=1): U_kept = {0} leaves nothing to fill,
    # so each token runs one expert with weight 1 and two empty slots.
    logits = np.array([[9, 8, 7, 6, 5, 4], [9, 7, 8, 6, 5, 4]], np.float32)
    p = np.exp(logits - 9)
    probs = (p / p.sum(1, keepdims=True)).astype(np.float32)
    sel, w = oracle_lib.reselect(logits, probs, 3, OEA, k0=1)
    assert sel.tolist() == [[0, -1, -1], [0, -1, -1]]
    assert w.tolist() == [[1.0, 0.0, 0.0], [1.0, 0.0, 0.0]]


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("budget", [4, 6, 8])
def test_xshare_brute_force_tiny(oracle_lib, seed, budget):
    # E=16, B=4, k=4: every subset of the batch union of size M' is tried
    rng = np.random.default_rng(1000 + seed)
    logits, probs = _random_router(rng, 4, 16, scale=1.0, skew=0.5)
    sel, w = oracle_lib.reselect(logits, probs, 4, XSHARE, budget=budget)
    check_xshare(logits, probs, sel, w, 4, budget, brute=True)


def test_xshare_brute_force_tiny_layer(oracle_lib):
    S = ms.SHAPES["tiny"]
    L = ms.make_weights(S, 0, experts=False)
    for seed in range(3):
        x = ms.make_tokens(S, 4, seed)
        logits, probs, ti, tw = oracle_lib.route(x, L["Wg"], L["bias"], S.k)
        for budget in (4, 6, 8):
            sel, w = oracle_lib.reselect(logits, probs, S.k, XSHARE, budget=budget)
            check_xshare(logits, probs, sel, w, S.k, budget, brute=True)


@pytest.mark.parametrize("budget", [24, 32, 48])
def test_xshare_speculative_batch(oracle_lib, budget):
    S = ms.SHAPES["q30b"]
    L = ms.make_weights(S, 0, experts=False)
    x = ms.make_tokens(S, 32, 0, kind="spec")
    logits, probs, ti, tw = oracle_lib.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle_lib.reselect(logits, probs, S.k, XSHARE, budget=budget)
    check_xshare(logits, probs, sel, w, S.k, budget)
    assert len(set(sel.ravel().tolist())) <= min(budget, len(set(ti.ravel().tolist())))


@pytest.mark.parametrize("seed", range(4))
def test_xshare_large_budget_is_standard_topk(oracle_lib, seed):
    rng = np.random.default_rng(50 + seed)
    logits, probs = _random_router(rng, 16, 128)
    s_none, w_none = oracle_lib.reselect(logits, probs, 8, NONE)
    s_x, w_x = oracle_lib.reselect(logits, probs, 8, XSHARE, budget=128)
    assert np.array_equal(s_none, s_x)
    assert np.array_equal(w_none.view(np.uint32), w_x.view(np.uint32))


def test_xshare_hand_worked_ties(oracle_lib):
    # B=2, E=6, k=2.  p0 = [.3 .3 .1 .1 .1 .1], p1 = [.1 .1 .3 .3 .1 .1].
    # T_0 = {0,1}, T_1 = {2,3} (equal logits go to the lower index).
    # Scores s = [.3 .3 .3 .3 0 0]; budget 2 -> four-way tie -> S = {0, 1}.
    # Token 1's order is 2 3 0 1 4 5, so within S it takes [0, 1].
    p = np.array([[.3, .3, .1, .1, .1, .1], [.1, .1, .3, .3, .1, .1]], np.float32)
    logits = np.log(p).astype(np.float32)
    sel, w = oracle_lib.reselect(logits, p, 2, XSHARE, budget=2)
    assert sel.tolist() == [[0, 1], [0, 1]]
    assert np.allclose(w, 0.5)
    sel3, _ = oracle_lib.reselect(logits, p, 2, XSHARE, budget=3)
    assert sel3.tolist() == [[0, 1], [2, 0]]


@pytest.mark.parametrize("mode,k0,budget", [(NONE, 0, 0), (OEA, 2, 0), (XSHARE, 0, 20)])
def test_lists_reconstruct_selection(oracle_lib, mode, k0, budget):
    rng = np.random.default_rng(7)
    B, E, k = 23, 64, 8
    logits, probs = _random_router(rng, B, E)
    sel, w = oracle_lib.reselect(logits, probs, k, mode, k0=k0, budget=budget)
    li = oracle_lib.lists(sel, w, E)
    n = li["n_active"]
    act = li["active"][:n]
    assert np.all(np.diff(act) > 0) and np.all(li["active"][n:] == -1)
    assert set(act.tolist()) == set(e for e in sel.ravel().tolist() if e >= 0)
    off = li["offsets"]
    total = int((sel >= 0).sum())
    assert off[0] == 0 and off[n] == total and np.all(off[n:] == total)
    rebuilt = {}
    for i, e in enumerate(act.tolist()):
        toks = li["tok"][off[i]:off[i + 1]]
        assert np.all(np.diff(toks) > 0)
        for j, t in enumerate(toks.tolist()):
            rebuilt[(t, e)] = li["w"][off[i] + j]
    want = {(b, int(sel[b, j])): w[b, j] for b in range(B) for j in range(k) if sel[b, j] >= 0}
    assert rebuilt == want
    assert np.all(li["tok"][total:] == -1) and np.all(li["w"][total:] == 0)


# ------------------------------------------------------------------ Lynx --
# Affinity binning ("Lynx: Enabling Efficient MoE Inference through Dynamic
# Batch-Aware Expert Selection", sections 2.1-2.2): a confidence per token
# from the gap of its top-ranked experts, bins fixed by k/E, exponentially
# weighted expert scores, a minimal critical set, and every token keeping
# exactly k experts inside it.  Pinned by invariants the reading fixes, the
# closed forms B = 1 and identical tokens (standard top-k), and two
# hand-worked cases.
AFFINITY = 3


def check_affinity(logits, probs, sel, w, k):
    order = _rank_order(logits)
    B = logits.shape[0]
    u_base = set(order[:, :k].ravel().tolist())
    S = set(sel.ravel().tolist())
    assert -1 not in S                                  # exactly k per token
    assert S <= u_base
    assert len(S) >= k
    assert {int(order[b, 0]) for b in range(B)} <= S    # rank-0 experts survive
    for b in range(B):
        inside = [int(e) for e in order[b] if int(e) in S][:k]
        assert sel[b].tolist() == inside                # first k of its order in S
    _check_weights(probs, sel, w)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("B,E,k", [(4, 16, 4), (16, 128, 8), (32, 64, 8), (7, 256, 16)])
def test_affinity_invariants_random(oracle_lib, seed, B, E, k):
    rng = np.random.default_rng(300 + seed)
    logits, probs = _random_router(rng, B, E)
    sel, w = oracle_lib.reselect(logits, probs, k, AFFINITY)
    check_affinity(logits, probs, sel, w, k)
    # never more experts than standard routing activates
    s_none, _ = oracle_lib.reselect(logits, probs, k, NONE)
    assert len(set(sel.ravel().tolist())) <= len(set(s_none.ravel().tolist()))


@pytest.mark.parametrize("shape,B", [("q30b", 16), ("q30b", 64), ("e64", 16)])
def test_affinity_invariants_layers(oracle_lib, shape, B):
    S = ms.SHAPES[shape]
    L = ms.make_weights(S, 0, experts=False)
    x = ms.make_tokens(S, B, 0)
    logits, probs, ti, tw = oracle_lib.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle_lib.reselect(logits, probs, S.k, AFFINITY)
    check_affinity(logits, probs, sel, w, S.k)


@pytest.mark.parametrize("seed", range(4))
def test_affinity_closed_forms_are_standard_topk(oracle_lib, seed):
    rng = np.random.default_rng(80 + seed)
    # one token: its k experts are the whole union, so the set cannot shrink
    logits, probs = _random_router(rng, 1, 64)
    s_none, w_none = oracle_lib.reselect(logits, probs, 8, NONE)
    s_a, w_a = oracle_lib.reselect(logits, probs, 8, AFFINITY)
    assert np.array_equal(s_none, s_a) and np.array_equal(w_none.view(np.uint32), w_a.view(np.uint32))
    # identical tokens: the union is one token's top-k
    logits5 = np.repeat(logits, 5, axis=0)
    probs5 = np.repeat(probs, 5, axis=0)
    s_none, w_none = oracle_lib.reselect(logits5, probs5, 8, NONE)
    s_a, w_a = oracle_lib.reselect(logits5, probs5, 8, AFFINITY)
    assert np.array_equal(s_none, s_a) and np.array_equal(w_none.view(np.uint32), w_a.view(np.uint32))


def test_affinity_hand_worked_example(oracle_lib):
    # E = 8, k = 2: 4 bins of width 2/8 on the gap c of the two top
    # probabilities; bin = largest j < 4 with 2 j <= 8 c.
    #  token 0: order 0 1 3 2 ..., c = .75 - .125 = .625, 8c = 5 -> bin 2 (weight 4)
    #  token 1: order 1 2 0 3 ..., c = .3125 - .25 = .0625, 8c = .5 -> bin 0 (weight 1)
    #  token 2: order 0 3 1 2 ..., c = .5 - .25 = .25, 8c = 2 -> bin 1 (weight 2: 2 <= 2 counts)
    # scores (top-2 memberships): e0 = 4 + 2 = 6, e1 = 4 + 1 = 5, e2 = 1, e3 = 2
    # score order e0 e1 e3 e2; rank-0 experts e0 e1 e0 sit at positions 0 1 0
    # -> M = max(2, 2) = 2, S = {0, 1}; each token takes its first two in S.
    logits = np.array([[8, 7, 1, 2, 0, -1, -2, -3],
                       [5, 9, 8, 1, 0, -1, -2, -3],
                       [9, 2, 1, 8, 0, -1, -2, -3]], np.float32)
    probs = np.array([[.75, .125, .03125, .0625, 0, 0, 0, 0],
                      [.125, .3125, .25, .0625, 0, 0, 0, 0],
                      [.5, .125, .0625, .25, 0, 0, 0, 0]], np.float32)
    sel, w = oracle_lib.reselect(logits, probs, 2, AFFINITY)
    assert sel.tolist() == [[0, 1], [1, 0], [0, 1]]
    expect = np.array([[.75 / .875, .125 / .875], [.3125 / .4375, .125 / .4375], [.5 / .625, .125 / .625]],
                      np.float32)
    assert np.allclose(w, expect, rtol=2e-7, atol=0)
    # standard routing would activate four experts
    s_none, _ = oracle_lib.reselect(logits, probs, 2, NONE)
    assert sorted(set(s_none.ravel().tolist())) == [0, 1, 2, 3]


def test_affinity_hand_worked_tie(oracle_lib):
    # E = 8, k = 2, both tokens in bin 0 (zero gaps).
    #  token 0: order 5 2 0 1 ...; token 1: order 2 6 7 5 ...
    # scores e2 = 2, e5 = 1, e6 = 1: the tie e5/e6 goes to the lower index,
    # so the order is e2 e5 e6 and the rank-0 experts (e5, e2) sit at 1, 0:
    # M = 2, S = {2, 5}.  (The opposite tie rule would give S = {2, 6, 5}.)
    logits = np.array([[4, 3, 8, 1, 0, 9, -1, -2],
                       [0, -1, 9, -2, -3, 6, 8, 7]], np.float32)
    probs = np.array([[.05, .04, .25, .02, .01, .25, 0, 0],
                      [.01, 0, .25, 0, 0, .125, .25, .2]], np.float32)
    sel, w = oracle_lib.reselect(logits, probs, 2, AFFINITY)
    assert sel.tolist() == [[5, 2], [2, 5]]
    assert np.allclose(w, [[.5, .5], [.25 / .375, .125 / .375]], rtol=2e-7, atol=0)


# ---------------------------------------------------------------- XShare,
# hierarchical: requests are runs of `group` consecutive tokens.

def _hier_brute(probs, order, k, budget, group):
    """Exhaustive restatement in fp64: each request's best k-subset of the
    experts its tokens' top-k sets hold (by summed request score), then the
    best min(budget, |picked|)-subset of the picked experts by batch score.
    Returns the batch set and the smallest margin between the best and the
    second-best subset seen at any level (near ties make the answer depend
    on rounding, so callers require a clear margin)."""
    B, E = probs.shape
    s = np.zeros(E)
    picked = set()
    margin = np.inf

    def best_two(pool, size, score):
        vals = sorted((score[list(c)].sum(), c) for c in itertools.combinations(pool, size))
        gap = vals[-1][0] - vals[-2][0] if len(vals) > 1 else np.inf
        return set(vals[-1][1]), gap

    for r0 in range(0, B, group):
        sr = np.zeros(E)
        for b in range(r0, min(B, r0 + group)):
            for e in order[b, :k]:
                sr[e] += float(probs[b, e])
        pool = [e for e in range(E) if sr[e] > 0]
        P, gap = best_two(pool, min(k, len(pool)), sr)
        margin = min(margin, gap)
        for e in P:
            s[e] += sr[e]
        picked |= P
    pool = sorted(picked)
    S, gap = best_two(pool, min(budget, len(pool)), s)
    return S, min(margin, gap)


def check_hier(logits, probs, sel, w, k, budget, group):
    """Invariants that hold at any size: the activated set A is the batch
    set (every member of it is in the top-k of some token that takes it),
    A lies in the union of the top-k sets, |A| <= min(budget, requests * k),
    each token takes its first k experts inside A, weights renormalised."""
    order = _rank_order(logits)
    B, E = logits.shape
    nreq = -(-B // group)
    u_base = set(order[:, :k].ravel().tolist())
    A = set(e for e in sel.ravel().tolist() if e >= 0)
    assert A <= u_base
    assert k <= len(A) <= min(budget, nreq * k)
    for b in range(B):
        row = sel[b].tolist()
        assert all(e >= 0 for e in row) and len(set(row)) == k
        assert row == [e for e in order[b].tolist() if e in A][:k]
    _check_weights(probs, sel, w)
    return A


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("budget", [8, 12, 20, 128])
def test_xshare_hier_one_token_per_request_is_xshare(oracle_lib, seed, budget):
    rng = np.random.default_rng(300 + seed)
    logits, probs = _random_router(rng, 19, 128)
    s_x, w_x = oracle_lib.reselect(logits, probs, 8, XSHARE, budget=budget)
    s_h, w_h = oracle_lib.reselect(logits, probs, 8, XSHARE_HIER, budget=budget, group=1)
    assert np.array_equal(s_x, s_h)
    assert np.array_equal(w_x.view(np.uint32), w_h.view(np.uint32))


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("group", [16, 17, 1000])
def test_xshare_hier_one_request_is_xshare_with_budget_k(oracle_lib, seed, group):
    # one request: its k picked experts are the batch's top-k by the summed
    # score, so any budget >= k gives plain XShare with budget k
    rng = np.random.default_rng(400 + seed)
    logits, probs = _random_router(rng, 16, 64)
    s_x, w_x = oracle_lib.reselect(logits, probs, 8, XSHARE, budget=8)
    for budget in (8, 13, 64):
        s_h, w_h = oracle_lib.reselect(logits, probs, 8, XSHARE_HIER, budget=budget, group=group)
        assert np.array_equal(s_x, s_h)
        assert np.array_equal(w_x.view(np.uint32), w_h.view(np.uint32))


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("B,group", [(4, 2), (6, 4), (6, 3), (5, 2)])
@pytest.mark.parametrize("budget", [4, 6, 8])
def test_xshare_hier_brute_force_tiny(oracle_lib, seed, B, group, budget):
    # E=16, k=4: every k-subset at the request level and every subset of the
    # picked experts at the batch level is tried
    rng = np.random.default_rng(2000 + 10 * seed + B)
    logits, probs = _random_router(rng, B, 16, scale=1.0, skew=0.5)
    sel, w = oracle_lib.reselect(logits, probs, 4, XSHARE_HIER, budget=budget, group=group)
    A = check_hier(logits, probs, sel, w, 4, budget, group)
    S, margin = _hier_brute(probs, _rank_order(logits), 4, budget, group)
    if margin > 1e-5:  # a clear optimum at every level
        assert A == S
    else:
        pytest.skip("near tie")


def test_xshare_hier_brute_force_has_clear_cases(oracle_lib):
    # the brute-force comparison above must not be skipped wholesale
    clear = 0
    for seed in range(8):
        for B, group in [(4, 2), (6, 4), (6, 3), (5, 2)]:
            rng = np.random.default_rng(2000 + 10 * seed + B)
            logits, probs = _random_router(rng, B, 16, scale=1.0, skew=0.5)
            for budget in (4, 6, 8):
                _, margin = _hier_brute(probs, _rank_order(logits), 4, budget, group)
                clear += margin > 1e-5
    assert clear >= 80


@pytest.mark.parametrize("budget", [24, 32, 48])
def test_xshare_hier_speculative_batch(oracle_lib, budget):
    # 8 requests x 4 drafts on the Qwen3-30B-shaped router
    S = ms.SHAPES["q30b"]
    L = ms.make_weights(S, 0, experts=False)
    x = ms.make_tokens(S, 32, 0, kind="spec")
    logits, probs, ti, tw = oracle_lib.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle_lib.reselect(logits, probs, S.k, XSHARE_HIER, budget=budget, group=4)
    check_hier(logits, probs, sel, w, S.k, budget, 4)


def test_xshare_hier_hand_worked_example(oracle_lib):
    # E=6, k=2, B=4 in two requests of two tokens (group=2).  Probabilities
    # are dyadic, so every sum below is exact; logits = log2 p.
    #   token 0: p = [.5 .25 .125 .0625 .03125 .03125]     T = {0, 1}
    #   token 1: p = [.5 .03125 .375 .03125 .03125 .03125] T = {0, 2}
    #   token 2: p = [.03125 .375 .03125 .5 .03125 .03125] T = {3, 1}
    #   token 3: p = [.0625 .0625 .0625 .25 .5 .0625]      T = {4, 3}
    # request 0 scores: e0 = 1, e1 = .25, e2 = .375   -> picks {0, 2}
    # request 1 scores: e3 = .75, e1 = .375, e4 = .5  -> picks {3, 4}
    # batch scores over the picks: e0 = 1, e3 = .75, e4 = .5, e2 = .375
    #   budget 3 -> S = {0, 3, 4}; budget 4 (or more) -> S = {0, 2, 3, 4}.
    # Flat XShare scores add e1 = .25 + .375 = .625 instead, so with budget 3
    # it keeps {0, 3, 1}: the request level drops e1, which neither request
    # ranks among its own two best.
    # Each token then takes its first two experts inside S (order by p,
    # equal p to the lower index): budget 3 -> [0 3] [0 3] [3 0] [4 3].
    p = np.array([[.5, .25, .125, .0625, .03125, .03125],
                  [.5, .03125, .375, .03125, .03125, .03125],
                  [.03125, .375, .03125, .5, .03125, .03125],
                  [.0625, .0625, .0625, .25, .5, .0625]], np.float32)
    logits = np.log2(p).astype(np.float32)
    sel, w = oracle_lib.reselect(logits, p, 2, XSHARE_HIER, budget=3, group=2)
    assert sel.tolist() == [[0, 3], [0, 3], [3, 0], [4, 3]]
    f = np.float32
    expect = [[f(.5) / f(.5625), f(.0625) / f(.5625)], [f(.5) / f(.53125), f(.03125) / f(.53125)],
              [f(.5) / f(.53125), f(.03125) / f(.53125)], [f(.5) / f(.75), f(.25) / f(.75)]]
    assert np.array_equal(w, np.array(expect, np.float32))
    sel4, _ = oracle_lib.reselect(logits, p, 2, XSHARE_HIER, budget=4, group=2)
    assert sel4.tolist() == [[0, 2], [0, 2], [3, 0], [4, 3]]
    flat, _ = oracle_lib.reselect(logits, p, 2, XSHARE, budget=3)
    assert flat.tolist() == [[0, 1], [0, 1], [3, 1], [3, 0]]


def test_xshare_hier_lists_reconstruct_selection(oracle_lib):
    rng = np.random.default_rng(9)
    B, E, k = 23, 64, 8
    logits, probs = _random_router(rng, B, E)
    sel, w = oracle_lib.reselect(logits, probs, k, XSHARE_HIER, budget=20, group=4)
    li = oracle_lib.lists(sel, w, E)
    n = li["n_active"]
    assert set(li["active"][:n].tolist()) == set(sel.ravel().tolist())
    assert li["offsets"][n] == B * k
