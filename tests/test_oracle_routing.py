"""Pins for the oracle router ("Router Caching and Optimization", section
"Analyzing Router Inference Cost", steps 1-3): logits against an fp64
matrix product within the fp32 forward error bound, probabilities against
an fp64 softmax, top-k against a stable library sort of the fp64 logits
(except provable near-ties), and the tie rule on constructed exact ties."""
import numpy as np
import pytest
import torch

import moe_synth as ms

U32 = 2.0 ** -24


def _rank_order(logits: np.ndarray) -> np.ndarray:
    """Library sort: logit descending, ties to the lower expert index."""
    B, E = logits.shape
    idx = np.arange(E)
    return np.stack([np.lexsort((idx, -logits[b].astype(np.float64))) for b in range(B)])


CASES = [("tiny", 4), ("e64", 16), ("q30b", 1), ("q30b", 16), ("q30b", 64), ("q235b", 8)]


@pytest.mark.parametrize("shape,B", CASES)
def test_route_against_fp64(oracle_lib, shape, B):
    S = ms.SHAPES[shape]
    L = ms.make_weights(S, seed=0, experts=False)
    x = ms.make_tokens(S, B, seed=0)
    logits, probs, ti, tw = oracle_lib.route(x, L["Wg"], L["bias"], S.k)

    x64 = torch.from_numpy(x.astype(np.float64))
    W64 = torch.from_numpy(L["Wg"].astype(np.float64))
    dot64 = (x64 @ W64.T).numpy()
    l64 = dot64 + L["bias"].astype(np.float64)
    n = -(-S.d // 256) * 8 + 5
    gamma = n * U32 / (1 - n * U32)
    bound = gamma * (torch.abs(x64) @ torch.abs(W64).T).numpy() + U32 * np.abs(l64) * 1.0001
    assert np.all(np.abs(logits - l64) <= bound)

    # softmax: against fp64 softmax of the fp32 logits; sum to one
    p64 = torch.softmax(torch.from_numpy(logits.astype(np.float64)), dim=1).numpy()
    assert np.all(np.abs(probs - p64) <= 1e-6 * p64 + 1e-30)
    assert np.all(np.abs(probs.astype(np.float64).sum(1) - 1.0) <= 1e-6)

    # top-k: equal to the stable sort of the fp64 logits unless the fp64 gap
    # at the k-th place is inside twice the error bound (flagged near-tie)
    order64 = _rank_order(l64)
    for b in range(B):
        kth, nxt = order64[b, S.k - 1], order64[b, S.k]
        gap = l64[b, kth] - l64[b, nxt]
        if gap > 2 * (bound[b, kth] + bound[b, nxt]):
            assert set(ti[b].tolist()) == set(order64[b, :S.k].tolist())
    # the oracle's own order: descending fp32 logits, ties to lower index
    order32 = _rank_order(logits)
    assert np.array_equal(ti, order32[:, :S.k])

    # top-k weights: renormalised probabilities of the chosen experts
    pk = np.take_along_axis(probs, ti, axis=1).astype(np.float64)
    assert np.allclose(tw, pk / pk.sum(1, keepdims=True), rtol=3e-7, atol=0)
    assert np.all(np.abs(tw.astype(np.float64).sum(1) - 1.0) <= 1e-6)


def test_route_without_bias(oracle_lib):
    S = ms.SHAPES["tiny"]
    L = ms.make_weights(S, seed=1, experts=False)
    x = ms.make_tokens(S, 5, seed=1)
    l0, *_ = oracle_lib.route(x, L["Wg"], None, S.k)
    l1, *_ = oracle_lib.route(x, L["Wg"], np.zeros(S.E, np.float32), S.k)
    assert np.array_equal(l0, l1)


def test_route_exact_ties_go_to_lower_index(oracle_lib):
    # experts 3, 5 and 9 share one weight row and bias: their logits are
    # bit-identical, so the order among them must be 3, 5, 9
    rng = np.random.default_rng(9)
    E, d, k = 12, 256, 5
    Wg = (rng.standard_normal((E, d)) * 0.02).astype(np.float32)
    Wg[5] = Wg[3]
    Wg[9] = Wg[3]
    bias = np.full(E, -10.0, np.float32)
    bias[[3, 5, 9]] = 10.0
    bias[7] = 20.0
    x = rng.standard_normal((2, d)).astype(np.float32)
    logits, probs, ti, tw = oracle_lib.route(x, Wg, bias, k)
    assert logits[0, 3] == logits[0, 5] == logits[0, 9]
    for b in range(2):
        assert ti[b, :4].tolist() == [7, 3, 5, 9]
        assert probs[b, 3] == probs[b, 5] == probs[b, 9]


def test_route_single_expert_saturates(oracle_lib):
    # one logit 100 above the rest: p = 1 for it and (for gaps > 87) exactly
    # 0 elsewhere
    E, d = 8, 256
    Wg = np.zeros((E, d), np.float32)
    bias = np.zeros(E, np.float32)
    bias[2] = 100.0
    x = np.ones((1, d), np.float32)
    _, probs, ti, tw = oracle_lib.route(x, Wg, bias, 2)
    assert probs[0, 2] == 1.0 and np.count_nonzero(probs[0]) == 1
    assert ti[0].tolist() == [2, 0]
    assert tw[0].tolist() == [1.0, 0.0]
