"""Pins for the oracle's channel top-k FFN and its sector-counted read bytes
("Channel Selection for Mixture-of-Experts Decoding Needs No Calibration
Data", methodology: a selector is a channel score plus a keep rule; top-k
keeps each token's highest-scoring channels; reads are charged in whole
32-byte sectors).

The FFN is checked against a torch fp64 restatement that gathers the kept
channels with a stable NumPy sort, against the dense FFN when every channel
is kept, and by complementarity (the kept and the skipped channels add up
to the dense output).  The byte count is checked against closed forms and
against brute force over every touched byte address."""
import numpy as np
import pytest
import torch

import moe_synth as ms


def _bf16_to_f64(bits: np.ndarray) -> torch.Tensor:
    f = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return torch.from_numpy(f.astype(np.float64))


def _shape():
    return ms.LayerShape("chan", d=256, E=8, k=3, F=128, bias="normal", bias_param=0.7)


def _case(oracle_lib, seed, B=5):
    S = _shape()
    L = ms.make_weights(S, seed)
    x = ms.make_tokens(S, B, seed)
    logits, probs, _, _ = oracle_lib.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle_lib.reselect(logits, probs, S.k, 1, k0=2)   # OEA: some short sets
    rng = np.random.default_rng(100 + seed)
    score = rng.standard_normal((B, S.k, S.F)).astype(np.float32)
    return S, L, x, sel, w, score


def _kept(score_row, c):
    # the c largest scores, equal scores to the lower index (stable sort)
    order = np.argsort(-score_row.astype(np.float64), kind="stable")
    return np.sort(order[:c])


def _restatement(x, L, sel, w, score, c):
    B, d = x.shape
    y = np.zeros((B, d))
    Wg, Wu, Wd = (_bf16_to_f64(L[n]) for n in ("Wgate", "Wup", "Wdown"))
    for b in range(B):
        xb = torch.from_numpy(x[b].astype(np.float64))
        for s in range(sel.shape[1]):
            e = int(sel[b, s])
            if e < 0:
                continue
            K = torch.from_numpy(_kept(score[b, s], c))
            h = torch.nn.functional.silu(Wg[e][K] @ xb) * (Wu[e][K] @ xb)
            y[b] += float(w[b, s]) * (Wd[e][:, K] @ h).numpy()
    return y


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("c", [1, 7, 16, 64, 127])
def test_channels_match_gathered_restatement(oracle_lib, seed, c):
    S, L, x, sel, w, score = _case(oracle_lib, seed)
    y, keep = oracle_lib.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, score, c)
    ref = _restatement(x, L, sel, w, score, c)
    assert np.max(np.abs(y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    assert np.linalg.norm(y) > 0
    for b in range(x.shape[0]):
        for s in range(S.k):
            if sel[b, s] < 0:
                assert not keep[b, s].any()
            else:
                assert np.array_equal(np.flatnonzero(keep[b, s]), _kept(score[b, s], c))


@pytest.mark.parametrize("seed", range(3))
def test_keeping_every_channel_is_the_dense_ffn(oracle_lib, seed):
    S, L, x, sel, w, score = _case(oracle_lib, seed)
    y, keep = oracle_lib.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, score, S.F)
    dense = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w)
    assert np.array_equal(y, dense)            # the same arithmetic, every channel kept
    assert np.array_equal(keep.sum(-1), np.where(sel >= 0, S.F, 0))


@pytest.mark.parametrize("c", [5, 40, 100])
def test_kept_and_skipped_channels_add_up(oracle_lib, c):
    # with distinct scores the top c of -score is the complement of the top
    # F - c of score, and the FFN is linear in the set of channels it keeps
    S, L, x, sel, w, score = _case(oracle_lib, 7)
    y_top, k_top = oracle_lib.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, score, S.F - c)
    y_rest, k_rest = oracle_lib.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, -score, c)
    dense = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w)
    assert not (k_top & k_rest).any()
    assert np.max(np.abs(y_top + y_rest - dense)) <= 1e-12 * np.max(np.abs(dense))


def test_equal_scores_keep_the_lower_channels(oracle_lib):
    S, L, x, sel, w, _ = _case(oracle_lib, 1, B=2)
    score = np.zeros((2, S.k, S.F), np.float32)
    score[:, :, 50] = 1.0                      # one clear winner, then a tie among the rest
    _, keep = oracle_lib.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, score, 4)
    for b in range(2):
        for s in range(S.k):
            if sel[b, s] >= 0:
                assert np.flatnonzero(keep[b, s]).tolist() == [0, 1, 2, 50]


def test_rows_subset_matches_full(oracle_lib):
    S, L, x, sel, w, score = _case(oracle_lib, 2)
    y, _ = oracle_lib.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, score, 20, threads=2)
    rows = np.array([4, 1], np.int32)
    yr, _ = oracle_lib.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, score, 20, rows=rows)
    assert np.array_equal(yr, y[rows])


# ------------------------------------------------------------ read bytes --
def _brute_bytes(keep, sel, E, d, F, channel_major):
    """Every byte address the kept channels touch, collected per weight
    array, then the distinct 32-byte sectors."""
    B, k, _ = keep.shape
    total = 0
    for arr in ("gate", "up", "down"):
        sectors = set()
        for b in range(B):
            for s in range(k):
                e = int(sel[b, s])
                if e < 0:
                    continue
                for f in np.flatnonzero(keep[b, s]):
                    if arr != "down" or channel_major:
                        base = ((e * F + int(f)) * d) * 2
                        addrs = range(base, base + 2 * d)
                    else:
                        addrs = [((e * d + i) * F + int(f)) * 2 + t for i in range(d) for t in (0, 1)]
                    sectors.update(a // 32 for a in addrs)
        total += 32 * len(sectors)
    return total


@pytest.mark.parametrize("channel_major", [False, True])
@pytest.mark.parametrize("c", [1, 3, 17])
def test_sector_bytes_brute_force(oracle_lib, channel_major, c):
    E, d, F, B, k = 4, 64, 48, 3, 2
    rng = np.random.default_rng(c)
    sel = np.array([[0, 2], [2, -1], [3, 0]], np.int32)
    keep = np.zeros((B, k, F), np.uint8)
    for b in range(B):
        for s in range(k):
            if sel[b, s] >= 0:
                keep[b, s, rng.permutation(F)[:c]] = 1
    got = oracle_lib.channel_sector_bytes(keep, sel, E, d, channel_major)
    assert got == _brute_bytes(keep, sel, E, d, F, channel_major)


def test_sector_bytes_closed_forms(oracle_lib):
    E, d, F = 4, 256, 128
    sel = np.array([[1, 3]], np.int32)
    keep = np.ones((1, 2, F), np.uint8)
    dense = 2 * 3 * d * F * 2                  # two experts, every byte of each
    assert oracle_lib.channel_sector_bytes(keep, sel, E, d) == dense
    assert oracle_lib.channel_sector_bytes(keep, sel, E, d, True) == dense
    one = np.zeros((1, 2, F), np.uint8)
    one[:, :, 37] = 1                          # one channel per expert
    # gate + up rows: 2 x 2d bytes; down: one sector in each of d rows
    assert oracle_lib.channel_sector_bytes(one, sel, E, d) == 2 * (2 * 2 * d + 32 * d)
    assert oracle_lib.channel_sector_bytes(one, sel, E, d, True) == 2 * (3 * 2 * d)
    group = np.zeros((1, 2, F), np.uint8)
    group[:, :, 16:32] = 1                     # sixteen channels sharing one down sector per row
    assert oracle_lib.channel_sector_bytes(group, sel, E, d) == 2 * (16 * 2 * 2 * d + 32 * d)
    # the same expert on two slots reads the union of its kept channels once
    sel2 = np.array([[1, 1]], np.int32)
    assert oracle_lib.channel_sector_bytes(one, sel2, E, d) == 2 * 2 * d + 32 * d
