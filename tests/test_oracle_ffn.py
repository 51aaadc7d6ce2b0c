"""Pins for the oracle's expert FFN and combine: a dense fp64 restatement
with torch library ops over ALL experts with a [B][E] weight matrix (zero
off the chosen set) must equal the oracle's sparse per-token loop; a single
expert with weight 1 must equal the SwiGLU formula written with
torch.nn.functional.silu; the output is linear in the gate weights."""
import numpy as np
import pytest
import torch

import moe_synth as ms

NONE, OEA, XSHARE = 0, 1, 2


def _bf16_to_f64(bits: np.ndarray) -> torch.Tensor:
    f = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return torch.from_numpy(f.astype(np.float64))


def _dense_reference(x, L, sel, w):
    E = L["Wgate"].shape[0]
    B = x.shape[0]
    x64 = torch.from_numpy(x.astype(np.float64))
    Wg, Wu, Wd = (_bf16_to_f64(L[n]) for n in ("Wgate", "Wup", "Wdown"))
    G = torch.einsum("bd,efd->bef", x64, Wg)
    U = torch.einsum("bd,efd->bef", x64, Wu)
    H = torch.nn.functional.silu(G) * U
    O = torch.einsum("bef,edf->bed", H, Wd)
    Wm = torch.zeros(B, E, dtype=torch.float64)
    for b in range(B):
        for j in range(sel.shape[1]):
            if sel[b, j] >= 0:
                Wm[b, sel[b, j]] += float(w[b, j])
    return torch.einsum("be,bed->bd", Wm, O).numpy()


def _small_shape():
    return ms.LayerShape("small", d=512, E=8, k=3, F=256, bias="normal", bias_param=0.7)


@pytest.mark.parametrize("shape", ["tiny", "small"])
@pytest.mark.parametrize("mode,k0,budget", [(NONE, 0, 0), (OEA, 1, 0), (OEA, 2, 0), (XSHARE, 0, 5)])
def test_ffn_equals_dense_restatement(oracle_lib, shape, mode, k0, budget):
    S = ms.SHAPES["tiny"] if shape == "tiny" else _small_shape()
    L = ms.make_weights(S, 2)
    x = ms.make_tokens(S, 6, 2)
    logits, probs, ti, tw = oracle_lib.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle_lib.reselect(logits, probs, S.k, mode, k0=k0, budget=budget)
    y = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, threads=2)
    ref = _dense_reference(x, L, sel, w)
    assert np.max(np.abs(y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    assert np.linalg.norm(y) > 0


def test_ffn_single_expert_matches_silu_formula(oracle_lib):
    S = _small_shape()
    L = ms.make_weights(S, 4)
    x = ms.make_tokens(S, 3, 4)
    e = 5
    sel = np.full((3, S.k), -1, np.int32)
    sel[:, 0] = e
    w = np.zeros((3, S.k), np.float32)
    w[:, 0] = 1.0
    y = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w)
    x64 = torch.from_numpy(x.astype(np.float64))
    Wg = _bf16_to_f64(L["Wgate"][e])
    Wu = _bf16_to_f64(L["Wup"][e])
    Wd = _bf16_to_f64(L["Wdown"][e])
    ref = ((torch.nn.functional.silu(x64 @ Wg.T) * (x64 @ Wu.T)) @ Wd.T).numpy()
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_ffn_is_linear_in_gate_weights(oracle_lib):
    S = _small_shape()
    L = ms.make_weights(S, 6)
    x = ms.make_tokens(S, 4, 6)
    rng = np.random.default_rng(0)
    sel = np.stack([rng.permutation(S.E)[:S.k] for _ in range(4)]).astype(np.int32)
    # multiples of 2^-8 so that w1 + w2 is exact in fp32
    w1 = (rng.integers(0, 256, (4, S.k)) / 256.0).astype(np.float32)
    w2 = (rng.integers(0, 256, (4, S.k)) / 256.0).astype(np.float32)
    y1 = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w1)
    y2 = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w2)
    y12 = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w1 + w2)
    assert np.max(np.abs(y12 - (y1 + y2))) <= 1e-12 * np.max(np.abs(y12))
    # zero weights give zero output; empty slots are skipped
    sel0 = np.full_like(sel, -1)
    y0 = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel0, w1)
    assert np.all(y0 == 0)


def test_ffn_row_subset_matches_full(oracle_lib):
    S = ms.SHAPES["tiny"]
    L = ms.make_weights(S, 0)
    x = ms.make_tokens(S, 9, 0)
    r = oracle_lib.layer(x, L, S.k, OEA, k0=2, threads=3)
    rows = np.array([7, 0, 4], np.int32)
    ys = oracle_lib.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], r["sel_idx"], r["sel_w"], rows=rows)
    assert np.array_equal(ys, r["y"][rows])
