"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded inputs.

Router and re-selection: bit-exact (logits, probabilities, indices,
weights, lists).  Layer output: max-abs 2e-2 and relative-L2 1e-2 against
the fp64 oracle, every row of y up to 64 tokens (sampled rows only for the
256-token and 100-token edge layers).  Sizes run from the tiny layer
(several tiles plus ragged tails) to the full Qwen3-30B-A3B- and
Qwen3-235B-A22B-shaped layers."""
import os

import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
import aware_expert_routing_moe_b200 as moe
from gpu_cases import assert_close_y, bits, device_layer, host_layer, shape

pytestmark = pytest.mark.gpu

NONE, OEA, XSHARE, AFFINITY, XSHARE_HIER = 0, 1, 2, 3, 4
THREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    moe.load_library()
    yield
    torch.cuda.synchronize()


def _tokens(name, B, seed, kind="normal"):
    return ms.make_tokens(shape(name), B, seed, kind=kind)


# ------------------------------------------------------------------ router --
ROUTE_CASES = [("tiny", 4, 0), ("tiny", 4, 1), ("tiny", 4, 2), ("e64", 16, 0), ("q30b", 1, 0),
               ("q30b", 4, 1), ("q30b", 16, 0), ("q30b", 32, 2), ("q30b", 64, 0), ("q235b", 1, 0),
               ("q235b", 16, 1), ("q235b", 64, 0), ("min", 3, 0), ("maxek", 256, 0), ("ragged", 37, 0)]


@pytest.mark.parametrize("name,B,seed", ROUTE_CASES)
def test_route_bit_exact(name, B, seed):
    S = shape(name)
    L = ms.make_weights(S, seed, experts=False)
    x = _tokens(name, B, seed)
    ref = oracle.route(x, L["Wg"], L["bias"], S.k)
    xd = torch.from_numpy(x).cuda()
    out = moe.moe_route(xd, torch.from_numpy(L["Wg"]).cuda(), torch.from_numpy(L["bias"]).cuda(), S.k)
    torch.cuda.synchronize()
    for got, want, what in zip(out, ref, ("logits", "probs", "topk_idx", "topk_w")):
        assert np.array_equal(bits(got), bits(want)), what


def test_route_without_bias_and_repeatable():
    S = shape("q30b")
    L = ms.make_weights(S, 3, experts=False)
    x = _tokens("q30b", 16, 3)
    ref = oracle.route(x, L["Wg"], None, S.k)
    xd, Wg = torch.from_numpy(x).cuda(), torch.from_numpy(L["Wg"]).cuda()
    a = moe.moe_route(xd, Wg, None, S.k)
    b = moe.moe_route(xd, Wg, None, S.k)
    torch.cuda.synchronize()
    for t1, t2, want in zip(a, b, ref):
        assert np.array_equal(bits(t1), bits(want)) and np.array_equal(bits(t1), bits(t2))


# -------------------------------------------------------------- reselect --
def _check_reselect(logits, probs, k, mode, k0=0, budget=0, group=1):
    sel_ref, w_ref = oracle.reselect(logits, probs, k, mode, k0, budget, group)
    li_ref = oracle.lists(sel_ref, w_ref, logits.shape[1])
    sel, w, li = moe.moe_reselect(torch.from_numpy(logits).cuda(), torch.from_numpy(probs).cuda(), k, mode,
                                  k0=k0, budget=budget, group=group)
    torch.cuda.synchronize()
    assert np.array_equal(sel.cpu().numpy(), sel_ref)
    assert np.array_equal(bits(w), bits(w_ref))
    n = int(li["n_active"][0].item())
    assert n == li_ref["n_active"]
    for key in ("active", "offsets", "tok"):
        assert np.array_equal(li[key].cpu().numpy(), li_ref[key]), key
    assert np.array_equal(bits(li["w"]), bits(li_ref["w"]))
    return n


RESELECT_RULES = [(NONE, 0, 0), (OEA, 1, 0), (OEA, 2, 0), (OEA, 4, 0), (OEA, 6, 0), (OEA, 8, 0),
                  (XSHARE, 0, 8), (XSHARE, 0, 24), (XSHARE, 0, 32), (XSHARE, 0, 48), (XSHARE, 0, 128),
                  (AFFINITY, 0, 0)]


@pytest.mark.parametrize("B", [1, 4, 16, 32, 64])
@pytest.mark.parametrize("mode,k0,budget", RESELECT_RULES)
def test_reselect_bit_exact_q30b(B, mode, k0, budget):
    S = shape("q30b")
    L = ms.make_weights(S, 0, experts=False)
    x = _tokens("q30b", B, 0)
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    _check_reselect(logits, probs, S.k, mode, k0, budget)


@pytest.mark.parametrize("B", [1, 4, 16, 32, 64, 256])
@pytest.mark.parametrize("group", [1, 3, 4, 256])
@pytest.mark.parametrize("budget", [8, 24, 48])
def test_reselect_xshare_hier_bit_exact_q30b(B, group, budget):
    S = shape("q30b")
    L = ms.make_weights(S, 0, experts=False)
    x = _tokens("q30b", B, 0, kind="spec" if B % 8 == 0 else "normal")
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    _check_reselect(logits, probs, S.k, XSHARE_HIER, budget=budget, group=group)


@pytest.mark.parametrize("budget", [24, 32, 48])
def test_reselect_speculative_batch(budget):
    S = shape("q30b")
    L = ms.make_weights(S, 0, experts=False)
    x = _tokens("q30b", 32, 0, kind="spec")
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    _check_reselect(logits, probs, S.k, XSHARE, budget=budget)
    _check_reselect(logits, probs, S.k, AFFINITY)
    _check_reselect(logits, probs, S.k, XSHARE_HIER, budget=budget, group=4)


@pytest.mark.parametrize("seed", range(6))
def test_reselect_random_edges(seed):
    rng = np.random.default_rng(seed)
    for B, E, k in [(1, 16, 4), (7, 20, 3), (256, 256, 16), (33, 256, 16), (100, 64, 8), (5, 16, 16)]:
        logits = (rng.standard_normal((B, E)) * 1.5 - 2.0 * np.log1p(rng.permutation(E))).astype(np.float32)
        # exact ties: duplicate some columns
        logits[:, E - 1] = logits[:, 0]
        p = np.exp(logits.astype(np.float64) - logits.max(1, keepdims=True))
        probs = (p / p.sum(1, keepdims=True)).astype(np.float32)
        for mode, k0, budget in [(NONE, 0, 0), (OEA, 1, 0), (OEA, max(1, k // 2), 0), (OEA, k, 0),
                                 (XSHARE, 0, k), (XSHARE, 0, min(E, 2 * k)), (XSHARE, 0, E), (AFFINITY, 0, 0)]:
            _check_reselect(logits, probs, k, mode, k0, budget)
        for budget, group in [(k, 1), (min(E, 2 * k), 3), (E, 2), (min(E, 3 * k), B)]:
            _check_reselect(logits, probs, k, XSHARE_HIER, budget=budget, group=group)


# ------------------------------------------------------------------- FFN --
def _run_layer(name, B, seed, mode, k0=0, budget=0, kind="normal", group=1):
    S = shape(name)
    L = host_layer(name, seed)
    D = device_layer(name, seed)
    x = _tokens(name, B, seed, kind)
    xd = torch.from_numpy(x).cuda()
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    sel = torch.empty(B, S.k, dtype=torch.int32, device="cuda")
    selw = torch.empty(B, S.k, dtype=torch.float32, device="cuda")
    nact = torch.empty(4, dtype=torch.int32, device="cuda")
    y = moe.moe_layer_decode(xd, D["Wg"], D["bias"], D["Wgate"], D["Wup"], D["Wdown"], S.k, mode, k0, budget,
                             ws=ws, sel_idx=sel, sel_w=selw, n_active=nact, group=group)
    assert moe.moe_check_error(ws) == 0
    return S, L, x, y.cpu().numpy(), sel.cpu().numpy(), selw.cpu().numpy(), int(nact[0].item())


def _oracle_layer(S, L, x, mode, k0, budget, rows, group=1):
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle.reselect(logits, probs, S.k, mode, k0, budget, group)
    li = oracle.lists(sel, w, S.E)
    y = oracle.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, rows=rows, threads=THREADS)
    return sel, w, li["n_active"], y


LAYER_CASES = [
    ("tiny", 4, 0, NONE, 0, 0), ("tiny", 4, 0, OEA, 2, 0), ("tiny", 4, 1, OEA, 2, 0),
    ("tiny", 4, 2, XSHARE, 0, 6), ("tiny", 16, 0, NONE, 0, 0),
    ("min", 1, 0, NONE, 0, 0), ("min", 5, 0, OEA, 3, 0),
    ("ragged", 37, 0, NONE, 0, 0), ("ragged", 37, 0, OEA, 2, 0), ("ragged", 37, 0, XSHARE, 0, 10),
    ("maxek", 256, 0, NONE, 0, 0), ("maxek", 256, 0, OEA, 8, 0), ("maxek", 100, 0, XSHARE, 0, 40),
    ("tiny", 4, 1, AFFINITY, 0, 0), ("ragged", 37, 0, AFFINITY, 0, 0), ("maxek", 256, 0, AFFINITY, 0, 0),
    ("e64", 16, 0, NONE, 0, 0), ("e64", 16, 0, OEA, 4, 0),
    ("ragged", 6, 0, OEA, 2, 0), ("ragged", 8, 0, XSHARE, 0, 10),
]


@pytest.mark.parametrize("name,B,seed,mode,k0,budget", LAYER_CASES)
def test_layer_decode_parity_small(name, B, seed, mode, k0, budget):
    S, L, x, y, sel, selw, n_act = _run_layer(name, B, seed, mode, k0, budget)
    rows = None if B <= 64 else np.arange(0, B, 7, dtype=np.int32)
    sel_r, w_r, n_r, y_r = _oracle_layer(S, L, x, mode, k0, budget, rows)
    assert np.array_equal(sel, sel_r)
    assert np.array_equal(bits(selw), bits(w_r))
    assert n_act == n_r
    assert_close_y(y if rows is None else y[rows], y_r, f"{name} B={B} mode={mode}")


Q30_CASES = [(1, NONE, 0, 0), (1, OEA, 2, 0), (4, OEA, 4, 0),
             # up to 8 tokens and at most 32 activated experts: warp-level
             # MMAs on 16-row gate/up units; 8 tokens top-8 and 9 tokens:
             # the tensor-core stream
             (5, XSHARE, 0, 12), (8, NONE, 0, 0), (8, OEA, 4, 0), (9, OEA, 4, 0),
             (16, NONE, 0, 0), (16, OEA, 2, 0),
             (16, OEA, 4, 0), (16, OEA, 6, 0), (16, OEA, 8, 0), (16, XSHARE, 0, 16), (16, AFFINITY, 0, 0),
             (64, AFFINITY, 0, 0), (32, NONE, 0, 0), (17, OEA, 4, 0),
             # 33..64 tokens: the 64-row ring (ragged token counts included)
             (33, OEA, 4, 0), (48, NONE, 0, 0), (57, XSHARE, 0, 40),
             (64, NONE, 0, 0), (64, OEA, 4, 0),
             # above 64 tokens: tiles of up to 64 dispatched pairs (several
             # tiles per expert at 256 tokens)
             (65, OEA, 4, 0), (96, NONE, 0, 0), (128, OEA, 4, 0), (256, NONE, 0, 0)]


@pytest.mark.parametrize("B,mode,k0,budget", Q30_CASES)
def test_layer_decode_parity_q30b(B, mode, k0, budget):
    # every row of y against the oracle
    S, L, x, y, sel, selw, n_act = _run_layer("q30b", B, 0, mode, k0, budget)
    sel_r, w_r, n_r, y_r = _oracle_layer(S, L, x, mode, k0, budget, None)
    assert np.array_equal(sel, sel_r)
    assert np.array_equal(bits(selw), bits(w_r))
    assert n_act == n_r
    assert_close_y(y, y_r, f"q30b B={B} mode={mode} k0={k0}")


@pytest.mark.parametrize("budget", [24, 32, 48])
def test_layer_decode_parity_speculative(budget):
    S, L, x, y, sel, selw, n_act = _run_layer("q30b", 32, 0, XSHARE, 0, budget, kind="spec")
    sel_r, w_r, n_r, y_r = _oracle_layer(S, L, x, XSHARE, 0, budget, None)
    assert np.array_equal(sel, sel_r) and n_act == n_r <= budget
    assert np.array_equal(bits(selw), bits(w_r))
    assert_close_y(y, y_r, f"spec budget={budget}")


HIER_LAYER_CASES = [("q30b", 16, 4, 16), ("q30b", 16, 3, 24), ("q30b", 32, 4, 24), ("q30b", 32, 4, 32),
                    ("q30b", 32, 4, 48), ("q30b", 64, 4, 48), ("q30b", 1, 1, 8), ("tiny", 4, 2, 6),
                    ("ragged", 37, 5, 10), ("maxek", 100, 8, 40), ("e64", 16, 4, 16)]


@pytest.mark.parametrize("name,B,group,budget", HIER_LAYER_CASES)
def test_layer_decode_parity_xshare_hier(name, B, group, budget):
    # B <= 64: the fused kernel's selection CTA publishes the batch set and
    # the other CTAs stream from it; larger batches take the dispatch path
    kind = "spec" if name == "q30b" and B % 8 == 0 else "normal"
    S, L, x, y, sel, selw, n_act = _run_layer(name, B, 0, XSHARE_HIER, 0, budget, kind=kind, group=group)
    rows = None if B <= 64 else np.arange(0, B, 7, dtype=np.int32)
    sel_r, w_r, n_r, y_r = _oracle_layer(S, L, x, XSHARE_HIER, 0, budget, rows, group=group)
    assert np.array_equal(sel, sel_r)
    assert np.array_equal(bits(selw), bits(w_r))
    assert n_act == n_r <= budget
    assert_close_y(y if rows is None else y[rows], y_r, f"{name} B={B} hierarchical group={group} budget={budget}")


@pytest.mark.parametrize("B,mode,k0", [(1, OEA, 4), (8, OEA, 4), (16, NONE, 0), (16, OEA, 4), (64, OEA, 4)])
def test_layer_decode_parity_q235b(B, mode, k0):
    S, L, x, y, sel, selw, n_act = _run_layer("q235b", B, 0, mode, k0)
    sel_r, w_r, n_r, y_r = _oracle_layer(S, L, x, mode, k0, 0, None)
    assert np.array_equal(sel, sel_r) and n_act == n_r
    assert np.array_equal(bits(selw), bits(w_r))
    assert_close_y(y, y_r, f"q235b B={B} mode={mode}")


@pytest.mark.parametrize("B", [4, 16])
@pytest.mark.parametrize("layout", ["up_below_gate", "gate_is_up"])
def test_gate_up_buffer_layouts(B, layout):
    # A gate/up stage is copied as one box of Wgate and Wup seen as a single
    # tensor whose matrix dimension steps from the lower buffer to the
    # higher; when Wup lies below Wgate the two halves swap, and when both
    # arguments are the same buffer the stage falls back to one box per
    # matrix.  Both cases must give the oracle's layer (4 tokens: warp-level
    # MMAs, 16: the tensor cores), through the fused layer and the expert
    # entry point.
    name = "q30b"
    S = shape(name)
    L = host_layer(name, 0)
    D = device_layer(name, 0)
    x = _tokens(name, B, 0)
    xd = torch.from_numpy(x).cuda()
    if layout == "up_below_gate":
        both = torch.empty((2,) + tuple(D["Wgate"].shape), dtype=D["Wgate"].dtype, device="cuda")
        both[0].copy_(D["Wup"])
        both[1].copy_(D["Wgate"])
        wgate, wup, up_host = both[1], both[0], L["Wup"]
        assert wup.data_ptr() < wgate.data_ptr()
    else:
        wgate, wup, up_host = D["Wgate"], D["Wgate"], L["Wgate"]
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    sel = torch.empty(B, S.k, dtype=torch.int32, device="cuda")
    selw = torch.empty(B, S.k, dtype=torch.float32, device="cuda")
    y = moe.moe_layer_decode(xd, D["Wg"], D["bias"], wgate, wup, D["Wdown"], S.k, OEA, 4, ws=ws, sel_idx=sel,
                             sel_w=selw)
    assert moe.moe_check_error(ws) == 0
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    sel_r, w_r = oracle.reselect(logits, probs, S.k, OEA, 4, 0)
    assert np.array_equal(sel.cpu().numpy(), sel_r)
    y_r = oracle.ffn(x, L["Wgate"], up_host, L["Wdown"], sel_r, w_r, threads=THREADS)
    assert_close_y(y.cpu().numpy(), y_r, f"layer, {layout}, B={B}")
    li = oracle.lists(sel_r, w_r, S.E)
    dl = {"n_active": torch.tensor([li["n_active"], 0, 0, 0], dtype=torch.int32).cuda(),
          "active": torch.from_numpy(li["active"]).cuda(), "offsets": torch.from_numpy(li["offsets"]).cuda(),
          "tok": torch.from_numpy(li["tok"]).cuda(), "w": torch.from_numpy(li["w"]).cuda()}
    ws.zero_()
    y2 = moe.moe_expert_ffn(xd, wgate, wup, D["Wdown"], dl, S.k, ws)
    assert moe.moe_check_error(ws) == 0
    assert_close_y(y2.cpu().numpy(), y_r, f"moe_expert_ffn, {layout}, B={B}")


@pytest.mark.parametrize("B", [4, 16])
def test_expert_ffn_entry_matches_oracle(B):
    # the FFN stage alone, fed the oracle's own lists (4 tokens: warp-level
    # MMAs, 16: the tensor cores)
    name = "q30b"
    S = shape(name)
    L = host_layer(name, 0)
    D = device_layer(name, 0)
    x = _tokens(name, B, 0)
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle.reselect(logits, probs, S.k, OEA, 4, 0)
    li = oracle.lists(sel, w, S.E)
    dl = {"n_active": torch.tensor([li["n_active"], 0, 0, 0], dtype=torch.int32).cuda(),
          "active": torch.from_numpy(li["active"]).cuda(), "offsets": torch.from_numpy(li["offsets"]).cuda(),
          "tok": torch.from_numpy(li["tok"]).cuda(), "w": torch.from_numpy(li["w"]).cuda()}
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    y = moe.moe_expert_ffn(torch.from_numpy(x).cuda(), D["Wgate"], D["Wup"], D["Wdown"], dl, S.k, ws)
    assert moe.moe_check_error(ws) == 0
    y_r = oracle.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, threads=THREADS)
    assert_close_y(y.cpu().numpy(), y_r, "moe_expert_ffn")


def test_layer_repeatable_and_workspace_reuse():
    name, B = "q30b", 16
    S = shape(name)
    D = device_layer(name, 0)
    x = torch.from_numpy(_tokens(name, B, 0)).cuda()
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    ys, sels = [], []
    for _ in range(3):
        sel = torch.empty(B, S.k, dtype=torch.int32, device="cuda")
        ys.append(moe.moe_layer_decode(x, D["Wg"], D["bias"], D["Wgate"], D["Wup"], D["Wdown"], S.k, OEA, 4,
                                       ws=ws, sel_idx=sel))
        sels.append(sel)
    assert moe.moe_check_error(ws) == 0
    for s in sels[1:]:
        assert torch.equal(s, sels[0])
    for yy in ys[1:]:
        # same routing; the combine's atomics may add in another order
        assert torch.allclose(yy, ys[0], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("name,B,mode,k0", [("q30b", 1, OEA, 4), ("q30b", 4, NONE, 0), ("q30b", 16, OEA, 4),
                                           ("q30b", 40, OEA, 4), ("tiny", 4, OEA, 2), ("q30b", 16, XSHARE, 0),
                                           ("q30b", 16, NONE, 0), ("q235b", 1, OEA, 4), ("q235b", 16, OEA, 4),
                                           ("q235b", 16, NONE, 0)])
def test_layer_graph_replays(name, B, mode, k0):
    # back-to-back calls on one workspace, as a serving loop issues them: a
    # CUDA graph of 4 calls replayed 25 times; the error word stays clear and
    # every replay gives the single call's selection and (up to the order of
    # the combine's atomic adds) its output, which matches the oracle
    S = shape(name)
    L = host_layer(name, 0)
    D = device_layer(name, 0)
    x = _tokens(name, B, 0)
    xd = torch.from_numpy(x).cuda()
    budget = 16 if mode == XSHARE else 0
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    ys = [torch.empty(B, S.d, dtype=torch.float32, device="cuda") for _ in range(4)]
    sels = [torch.empty(B, S.k, dtype=torch.int32, device="cuda") for _ in range(4)]
    s = torch.cuda.Stream()
    # the workspace was zero-filled on the default stream
    s.wait_stream(torch.cuda.current_stream())

    def calls():
        for i in range(4):
            moe.moe_layer_decode(xd, D["Wg"], D["bias"], D["Wgate"], D["Wup"], D["Wdown"], S.k, mode, k0, budget,
                                 ws=ws, y=ys[i], sel_idx=sels[i], stream=s)

    with torch.cuda.stream(s):
        calls()
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        calls()
    with torch.cuda.stream(s):
        for _ in range(25):
            g.replay()
    s.synchronize()
    assert moe.moe_check_error(ws, s) == 0
    sel_r, w_r, n_r, y_r = _oracle_layer(S, L, x, mode, k0, budget, None)
    for i in range(4):
        assert np.array_equal(sels[i].cpu().numpy(), sel_r)
        assert_close_y(ys[i].cpu().numpy(), y_r, f"{name} B={B} replay call {i}")
    del g
