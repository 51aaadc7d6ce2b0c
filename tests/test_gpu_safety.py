"""Failure paths of the CUDA kernels that a caller can reach without a GPU
fault: token lists from the caller that are inconsistent with the dims.

moe_expert_ffn takes its lists from the caller.  The kernels check
n_active, the active ids, the offsets and the token ids before using any
of them as an index; an inconsistent list records an error word that
moe_check_error reports as MOE_ERR_INTERNAL, and every access stays inside
the caller's buffers and the workspace.  After such a call the workspace is
zeroed again (as the header asks) and a valid call matches the oracle."""
import os

import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
import aware_expert_routing_moe_b200 as moe
from gpu_cases import assert_close_y, device_layer, host_layer, shape

pytestmark = pytest.mark.gpu

OEA = 1
MOE_ERR_INTERNAL = 6
THREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    moe.load_library()
    yield
    torch.cuda.synchronize()


def _oracle_lists(name, B, k0):
    S = shape(name)
    L = host_layer(name, 0)
    x = ms.make_tokens(S, B, 0)
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle.reselect(logits, probs, S.k, OEA, k0, 0)
    li = oracle.lists(sel, w, S.E)
    return S, L, x, sel, w, li


def _device_lists(li, E, B, k):
    return {"n_active": torch.tensor([li["n_active"], 0, 0, 0], dtype=torch.int32).cuda(),
            "active": torch.from_numpy(li["active"].copy()).cuda(),
            "offsets": torch.from_numpy(li["offsets"].copy()).cuda(),
            "tok": torch.from_numpy(li["tok"].copy()).cuda(),
            "w": torch.from_numpy(li["w"].copy()).cuda()}


def _ffn(name, x, dl, ws):
    S = shape(name)
    D = device_layer(name, 0)
    y = moe.moe_expert_ffn(torch.from_numpy(x).cuda(), D["Wgate"], D["Wup"], D["Wdown"], dl, S.k, ws)
    return y, moe.moe_check_error(ws)


# tiny (B = 4): dense mode on warp-level MMAs; ragged (B = 9, 37): dense
# mode on the tensor cores; ragged (B = 70): token tiles of the dispatched
# pairs
@pytest.mark.parametrize("name,B,k0", [("tiny", 4, 2), ("ragged", 37, 2), ("ragged", 70, 2), ("ragged", 9, 2)])
@pytest.mark.parametrize("damage", ["n_active_above_E", "n_active_negative", "active_id_out_of_range",
                                    "offsets_decreasing", "offsets_past_pairs"])
def test_inconsistent_lists_are_reported_and_contained(name, B, k0, damage):
    S, L, x, sel, w, li = _oracle_lists(name, B, k0)
    dl = _device_lists(li, S.E, B, S.k)
    n = li["n_active"]
    if damage == "n_active_above_E":
        dl["n_active"][0] = S.E + 1
    elif damage == "n_active_negative":
        dl["n_active"][0] = -3
    elif damage == "active_id_out_of_range":
        dl["active"][n - 1] = S.E + 7
    elif damage == "offsets_decreasing":
        dl["offsets"][1] = li["offsets"][2] + 1
    elif damage == "offsets_past_pairs":
        dl["offsets"][n] = B * S.k + 64
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    y, status = _ffn(name, x, dl, ws)
    assert status == MOE_ERR_INTERNAL, damage
    # the kernel ran the call as empty: y was zeroed and nothing added
    assert torch.count_nonzero(y) == 0, damage
    # recovery: zero the workspace, then a valid call matches the oracle
    ws.zero_()
    y2, status2 = _ffn(name, x, _device_lists(li, S.E, B, S.k), ws)
    assert status2 == 0
    y_r = oracle.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, threads=THREADS)
    assert_close_y(y2.cpu().numpy(), y_r, f"{name} after {damage}")


@pytest.mark.parametrize("name,B,k0", [("tiny", 4, 2), ("ragged", 37, 2), ("ragged", 70, 2)])
def test_token_outside_batch_is_skipped_and_reported(name, B, k0):
    # one list entry names token B + 5; that pair is skipped, the other
    # pairs are combined as usual (dense mode: the preparation leaves its
    # weight at 0; token tiles: the down epilogue skips it)
    S, L, x, sel, w, li = _oracle_lists(name, B, k0)
    dl = _device_lists(li, S.E, B, S.k)
    p = int(li["offsets"][0])  # first pair of the first active expert
    t_bad = int(li["tok"][p])
    e_bad = int(li["active"][0])
    dl["tok"][p] = B + 5
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    y, status = _ffn(name, x, dl, ws)
    assert status == MOE_ERR_INTERNAL
    # oracle with that one pair's weight set to 0
    w2 = w.copy()
    slot = int(np.nonzero(sel[t_bad] == e_bad)[0][0])
    w2[t_bad, slot] = 0.0
    y_r = oracle.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w2, threads=THREADS)
    assert_close_y(y.cpu().numpy(), y_r, "bad token skipped")


# ------------------------------------------------------------ bounded waits --
@pytest.mark.parametrize("path", ["layer_fused", "expert_ffn", "layer_tiled", "layer_fused_b4", "expert_ffn_b4"])
def test_bounded_waits_expire_and_report(path):
    # With a 200 ns limit every wait on a copy, on another CTA or on a flag
    # runs out: each CTA records the error, lets its copies in flight land,
    # ends its share of the call and exits; the call completes and
    # moe_check_error reports MOE_ERR_INTERNAL.  After the default limit is
    # restored and the workspace zeroed, the same call matches the oracle.
    # the four-kernel path starts above 64 tokens; up to 8 tokens the expert
    # stream runs on warp-level MMAs
    name, B = {"layer_tiled": ("q30b", 96), "layer_fused_b4": ("q30b", 4),
               "expert_ffn_b4": ("q30b", 4)}.get(path, ("q30b", 16))
    S = shape(name)
    L = host_layer(name, 0)
    D = device_layer(name, 0)
    x = ms.make_tokens(S, B, 0)
    xd = torch.from_numpy(x).cuda()
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle.reselect(logits, probs, S.k, OEA, 4, 0)
    li = oracle.lists(sel, w, S.E)

    def call():
        if path.startswith("expert_ffn"):
            y = moe.moe_expert_ffn(xd, D["Wgate"], D["Wup"], D["Wdown"], _device_lists(li, S.E, B, S.k), S.k, ws)
        else:
            y = moe.moe_layer_decode(xd, D["Wg"], D["bias"], D["Wgate"], D["Wup"], D["Wdown"], S.k, OEA, 4, ws=ws)
        return y, moe.moe_check_error(ws)

    moe.moe_set_wait_limit_ns(200)
    try:
        _, status = call()
    finally:
        moe.moe_set_wait_limit_ns(0)
    assert status == MOE_ERR_INTERNAL
    ws.zero_()
    y, status = call()
    assert status == 0
    y_r = oracle.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, threads=THREADS)
    assert_close_y(y.cpu().numpy(), y_r, f"{path} after expired waits")
