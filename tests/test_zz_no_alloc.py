"""moe_expert_ffn_noalloc: the expert FFN for callers that cannot allocate
device memory (no workspace argument; scratch in the library's static
device array).  Checked through the C ABI, on two calls in a row, against
the fp64 oracle and against moe_expert_ffn (the entry point with a caller
workspace), both within the layer tolerance (max-abs 2e-2, relative-L2
1e-2).  A call with inconsistent lists, which the kernels run as an empty
call, must leave the shared scratch fit for the next valid call.

This file is collected last on purpose, and it is self-contained so that it
passes both alone in a fresh process and after every other test."""
import os

import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
import aware_expert_routing_moe_b200 as moe

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 1e-2
THREADS = max(1, len(os.sched_getaffinity(0)))


def _device_layer(S, seed, B):
    L = ms.make_weights(S, seed)
    x = ms.make_tokens(S, B, seed)
    t = lambda a: torch.from_numpy(a).cuda()
    return (t(x), t(L["Wg"]), t(L["bias"]), t(L["Wgate"].view(np.int16)), t(L["Wup"].view(np.int16)),
            t(L["Wdown"].view(np.int16)))


def _close(a, b):
    a = torch.as_tensor(a).double().cpu()
    b = torch.as_tensor(b).double().cpu()
    rel = float(torch.linalg.norm(a - b) / torch.linalg.norm(b))
    return float((a - b).abs().max()) <= MAX_ABS and rel <= REL_L2


def _oracle_y(S, seed, B, mode, k0):
    L = ms.make_weights(S, seed)
    x = ms.make_tokens(S, B, seed)
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle.reselect(logits, probs, S.k, mode, k0, 0)
    return oracle.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, threads=THREADS)


@pytest.mark.parametrize("shape,B,mode,k0", [("tiny", 4, moe.MOE_RESELECT_OEA, 2),
                                             ("q30b", 16, moe.MOE_RESELECT_OEA, 4),
                                             ("q30b", 64, moe.MOE_RESELECT_NONE, 0)])
def test_noalloc_matches_workspace_entry_point(shape, B, mode, k0):
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    S = ms.SHAPES[shape]
    x, Wg, bias, Wgate, Wup, Wdown = _device_layer(S, 0, B)
    logits, probs, _, _ = moe.moe_route(x, Wg, bias, S.k)
    _, _, lists = moe.moe_reselect(logits, probs, S.k, mode, k0=k0)
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    y_ref = moe.moe_expert_ffn(x, Wgate, Wup, Wdown, lists, S.k, ws)
    assert moe.moe_check_error(ws) == 0
    y1 = moe.moe_expert_ffn_noalloc(x, Wgate, Wup, Wdown, lists, S.k)
    torch.cuda.synchronize()
    y1 = y1.clone()
    y2 = moe.moe_expert_ffn_noalloc(x, Wgate, Wup, Wdown, lists, S.k)
    torch.cuda.synchronize()
    assert torch.isfinite(y1).all() and torch.isfinite(y2).all()
    y_or = _oracle_y(S, 0, B, mode, k0)
    assert _close(y1, y_or), "first call vs oracle"
    assert _close(y2, y_or), "second call vs oracle"
    assert _close(y1, y_ref), "first call vs moe_expert_ffn"
    assert _close(y2, y_ref), "second call vs moe_expert_ffn"


@pytest.mark.parametrize("shape,B", [("tiny", 4), ("q30b", 64)])
def test_noalloc_call_after_inconsistent_lists(shape, B):
    # n_active = E + 1 is caught on the device: the call runs as an empty
    # one (y = 0); the error word lives in the static scratch, where no one
    # reads it.  The next valid call must match the oracle.
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    S = ms.SHAPES[shape]
    mode, k0 = moe.MOE_RESELECT_OEA, 2
    x, Wg, bias, Wgate, Wup, Wdown = _device_layer(S, 0, B)
    logits, probs, _, _ = moe.moe_route(x, Wg, bias, S.k)
    _, _, lists = moe.moe_reselect(logits, probs, S.k, mode, k0=k0)
    bad = {key: v.clone() for key, v in lists.items()}
    bad["n_active"][0] = S.E + 1
    y_bad = moe.moe_expert_ffn_noalloc(x, Wgate, Wup, Wdown, bad, S.k)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y_bad) == 0
    y = moe.moe_expert_ffn_noalloc(x, Wgate, Wup, Wdown, lists, S.k)
    torch.cuda.synchronize()
    assert _close(y, _oracle_y(S, 0, B, mode, k0))


def test_noalloc_rejects_dims_beyond_the_static_scratch():
    # B=256, d=16384, k=16, d_ff=8192 needs far more scratch than the
    # static array holds (moe.NOALLOC_SCRATCH_BYTES); rejected on the host
    # before anything is enqueued
    lib = moe.load_library()
    A = 0x10000
    st = lib.moe_expert_ffn_noalloc(A, A, A, A, moe.Dims(256, 16384, 256, 16, 8192),
                                    moe.Lists(A, A, A, A, A), A, None)
    assert st == 4  # MOE_ERR_UNSUPPORTED
