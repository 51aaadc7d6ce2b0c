"""moe_decode_stack: MoE layers back to back on a residual stream,
xs[l + 1] = xs[l] + layer_l(xs[l]), consecutive layers chained on the
device.  Checked against the oracle applied layer by layer: layer l's
routing, computed by the oracle from the GPU's own xs[l], matches the GPU's
bit for bit, and xs[l + 1] - xs[l] is within the layer tolerance (max-abs
2e-2, relative-L2 1e-2) of the oracle's layer output for xs[l].  The
prefill phase bypasses re-selection (standard top-k)."""
import os

import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
import aware_expert_routing_moe_b200 as moe
from gpu_cases import assert_close_y, shape

pytestmark = pytest.mark.gpu

NONE, OEA, XSHARE = 0, 1, 2
THREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    moe.load_library()
    yield
    torch.cuda.synchronize()
    _CACHE.clear()


_CACHE = {}


def _stack_layers(name, n):
    # one set of layers per shape, grown as needed and shared by the tests
    S = shape(name)
    host, dev = _CACHE.setdefault(name, ([], []))
    t = lambda a: torch.from_numpy(a).cuda()
    while len(host) < n:
        L = ms.make_weights(S, len(host))
        host.append(L)
        dev.append((t(L["Wg"]), t(L["bias"]), t(L["Wgate"].view(np.int16)), t(L["Wup"].view(np.int16)),
                    t(L["Wdown"].view(np.int16))))
    return S, host[:n], dev[:n]


def _check_stack(name, B, n, mode, k0=0, budget=0, phase=moe.MOE_PHASE_DECODE, kind="normal"):
    S, host, dev = _stack_layers(name, n)
    x0 = ms.make_tokens(S, B, 0, kind=kind)
    xs = torch.zeros(n + 1, B, S.d, dtype=torch.float32, device="cuda")
    xs[0] = torch.from_numpy(x0).cuda()
    sel = torch.full((n, B, S.k), -7, dtype=torch.int32, device="cuda")
    nact = torch.zeros(n, dtype=torch.int32, device="cuda")
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    moe.moe_decode_stack(xs, dev, S.k, mode, k0, budget, phase=phase, ws=ws, sel_idx=sel, n_active=nact)
    assert moe.moe_check_error(ws) == 0
    xs_h = xs.cpu().numpy()
    sel_h = sel.cpu().numpy()
    eff = (NONE, 0, 0) if phase == moe.MOE_PHASE_PREFILL else (mode, k0, budget)
    for l in range(n):
        L = host[l]
        x_l = np.ascontiguousarray(xs_h[l])
        logits, probs, _, _ = oracle.route(x_l, L["Wg"], L["bias"], S.k)
        sel_r, w_r = oracle.reselect(logits, probs, S.k, *eff)
        li = oracle.lists(sel_r, w_r, S.E)
        assert np.array_equal(sel_h[l], sel_r), f"layer {l} selection"
        assert int(nact[l].item()) == li["n_active"], f"layer {l} n_active"
        y_r = oracle.ffn(x_l, L["Wgate"], L["Wup"], L["Wdown"], sel_r, w_r, threads=THREADS)
        y_gpu = xs_h[l + 1].astype(np.float64) - x_l.astype(np.float64)
        assert_close_y(y_gpu, y_r, f"{name} B={B} layer {l}")
    return xs


@pytest.mark.parametrize("mode,k0,budget", [(OEA, 4, 0), (NONE, 0, 0), (XSHARE, 0, 16)])
def test_stack_of_four_q30b_b16(mode, k0, budget):
    _check_stack("q30b", 16, 4, mode, k0, budget)


def test_stack_fused_path_q30b_b64():
    _check_stack("q30b", 64, 2, OEA, 4)


def test_stack_tiled_path_q30b_b96():
    # above 64 tokens: the four chained kernels per layer
    _check_stack("q30b", 96, 2, OEA, 4)


def test_stack_small_shapes():
    _check_stack("tiny", 4, 3, OEA, 2)
    _check_stack("ragged", 37, 3, OEA, 2)


@pytest.mark.parametrize("B", [16, 64])
def test_stack_prefill_bypasses_reselection(B):
    # the rule given is OEA, but the prefill phase routes standard top-k
    _check_stack("q30b", B, 2, OEA, 2, phase=moe.MOE_PHASE_PREFILL)


def test_stack_of_one_equals_residual_layer_call():
    S, host, dev = _stack_layers("q30b", 1)
    B = 16
    x = torch.from_numpy(ms.make_tokens(S, B, 1)).cuda()
    xs = torch.stack([x, torch.zeros_like(x)])
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    moe.moe_decode_stack(xs, dev, S.k, OEA, 4, ws=ws)
    Wg, bias, g, u, dn = dev[0]
    y = moe.moe_layer_decode(x, Wg, bias, g, u, dn, S.k, OEA, 4, ws=ws)
    assert moe.moe_check_error(ws) == 0
    # same routing and the same experts; the combine's atomics may add in
    # another order
    assert torch.allclose(xs[1], x + y, rtol=1e-5, atol=1e-5)
