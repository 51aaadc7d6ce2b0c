"""GPU parity of per-token channel top-k inside the activated experts
("Channel Selection for Mixture-of-Experts Decoding Needs No Calibration
Data", methodology: each token keeps its c highest-scoring channels of an
expert; only those channels' weights are read).

Through the C ABI against the oracle: the keep masks bit for bit (equal
scores to the lower channel index, exact ties included), y within the layer
tolerance (max-abs 2e-2, relative-L2 1e-2) of the fp64 oracle; the
channel-major down copy element for element."""
import os

import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
import aware_expert_routing_moe_b200 as moe
from gpu_cases import assert_close_y, host_layer, shape

pytestmark = pytest.mark.gpu

NONE, OEA = 0, 1
THREADS = max(1, len(os.sched_getaffinity(0)))
SMALL = ms.LayerShape("chan", d=256, E=8, k=3, F=128, bias="normal", bias_param=0.7)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    moe.load_library()
    yield
    torch.cuda.synchronize()


def _packed(keep_u8):
    """[B][k][F] 0/1 bytes -> [B][k][F/32] uint32 bit masks (bit f % 32 of word f / 32)."""
    B, k, F = keep_u8.shape
    bits = keep_u8.reshape(B, k, F // 32, 32).astype(np.uint64)
    return (bits << np.arange(32, dtype=np.uint64)).sum(-1).astype(np.uint32)


def _scores(rng, B, k, F, ties):
    s = rng.standard_normal((B, k, F)).astype(np.float32)
    if ties:
        # coarse values: many exact ties, also at the keep boundary
        s = np.round(s * 2.0).astype(np.float32) / 2.0
    return s


def _run(S, B, mode, k0, c, seed, ties=False, L=None):
    L = L if L is not None else ms.make_weights(S, seed)
    x = ms.make_tokens(S, B, seed)
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    sel, w = oracle.reselect(logits, probs, S.k, mode, k0, 0)
    score = _scores(np.random.default_rng(1000 + seed), B, S.k, S.F, ties)
    y_r, keep_r = oracle.ffn_channels(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, score, c, threads=THREADS)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    dims = (B, S.d, S.E, S.k, S.F)
    # every device buffer stays referenced until the kernels have run
    Wg_d, Wu_d, Wdn = (t(L[n].view(np.int16)) for n in ("Wgate", "Wup", "Wdown"))
    WdT = torch.empty(S.E, S.F, S.d, dtype=torch.int16, device="cuda")
    lib = moe.load_library()
    assert lib.moe_down_channel_major(Wdn.data_ptr(), moe.Dims(*dims), WdT.data_ptr(), None) == 0
    nbytes = lib.moe_channels_workspace_bytes(moe.Dims(*dims))
    assert nbytes > 0
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    xd, seld, wd, scd = t(x), t(sel), t(w), t(score)
    y = torch.empty(B, S.d, dtype=torch.float32, device="cuda")
    keep = torch.empty(B, S.k, S.F // 32, dtype=torch.int32, device="cuda")
    st = lib.moe_expert_ffn_channels(xd.data_ptr(), Wg_d.data_ptr(), Wu_d.data_ptr(), WdT.data_ptr(),
                                     moe.Dims(*dims), seld.data_ptr(), wd.data_ptr(), scd.data_ptr(), c,
                                     y.data_ptr(), keep.data_ptr(), ws.data_ptr(), nbytes, None)
    assert st == 0
    torch.cuda.synchronize()
    assert moe.moe_check_error(ws) == 0
    return L, sel, keep.cpu().numpy().view(np.uint32), keep_r, y.cpu().numpy(), y_r, WdT


def test_down_channel_major_is_the_transpose():
    S = shape("q30b")
    L = host_layer("q30b", 0)
    Wdn = torch.from_numpy(L["Wdown"].view(np.int16)).cuda()
    WdT = torch.empty(S.E, S.F, S.d, dtype=torch.int16, device="cuda")
    lib = moe.load_library()
    assert lib.moe_down_channel_major(Wdn.data_ptr(), moe.Dims(1, S.d, S.E, S.k, S.F), WdT.data_ptr(), None) == 0
    torch.cuda.synchronize()
    assert np.array_equal(WdT.cpu().numpy(), np.ascontiguousarray(L["Wdown"].view(np.int16).transpose(0, 2, 1)))


@pytest.mark.parametrize("B,mode,k0", [(1, NONE, 0), (3, OEA, 2), (5, NONE, 0), (8, OEA, 1)])
@pytest.mark.parametrize("c", [1, 17, 64, 128])
@pytest.mark.parametrize("ties", [False, True])
def test_channels_small_shape(B, mode, k0, c, ties):
    L, sel, keep, keep_r, y, y_r, _ = _run(SMALL, B, mode, k0, c, seed=B + c, ties=ties)
    assert np.array_equal(keep, _packed(keep_r) * (sel[:, :, None] >= 0))
    assert_close_y(y, y_r, f"B={B} c={c} ties={ties}")


@pytest.mark.parametrize("B,mode,k0,frac", [(1, NONE, 0, 0.13), (1, OEA, 4, 0.18), (4, NONE, 0, 0.13),
                                            (4, OEA, 4, 0.13), (8, OEA, 4, 0.18)])
def test_channels_q30b(B, mode, k0, frac):
    S = shape("q30b")
    c = int(round(frac * S.F))
    L, sel, keep, keep_r, y, y_r, _ = _run(S, B, mode, k0, c, seed=0, L=host_layer("q30b", 0))
    assert np.array_equal(keep, _packed(keep_r) * (sel[:, :, None] >= 0))
    assert_close_y(y, y_r, f"q30b B={B} c={c}")


def test_channels_q235b_b4():
    S = shape("q235b")
    L, sel, keep, keep_r, y, y_r, _ = _run(S, 4, OEA, 4, 200, seed=0, L=host_layer("q235b", 0))
    assert np.array_equal(keep, _packed(keep_r) * (sel[:, :, None] >= 0))
    assert_close_y(y, y_r, "q235b B=4 c=200")


def test_all_channels_kept_is_the_dense_ffn():
    S = shape("q30b")
    L, sel, keep, keep_r, y, _, _ = _run(S, 2, OEA, 4, S.F, seed=3, L=host_layer("q30b", 0))
    x = ms.make_tokens(S, 2, 3)
    logits, probs, _, _ = oracle.route(x, L["Wg"], L["bias"], S.k)
    s2, w2 = oracle.reselect(logits, probs, S.k, OEA, 4, 0)
    y_dense = oracle.ffn(x, L["Wgate"], L["Wup"], L["Wdown"], s2, w2, threads=THREADS)
    assert_close_y(y, y_dense, "c = d_ff")
