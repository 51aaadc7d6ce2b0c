"""Host-side checks of the C ABI that need no GPU: the library loads,
exports every function include/moe_decode.h declares, sizes workspaces,
and rejects bad arguments with the documented status before touching CUDA.

Every call below with fake addresses carries at least one argument that the
host validation rejects, so none of them can reach a kernel launch."""
import ctypes
import os
import re

import pytest
import torch

import aware_expert_routing_moe_b200 as moe
from aware_expert_routing_moe_b200 import Dims, Lists, Rule

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, MISALIGNED, WORKSPACE, UNSUPPORTED, CUDA, INTERNAL = range(7)


@pytest.fixture(scope="module")
def lib():
    from aware_expert_routing_moe_b200 import build
    build.build()
    return moe.load_library()


def _declared_functions():
    with open(os.path.join(ROOT, "include", "moe_decode.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert _declared_functions() == sorted(moe.ABI_SYMBOLS)


def _header_text():
    with open(os.path.join(ROOT, "include", "moe_decode.h")) as f:
        return re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)


def test_binding_structs_and_constants_match_the_header():
    text = _header_text()
    # enum constants: status codes and re-selection modes
    consts = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(MOE_[A-Z_]+)\s*=\s*(\d+)", text)}
    status = {k: v for k, v in consts.items() if k.startswith("MOE_ERR") or k == "MOE_OK"}
    assert {v: k for k, v in moe.STATUS.items()} == status
    for name in ("MOE_RESELECT_NONE", "MOE_RESELECT_OEA", "MOE_RESELECT_XSHARE", "MOE_RESELECT_AFFINITY",
                 "MOE_RESELECT_XSHARE_HIER"):
        assert getattr(moe, name) == consts[name], name
    assert sorted(k for k in consts if k.startswith("MOE_RESELECT_")) == sorted(
        k for k in dir(moe) if k.startswith("MOE_RESELECT_"))
    # struct fields, in order, all 32-bit integers (pointers for the lists)
    def fields(tag):
        body = re.search(r"typedef struct \{([^{}]*)\}\s*" + tag + r"\s*;", text).group(1)
        names = []
        for decl in body.split(";"):
            decl = decl.strip()
            if decl:
                names += [n.strip().lstrip("*") for n in decl.split(None, 1)[1].split(",")]
        return names
    assert fields("moe_dims_t") == [f[0] for f in Dims._fields_]
    assert fields("moe_reselect_t") == [f[0] for f in Rule._fields_]
    assert fields("moe_lists_t") == [f[0] for f in Lists._fields_]
    assert ctypes.sizeof(Rule) == 4 * len(Rule._fields_) and ctypes.sizeof(Dims) == 4 * len(Dims._fields_)
    m = re.search(r"#define MOE_NOALLOC_SCRATCH_BYTES \((\d+)u? \* (\d+)u? \* (\d+)u?\)",
                  open(os.path.join(ROOT, "include", "moe_decode.h")).read())
    if m:
        assert moe.NOALLOC_SCRATCH_BYTES == int(m.group(1)) * int(m.group(2)) * int(m.group(3))


def test_library_exports_every_declared_function(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    seen = set()
    for s in range(7):
        txt = moe.moe_status_string(s)
        assert txt and txt not in seen
        seen.add(txt)
    assert moe.moe_status_string(99) == "unknown status"


def test_workspace_bytes(lib):
    q30 = moe.moe_workspace_bytes(16, 2048, 128, 8, 768)
    assert q30 > 0 and q30 % 256 == 0
    # B <= 64: token-indexed activations [min(E, B*k)][B][d_ff] bf16 + dense weights
    assert q30 >= 128 * 16 * 768 * 2 + 128 * 16 * 4
    q30_64 = moe.moe_workspace_bytes(64, 2048, 128, 8, 768)
    assert q30_64 >= 128 * 64 * 768 * 2 + 128 * 64 * 4
    # larger batches: pair-indexed activations [B*k][d_ff] bf16 + dispatched x rows
    q30_65 = moe.moe_workspace_bytes(65, 2048, 128, 8, 768)
    assert q30_65 >= 65 * 8 * 768 * 2 + 65 * 8 * 2048 * 2
    assert q30_65 < 128 * 65 * 768 * 2
    assert moe.moe_workspace_bytes(16, 4096, 128, 8, 1536) > q30
    for bad in [(0, 2048, 128, 8, 768), (257, 2048, 128, 8, 768), (16, 2048, 128, 0, 768),
                (16, 2048, 128, 17, 768), (16, 2048, 7, 8, 768), (16, 2048, 257, 8, 768),
                (16, 2000, 128, 8, 768), (16, 2048, 128, 8, 700), (16, 32, 128, 8, 768),
                (16, 2048, 128, 8, 32)]:
        assert moe.moe_workspace_bytes(*bad) == 0, bad


A = 0x10000  # fake, 256-byte aligned address (never dereferenced)


def _layer_call(lib, dims=Dims(16, 2048, 128, 8, 768), rule=Rule(1, 4, 0), x=A, Wg=A, bias=A, Wgate=A,
                Wup=A, Wdown=A, y=A, sel=None, selw=None, nact=None, ws=A, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.moe_workspace_bytes(dims) if lib.moe_workspace_bytes(dims) else 1 << 30
    return lib.moe_layer_decode(x, Wg, bias, Wgate, Wup, Wdown, dims, rule, y, sel, selw, nact, ws,
                                ws_bytes, None)


def test_layer_decode_rejects_bad_arguments(lib):
    small = lib.moe_workspace_bytes(Dims(16, 2048, 128, 8, 768)) - 256
    assert _layer_call(lib, dims=Dims(0, 2048, 128, 8, 768)) == INVALID
    assert _layer_call(lib, dims=Dims(16, 2048, 128, 8, 700)) == INVALID
    assert _layer_call(lib, rule=Rule(1, 0, 0)) == INVALID          # k0 < 1
    assert _layer_call(lib, rule=Rule(1, 9, 0)) == INVALID          # k0 > k
    assert _layer_call(lib, rule=Rule(2, 0, 7)) == INVALID          # budget < k
    assert _layer_call(lib, rule=Rule(2, 0, 129)) == INVALID        # budget > E
    assert _layer_call(lib, rule=Rule(5, 0, 0)) == INVALID          # unknown rule
    assert _layer_call(lib, rule=Rule(4, 0, 16, 0)) == INVALID      # hierarchical: group < 1
    assert _layer_call(lib, rule=Rule(4, 0, 16, 257)) == INVALID    # group > 256
    assert _layer_call(lib, rule=Rule(4, 0, 7, 4)) == INVALID       # budget < k
    assert _layer_call(lib, rule=Rule(4, 0, 129, 4)) == INVALID     # budget > E
    assert _layer_call(lib, x=None) == INVALID
    assert _layer_call(lib, Wdown=None) == INVALID
    assert _layer_call(lib, y=None) == INVALID
    assert _layer_call(lib, x=A + 4) == MISALIGNED
    assert _layer_call(lib, Wup=A + 8) == MISALIGNED
    assert _layer_call(lib, bias=A + 2) == MISALIGNED
    assert _layer_call(lib, sel=A + 4) == MISALIGNED
    assert _layer_call(lib, ws=None) == WORKSPACE
    assert _layer_call(lib, ws_bytes=small) == WORKSPACE
    assert _layer_call(lib, ws=A + 16) == MISALIGNED                # workspace wants 256 B


def test_route_and_reselect_reject_bad_arguments(lib):
    d = Dims(16, 2048, 128, 8, 0)
    assert lib.moe_route(None, A, None, d, A, A, A, A, None) == INVALID
    assert lib.moe_route(A, A, None, Dims(16, 2000, 128, 8, 0), A, A, A, A, None) == INVALID
    assert lib.moe_route(A, A, None, Dims(16, 2048, 4, 8, 0), A, A, A, A, None) == INVALID
    assert lib.moe_route(A, A + 4, None, d, A, A, A, A, None) == MISALIGNED
    lists = Lists(A, A, A, A, A)
    assert lib.moe_reselect(A, A, d, Rule(1, 9, 0), A, A, lists, None) == INVALID
    assert lib.moe_reselect(A, A, d, Rule(0, 0, 0), None, A, lists, None) == INVALID
    assert lib.moe_reselect(A, A, d, Rule(0, 0, 0), A, A, Lists(A, None, A, A, A), None) == INVALID
    assert lib.moe_reselect(A, A, d, Rule(0, 0, 0), A, A, Lists(A, A, A + 4, A, A), None) == MISALIGNED
    assert lib.moe_reselect(A, A, Dims(300, 0, 128, 8, 0), Rule(0, 0, 0), A, A, lists, None) == INVALID


def test_expert_ffn_rejects_bad_arguments(lib):
    d = Dims(16, 2048, 128, 8, 768)
    lists = Lists(A, A, A, A, A)
    n = lib.moe_workspace_bytes(d)
    assert lib.moe_expert_ffn(A, A, A, A, Dims(16, 2048, 128, 8, 0), lists, A, A, n, None) == INVALID
    assert lib.moe_expert_ffn(A, None, A, A, d, lists, A, A, n, None) == INVALID
    assert lib.moe_expert_ffn(A, A, A, A, d, Lists(None, A, A, A, A), A, A, n, None) == INVALID
    assert lib.moe_expert_ffn(A, A, A, A + 2, d, lists, A, A, n, None) == MISALIGNED
    assert lib.moe_expert_ffn(A, A, A, A, d, lists, A, A, n - 1, None) == WORKSPACE
    assert lib.moe_check_error(None, 0, None) == WORKSPACE
    assert lib.moe_check_error(A + 16, 1 << 16, None) == MISALIGNED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_cuda_error(lib):
    # all arguments valid: validation passes, the device query fails cleanly
    assert _layer_call(lib) == CUDA
    assert _layer_call(lib, rule=Rule(3, 0, 0)) == CUDA            # affinity binning: no parameters
    assert _layer_call(lib, rule=Rule(4, 0, 16, 4)) == CUDA        # hierarchical XShare
    assert _layer_call(lib, rule=Rule(4, 0, 128, 256)) == CUDA
    assert lib.moe_route(A, A, None, Dims(16, 2048, 128, 8, 0), A, A, A, A, None) == CUDA


def test_binding_raises_on_error(lib):
    with pytest.raises(moe.MoeError) as ei:
        moe._check(MISALIGNED, "x")
    assert ei.value.status == MISALIGNED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_noalloc_size_limit(lib):
    # the static scratch holds both model shapes at every batch size: valid
    # dims pass the size check and only the device query fails here
    lists = Lists(A, A, A, A, A)
    for B in (1, 16, 32, 33, 64, 256):
        for d, F in ((2048, 768), (4096, 1536)):
            st = lib.moe_expert_ffn_noalloc(A, A, A, A, Dims(B, d, 128, 8, F), lists, A, None)
            assert st == CUDA, (B, d, F, st)
    # the largest dims do not fit: rejected before anything is enqueued
    assert lib.moe_expert_ffn_noalloc(A, A, A, A, Dims(256, 16384, 256, 16, 8192), lists, A, None) == UNSUPPORTED
    # invalid dims and misaligned buffers are reported first
    assert lib.moe_expert_ffn_noalloc(A, A, A, A, Dims(257, 2048, 128, 8, 768), lists, A, None) == INVALID
    assert lib.moe_expert_ffn_noalloc(A + 4, A, A, A, Dims(16, 2048, 128, 8, 768), lists, A, None) == MISALIGNED


def test_stack_rejects_bad_arguments(lib):
    # host validation only: every layer is checked before anything is enqueued
    A = 0x10000
    w = (moe.LayerWeights * 2)(moe.LayerWeights(A, 0, A, A, A), moe.LayerWeights(A, 0, 0, A, A))
    d = moe.Dims(16, 2048, 128, 8, 768)
    r = moe.Rule(1, 4, 0, 1)
    assert lib.moe_decode_stack(w, 0, d, r, 0, A, None, None, A, 1 << 30, None) == 1  # no layers
    assert lib.moe_decode_stack(w, 2, d, r, 0, A, None, None, A, 1 << 30, None) == 1  # layer 1 lacks Wgate
    assert lib.moe_decode_stack(w, 1, d, r, 7, A, None, None, A, 1 << 30, None) == 1  # unknown phase
    assert lib.moe_decode_stack(w, 1, d, moe.Rule(1, 9, 0, 1), 0, A, None, None, A, 1 << 30, None) == 1  # k0 > k
    # prefill ignores the decode rule, so an invalid rule passes there
    assert lib.moe_decode_stack(w, 1, d, moe.Rule(1, 9, 0, 1), 1, A + 4, None, None, A, 1 << 30, None) == 2
    assert lib.moe_decode_stack(w, 1, d, r, 0, A + 4, None, None, A, 1 << 30, None) == 2  # misaligned xs


def test_channels_rejects_bad_arguments(lib):
    A = 0x10000
    d = moe.Dims(4, 2048, 128, 8, 768)
    nb = lib.moe_channels_workspace_bytes(d)
    assert nb > 0
    assert lib.moe_channels_workspace_bytes(moe.Dims(9, 2048, 128, 8, 768)) == 0  # B above MOE_CHANNELS_B_MAX
    assert lib.moe_channels_workspace_bytes(moe.Dims(8, 16384, 128, 8, 768)) == 0  # rows exceed shared memory
    call = lambda dims, c, ws=A, n=nb, x=A: lib.moe_expert_ffn_channels(x, A, A, A, dims, A, A, A, c, A, None, ws, n,
                                                                        None)
    assert call(d, 0) == 1            # c < 1
    assert call(d, 769) == 1          # c > d_ff
    assert call(moe.Dims(9, 2048, 128, 8, 768), 10) == 4
    assert call(d, 10, x=A + 4) == 2  # misaligned x
    assert call(d, 10, ws=None) == 3
    assert call(d, 10, n=nb - 1) == 3
    assert lib.moe_down_channel_major(A, moe.Dims(1, 2048, 128, 8, 768), A + 8, None) == 2
