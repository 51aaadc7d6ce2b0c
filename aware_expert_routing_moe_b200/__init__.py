"""Python binding of libmoe_decode.so: the decode-time MoE layer with
batch-aware expert re-routing on one B200.

This module only marshals arguments: torch tensors supply device memory and
the current CUDA stream; every step of the layer runs in the library's CUDA
kernels.  There is no fallback: if the shared library is missing or was not
built for this machine, importing the binding's functions raises.

Entry points mirror the C ABI in include/moe_decode.h:
``moe_route``, ``moe_reselect``, ``moe_expert_ffn``, ``moe_layer_decode``,
``moe_workspace_bytes``, ``moe_check_error``, ``moe_status_string``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MOE_RESELECT_NONE", "MOE_RESELECT_OEA", "MOE_RESELECT_XSHARE", "MOE_RESELECT_AFFINITY",
    "MOE_RESELECT_XSHARE_HIER", "MoeError",
    "Dims", "Rule", "Lists", "load_library", "library_path", "moe_workspace_bytes",
    "moe_status_string", "moe_route", "moe_reselect", "moe_expert_ffn", "moe_layer_decode",
    "moe_check_error", "moe_expert_ffn_noalloc", "new_workspace", "alloc_lists", "ABI_SYMBOLS",
    "NOALLOC_SCRATCH_BYTES", "moe_set_wait_limit_ns", "moe_decode_stack", "LayerWeights",
    "MOE_PHASE_DECODE", "MOE_PHASE_PREFILL", "moe_down_channel_major", "moe_expert_ffn_channels",
]

MOE_RESELECT_NONE, MOE_RESELECT_OEA, MOE_RESELECT_XSHARE = 0, 1, 2
MOE_RESELECT_AFFINITY, MOE_RESELECT_XSHARE_HIER = 3, 4
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_MISALIGNED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_UNSUPPORTED", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_INTERNAL"}
ABI_SYMBOLS = ("moe_workspace_bytes", "moe_route", "moe_reselect", "moe_expert_ffn",
               "moe_layer_decode", "moe_expert_ffn_noalloc", "moe_check_error", "moe_status_string",
               "moe_set_wait_limit_ns", "moe_decode_stack", "moe_down_channel_major",
               "moe_channels_workspace_bytes", "moe_expert_ffn_channels")
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoe_decode.so")
_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({moe_status_string(status)})")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("d_ff", ctypes.c_int32)]


class Rule(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("k0", ctypes.c_int32), ("budget", ctypes.c_int32),
                ("group", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("Wg", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("Wgate", ctypes.c_void_p),
                ("Wup", ctypes.c_void_p), ("Wdown", ctypes.c_void_p)]


class Lists(ctypes.Structure):
    _fields_ = [("n_active", ctypes.c_void_p), ("active", ctypes.c_void_p),
                ("offsets", ctypes.c_void_p), ("tok", ctypes.c_void_p), ("w", ctypes.c_void_p)]


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libmoe_decode.so (raises OSError if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise OSError(f"{_LIB_PATH} not built: run `python -m aware_expert_routing_moe_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.c_size_t
        lib.moe_workspace_bytes.restype = S
        lib.moe_workspace_bytes.argtypes = [Dims]
        lib.moe_status_string.restype = ctypes.c_char_p
        lib.moe_status_string.argtypes = [ctypes.c_int]
        lib.moe_route.restype = ctypes.c_int
        lib.moe_route.argtypes = [P, P, P, Dims, P, P, P, P, P]
        lib.moe_reselect.restype = ctypes.c_int
        lib.moe_reselect.argtypes = [P, P, Dims, Rule, P, P, Lists, P]
        lib.moe_expert_ffn.restype = ctypes.c_int
        lib.moe_expert_ffn.argtypes = [P, P, P, P, Dims, Lists, P, P, S, P]
        lib.moe_layer_decode.restype = ctypes.c_int
        lib.moe_layer_decode.argtypes = [P, P, P, P, P, P, Dims, Rule, P, P, P, P, P, S, P]
        lib.moe_expert_ffn_noalloc.restype = ctypes.c_int
        lib.moe_expert_ffn_noalloc.argtypes = [P, P, P, P, Dims, Lists, P, P]
        lib.moe_check_error.restype = ctypes.c_int
        lib.moe_check_error.argtypes = [P, S, P]
        lib.moe_decode_stack.restype = ctypes.c_int
        lib.moe_decode_stack.argtypes = [ctypes.POINTER(LayerWeights), ctypes.c_int32, Dims, Rule, ctypes.c_int32,
                                         P, P, P, P, S, P]
        lib.moe_down_channel_major.restype = ctypes.c_int
        lib.moe_down_channel_major.argtypes = [P, Dims, P, P]
        lib.moe_channels_workspace_bytes.restype = S
        lib.moe_channels_workspace_bytes.argtypes = [Dims]
        lib.moe_expert_ffn_channels.restype = ctypes.c_int
        lib.moe_expert_ffn_channels.argtypes = [P, P, P, P, Dims, P, P, P, ctypes.c_int32, P, P, P, S, P]
        lib.moe_set_wait_limit_ns.restype = None
        lib.moe_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        _lib = lib
    return _lib


def moe_status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise MoeError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return int(t)  # raw address, for boundary tests
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def dims(B: int, d: int, E: int, k: int, d_ff: int) -> Dims:
    return Dims(B, d, E, k, d_ff)


def moe_workspace_bytes(B: int, d: int, E: int, k: int, d_ff: int) -> int:
    return int(load_library().moe_workspace_bytes(Dims(B, d, E, k, d_ff)))


def new_workspace(B: int, d: int, E: int, k: int, d_ff: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace (uint8) of moe_workspace_bytes() bytes."""
    n = moe_workspace_bytes(B, d, E, k, d_ff)
    if n == 0:
        raise MoeError(1, "moe_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def alloc_lists(B: int, E: int, k: int, device="cuda") -> dict:
    i32 = dict(dtype=torch.int32, device=device)
    return {"n_active": torch.empty(4, **i32), "active": torch.empty(E, **i32),
            "offsets": torch.empty(E + 1, **i32), "tok": torch.empty(B * k, **i32),
            "w": torch.empty(B * k, dtype=torch.float32, device=device)}


def _lists(l: dict) -> Lists:
    return Lists(_ptr(l["n_active"]), _ptr(l["active"]), _ptr(l["offsets"]), _ptr(l["tok"]), _ptr(l["w"]))


def moe_route(x, Wg, bias, k: int, out=None, stream=None):
    """-> (logits[B][E], probs[B][E], topk_idx[B][k], topk_w[B][k])."""
    B, d = x.shape
    E = Wg.shape[0]
    if out is None:
        out = (torch.empty(B, E, dtype=torch.float32, device=x.device),
               torch.empty(B, E, dtype=torch.float32, device=x.device),
               torch.empty(B, k, dtype=torch.int32, device=x.device),
               torch.empty(B, k, dtype=torch.float32, device=x.device))
    logits, probs, ti, tw = out
    st = load_library().moe_route(_ptr(x), _ptr(Wg), _ptr(bias), Dims(B, d, E, k, 0), _ptr(logits),
                                  _ptr(probs), _ptr(ti), _ptr(tw), _stream(stream))
    _check(st, "moe_route")
    return logits, probs, ti, tw


def moe_reselect(logits, probs, k: int, mode: int, k0: int = 0, budget: int = 0,
                 out=None, lists=None, stream=None, group: int = 1):
    """-> (sel_idx[B][k], sel_w[B][k], lists dict).  ``group``: tokens per
    request (hierarchical XShare)."""
    B, E = logits.shape
    if out is None:
        out = (torch.empty(B, k, dtype=torch.int32, device=logits.device),
               torch.empty(B, k, dtype=torch.float32, device=logits.device))
    if lists is None:
        lists = alloc_lists(B, E, k, logits.device)
    sel, w = out
    st = load_library().moe_reselect(_ptr(logits), _ptr(probs), Dims(B, 0, E, k, 0),
                                     Rule(mode, k0, budget, group),
                                     _ptr(sel), _ptr(w), _lists(lists), _stream(stream))
    _check(st, "moe_reselect")
    return sel, w, lists


def moe_expert_ffn(x, Wgate, Wup, Wdown, lists: dict, k: int, ws, y=None, stream=None):
    """-> y[B][d] fp32 (overwritten)."""
    B, d = x.shape
    E, F, _ = Wgate.shape
    if y is None:
        y = torch.empty(B, d, dtype=torch.float32, device=x.device)
    st = load_library().moe_expert_ffn(_ptr(x), _ptr(Wgate), _ptr(Wup), _ptr(Wdown), Dims(B, d, E, k, F),
                                       _lists(lists), _ptr(y), _ptr(ws), ws.numel() * ws.element_size()
                                       if isinstance(ws, torch.Tensor) else 0, _stream(stream))
    _check(st, "moe_expert_ffn")
    return y


def moe_layer_decode(x, Wg, bias, Wgate, Wup, Wdown, k: int, mode: int, k0: int = 0, budget: int = 0,
                     ws=None, y=None, sel_idx=None, sel_w=None, n_active=None, stream=None, group: int = 1):
    """Whole layer; -> y[B][d] fp32.  Optional device outputs sel_idx[B][k],
    sel_w[B][k], n_active[1] are filled when given."""
    B, d = x.shape
    E, F, _ = Wgate.shape
    if ws is None:
        ws = new_workspace(B, d, E, k, F, x.device)
    if y is None:
        y = torch.empty(B, d, dtype=torch.float32, device=x.device)
    st = load_library().moe_layer_decode(
        _ptr(x), _ptr(Wg), _ptr(bias), _ptr(Wgate), _ptr(Wup), _ptr(Wdown), Dims(B, d, E, k, F),
        Rule(mode, k0, budget, group), _ptr(y), _ptr(sel_idx), _ptr(sel_w), _ptr(n_active), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "moe_layer_decode")
    return y


MOE_PHASE_DECODE, MOE_PHASE_PREFILL = 0, 1


def moe_decode_stack(xs, layers, k: int, mode: int, k0: int = 0, budget: int = 0, phase: int = MOE_PHASE_DECODE,
                     ws=None, sel_idx=None, n_active=None, stream=None, group: int = 1):
    """n_layers residual MoE layers: xs[l + 1] = xs[l] + layer_l(xs[l]).
    ``xs``: [n_layers + 1][B][d] fp32 device tensor, xs[0] the input;
    ``layers``: list of (Wg, bias, Wgate, Wup, Wdown) device tensors.
    Optional device outputs sel_idx[n_layers][B][k], n_active[n_layers].
    -> xs."""
    n = len(layers)
    _, B, d = xs.shape
    E, F, _ = layers[0][2].shape
    if ws is None:
        ws = new_workspace(B, d, E, k, F, xs.device)
    arr = (LayerWeights * n)(*[LayerWeights(_ptr(Wg), _ptr(bias), _ptr(g), _ptr(u), _ptr(dn))
                               for (Wg, bias, g, u, dn) in layers])
    st = load_library().moe_decode_stack(arr, n, Dims(B, d, E, k, F), Rule(mode, k0, budget, group), int(phase),
                                         _ptr(xs), _ptr(sel_idx), _ptr(n_active), _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "moe_decode_stack")
    return xs


def moe_down_channel_major(Wdown, out=None, stream=None):
    """Channel-major copy of the down weights: out[E][d_ff][d] = Wdown[E][d][d_ff]
    transposed per expert (bf16 bits as int16/uint16 tensors)."""
    E, d, F = Wdown.shape
    if out is None:
        out = torch.empty(E, F, d, dtype=Wdown.dtype, device=Wdown.device)
    st = load_library().moe_down_channel_major(_ptr(Wdown), Dims(1, d, E, 1, F), _ptr(out), _stream(stream))
    _check(st, "moe_down_channel_major")
    return out


def moe_expert_ffn_channels(x, Wgate, Wup, WdownT, sel_idx, sel_w, score, c: int, y=None, keep=None, ws=None,
                            stream=None):
    """Expert FFN where each (token, slot) keeps its c highest-scoring
    channels (score[B][k][d_ff]); WdownT from moe_down_channel_major.
    -> y[B][d] fp32.  ``keep``: optional [B][k][d_ff/32] int32 output."""
    B, d = x.shape
    E, F, _ = Wgate.shape
    k = sel_idx.shape[1]
    lib = load_library()
    dims = Dims(B, d, E, k, F)
    n = int(lib.moe_channels_workspace_bytes(dims))
    if n == 0:
        raise MoeError(4, "moe_channels_workspace_bytes")
    if ws is None:
        ws = torch.zeros(n, dtype=torch.uint8, device=x.device)
    if y is None:
        y = torch.empty(B, d, dtype=torch.float32, device=x.device)
    st = lib.moe_expert_ffn_channels(_ptr(x), _ptr(Wgate), _ptr(Wup), _ptr(WdownT), dims, _ptr(sel_idx),
                                     _ptr(sel_w), _ptr(score), int(c), _ptr(y), _ptr(keep), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "moe_expert_ffn_channels")
    return y


def moe_expert_ffn_noalloc(x, Wgate, Wup, Wdown, lists: dict, k: int, y=None, stream=None):
    """moe_expert_ffn without a workspace, for callers that cannot allocate
    device memory: the library's static 32 MiB device scratch is used instead
    (shared by all calls on a device; overlapping calls race).  -> y[B][d]."""
    B, d = x.shape
    E, F, _ = Wgate.shape
    if y is None:
        y = torch.empty(B, d, dtype=torch.float32, device=x.device)
    st = load_library().moe_expert_ffn_noalloc(_ptr(x), _ptr(Wgate), _ptr(Wup), _ptr(Wdown),
                                               Dims(B, d, E, k, F), _lists(lists), _ptr(y), _stream(stream))
    _check(st, "moe_expert_ffn_noalloc")
    return y


def moe_set_wait_limit_ns(ns: int) -> None:
    """Limit of the kernels' bounded waits for later launches (0 = 1 s)."""
    load_library().moe_set_wait_limit_ns(int(ns))


def moe_check_error(ws, stream=None) -> int:
    """Synchronise and return the status of kernels' error word (0 = ok)."""
    return int(load_library().moe_check_error(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
