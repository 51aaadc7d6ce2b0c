"""CPU oracle for the decode-time MoE layer with batch-aware re-routing.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference leg of ``bench.py`` may import this package.
The product library never imports, links or calls it.

``moe_oracle.c`` holds the arithmetic; this module compiles it with gcc
(``-O2 -ffp-contract=off -fno-fast-math -fopenmp``) into
``oracle/libmoe_oracle.so`` and marshals NumPy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

MODE_NONE, MODE_OEA, MODE_XSHARE, MODE_AFFINITY, MODE_XSHARE_HIER = 0, 1, 2, 3, 4

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (idempotent)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_exp_spec.restype = ctypes.c_float
        lib.oracle_exp_spec.argtypes = [ctypes.c_float]
        lib.oracle_exp_spec_n.restype = None
        lib.oracle_exp_spec_n.argtypes = [P, P, I]
        lib.oracle_canon_dot.restype = ctypes.c_float
        lib.oracle_canon_dot.argtypes = [P, P, I]
        lib.oracle_canon_sum.restype = ctypes.c_float
        lib.oracle_canon_sum.argtypes = [P, I]
        lib.oracle_route.restype = None
        lib.oracle_route.argtypes = [P, P, P, I, I, I, I, P, P, P, P]
        lib.oracle_reselect.restype = None
        lib.oracle_reselect.argtypes = [P, P, I, I, I, I, I, I, I, P, P]
        lib.oracle_lists.restype = I
        lib.oracle_lists.argtypes = [P, P, I, I, I, P, P, P, P]
        lib.oracle_ffn.restype = None
        lib.oracle_ffn.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P, I, I, P]
        lib.oracle_ffn_channels.restype = None
        lib.oracle_ffn_channels.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P, I, P, I, I, P, P]
        lib.oracle_channel_sector_bytes.restype = ctypes.c_longlong
        lib.oracle_channel_sector_bytes.argtypes = [P, P, I, I, I, I, I, I]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def exp_spec(x) -> np.ndarray:
    """Element-wise exp_spec over a float32 array (for pins)."""
    lib = _load()
    xs = _c(x, np.float32).ravel()
    out = np.empty_like(xs)
    lib.oracle_exp_spec_n(_p(xs), _p(out), xs.size)
    return out.reshape(np.shape(x))


def canon_dot(a, b) -> np.float32:
    lib = _load()
    a = _c(a, np.float32)
    b = _c(b, np.float32)
    assert a.shape == b.shape and a.ndim == 1 and a.size % 8 == 0
    return np.float32(lib.oracle_canon_dot(_p(a), _p(b), a.size))


def canon_sum(q) -> np.float32:
    lib = _load()
    q = _c(q, np.float32)
    return np.float32(lib.oracle_canon_sum(_p(q), q.size))


def route(x, Wg, bias, k: int):
    """-> logits[B][E], probs[B][E] fp32, topk_idx[B][k] int32, topk_w[B][k] fp32."""
    lib = _load()
    x = _c(x, np.float32)
    Wg = _c(Wg, np.float32)
    B, d = x.shape
    E = Wg.shape[0]
    assert Wg.shape == (E, d)
    bp = None
    if bias is not None:
        bias = _c(bias, np.float32)
        assert bias.shape == (E,)
        bp = _p(bias)
    logits = np.empty((B, E), np.float32)
    probs = np.empty((B, E), np.float32)
    ti = np.empty((B, k), np.int32)
    tw = np.empty((B, k), np.float32)
    lib.oracle_route(_p(x), _p(Wg), bp, B, d, E, k, _p(logits), _p(probs), _p(ti), _p(tw))
    return logits, probs, ti, tw


def reselect(logits, probs, k: int, mode: int, k0: int = 0, budget: int = 0, group: int = 1):
    """-> sel_idx[B][k] int32 (-1 padded), sel_w[B][k] fp32.  ``group``:
    tokens per request (MODE_XSHARE_HIER only)."""
    lib = _load()
    logits = _c(logits, np.float32)
    probs = _c(probs, np.float32)
    B, E = logits.shape
    sel = np.empty((B, k), np.int32)
    w = np.empty((B, k), np.float32)
    assert group >= 1
    lib.oracle_reselect(_p(logits), _p(probs), B, E, k, mode, k0, budget, group, _p(sel), _p(w))
    return sel, w


def lists(sel_idx, sel_w, E: int):
    """-> dict(n_active, active[E], offsets[E+1], tok[B*k], w[B*k])."""
    lib = _load()
    sel_idx = _c(sel_idx, np.int32)
    sel_w = _c(sel_w, np.float32)
    B, k = sel_idx.shape
    active = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    tok = np.empty(B * k, np.int32)
    w = np.empty(B * k, np.float32)
    n = lib.oracle_lists(_p(sel_idx), _p(sel_w), B, E, k, _p(active), _p(offsets), _p(tok), _p(w))
    return {"n_active": int(n), "active": active, "offsets": offsets, "tok": tok, "w": w}


def ffn(x, Wgate, Wup, Wdown, sel_idx, sel_w, rows=None, threads: int = 1) -> np.ndarray:
    """-> y[len(rows) or B][d] fp64 for the chosen experts of each token."""
    lib = _load()
    x = _c(x, np.float32)
    Wgate = _c(Wgate, np.uint16)
    Wup = _c(Wup, np.uint16)
    Wdown = _c(Wdown, np.uint16)
    sel_idx = _c(sel_idx, np.int32)
    sel_w = _c(sel_w, np.float32)
    B, d = x.shape
    E, F, _ = Wgate.shape
    k = sel_idx.shape[1]
    if rows is None:
        rp, nr = None, B
    else:
        rows = _c(rows, np.int32)
        rp, nr = _p(rows), rows.size
    y = np.empty((nr, d), np.float64)
    lib.oracle_ffn(_p(x), _p(Wgate), _p(Wup), _p(Wdown), B, d, E, k, F,
                   _p(sel_idx), _p(sel_w), rp, nr, int(threads), _p(y))
    return y


def ffn_channels(x, Wgate, Wup, Wdown, sel_idx, sel_w, score, c: int, rows=None, threads: int = 1):
    """Expert FFN with per-(token, slot) channel top-k: each pair keeps the
    c channels with the largest ``score[b][s][f]`` (ties to the lower
    index).  -> (y[len(rows) or B][d] fp64, keep[B][k][F] uint8)."""
    lib = _load()
    x = _c(x, np.float32)
    Wgate = _c(Wgate, np.uint16)
    Wup = _c(Wup, np.uint16)
    Wdown = _c(Wdown, np.uint16)
    sel_idx = _c(sel_idx, np.int32)
    sel_w = _c(sel_w, np.float32)
    score = _c(score, np.float32)
    B, d = x.shape
    E, F, _ = Wgate.shape
    k = sel_idx.shape[1]
    assert score.shape == (B, k, F) and 1 <= c <= F
    if rows is None:
        rp, nr = None, B
    else:
        rows = _c(rows, np.int32)
        rp, nr = _p(rows), rows.size
    y = np.empty((nr, d), np.float64)
    keep = np.empty((B, k, F), np.uint8)
    lib.oracle_ffn_channels(_p(x), _p(Wgate), _p(Wup), _p(Wdown), B, d, E, k, F, _p(sel_idx), _p(sel_w),
                            _p(score), int(c), rp, nr, int(threads), _p(y), _p(keep))
    return y, keep


def channel_sector_bytes(keep, sel_idx, E: int, d: int, down_channel_major: bool = False) -> int:
    """Expert-weight bytes one call reads under channel top-k, counted in
    whole 32-byte sectors (see moe_oracle.c)."""
    lib = _load()
    keep = _c(keep, np.uint8)
    sel_idx = _c(sel_idx, np.int32)
    B, k, F = keep.shape
    return int(lib.oracle_channel_sector_bytes(_p(keep), _p(sel_idx), B, E, k, d, F, int(down_channel_major)))


def layer(x, L: dict, k: int, mode: int, k0: int = 0, budget: int = 0,
          rows=None, threads: int = 1, group: int = 1):
    """Whole layer: route -> reselect -> lists -> FFN.  ``L`` holds the
    arrays of ``moe_synth.make_weights``."""
    logits, probs, ti, tw = route(x, L["Wg"], L.get("bias"), k)
    sel, w = reselect(logits, probs, k, mode, k0, budget, group)
    li = lists(sel, w, L["Wg"].shape[0])
    y = ffn(x, L["Wgate"], L["Wup"], L["Wdown"], sel, w, rows=rows, threads=threads)
    return {"logits": logits, "probs": probs, "topk_idx": ti, "topk_w": tw,
            "sel_idx": sel, "sel_w": w, "lists": li, "y": y}
