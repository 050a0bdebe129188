"""CPU oracle for the ReAttention top-k span attention step.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the benchmark's ``cpu_baseline`` / ``--impl reference`` legs may import this
package.  The product library (``top_kv_span_b200``) never imports it and
shares no code with it.

The arithmetic lives in ``reatt_oracle.c`` (plain C, fp64); this module only
compiles it with gcc and marshals numpy arrays.  See the header of the C file
for the passages each function follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "reatt_oracle.c")
_LIB = os.path.join(_HERE, "libreatt_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (portable flags: the .so may run on another host)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i32, i64, dbl, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.ora_partition.argtypes = [i64, i32, i32, i32, vp]
            lib.ora_span_scores.argtypes = [i32, i32, i32, i32, i32, i64, i32, i32, i32, i32,
                                            vp, vp, vp]
            lib.ora_span_scores_list.argtypes = [i32, i32, i32, i32, i32, i64, i32, i32, i32, i32,
                                                 vp, vp, vp, i64, vp]
            lib.ora_topk.argtypes = [vp, i64, i32, vp]
            lib.ora_topk.restype = i32
            lib.ora_window.argtypes = [i64, i32, i32, i32, i32, vp, i32, vp]
            lib.ora_window.restype = i64
            lib.ora_rope_row.argtypes = [vp, i32, dbl, dbl]
            lib.ora_step.argtypes = [i32, i32, i32, i32, i32, i64, i32, i32, i32, i32, dbl, i32,
                                     vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp]
            lib.ora_set_threads.argtypes = [i32]
            lib.ora_max_threads.restype = i32
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _raw(x):
    """numpy float32 array, or a bf16 payload given as uint16 bits."""
    a = np.ascontiguousarray(x)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle inputs must be float32 or uint16 (bf16 bits), got {a.dtype}")


def set_threads(n: int) -> None:
    _load().ora_set_threads(int(n))


def max_threads() -> int:
    return int(_load().ora_max_threads())


def partition(T, G, L, S):
    """(global_end, local_begin, M, NS) of the T cached tokens."""
    out = np.zeros(4, np.int64)
    _load().ora_partition(int(T), int(G), int(L), int(S), _ptr(out))
    return tuple(int(v) for v in out)


def span_scores(q, k_cache, G, L, S):
    """Span scores [B,Hkv,NS] (fp64) from q [B,Hq,C,d] and the pre-RoPE key cache [B,Hkv,T,d]."""
    q, dt = _raw(q)
    k_cache, dt2 = _raw(k_cache)
    assert dt == dt2
    B, Hq, C, d = q.shape
    _, Hkv, T, _ = k_cache.shape
    NS = partition(T, G, L, S)[3]
    out = np.zeros((B, Hkv, NS), np.float64)
    _load().ora_span_scores(B, Hq, Hkv, d, C, T, G, L, S, dt, _ptr(q), _ptr(k_cache), _ptr(out))
    return out


def span_scores_list(q, k_cache, G, L, S, pairs):
    """Scores of the listed spans; pairs is an int64 array of (b*Hkv+h, span) rows."""
    q, dt = _raw(q)
    k_cache, _ = _raw(k_cache)
    B, Hq, C, d = q.shape
    _, Hkv, T, _ = k_cache.shape
    pairs = np.ascontiguousarray(pairs, np.int64).reshape(-1, 2)
    out = np.zeros(len(pairs), np.float64)
    _load().ora_span_scores_list(B, Hq, Hkv, d, C, T, G, L, S, dt, _ptr(q), _ptr(k_cache),
                                 _ptr(pairs), len(pairs), _ptr(out))
    return out


def topk(scores, k):
    """Chosen span ids (ascending, -1 padded) of one head's fp64 scores."""
    s = np.ascontiguousarray(scores, np.float64)
    sel = np.zeros(max(k, 1), np.int32)
    _load().ora_topk(_ptr(s), len(s), int(k), _ptr(sel))
    return sel[:k]


def window(T, G, L, S, C, sel):
    """Source rows of the window (cache row, or -(1+c) for current token c)."""
    sel = np.ascontiguousarray(sel, np.int32)
    k = len(sel)
    buf = np.zeros(G + k * S + L + C + 1, np.int64)
    W = _load().ora_window(int(T), G, L, S, C, _ptr(sel), k, _ptr(buf))
    return buf[:W].copy()


def rope_row(x, pos, base):
    """RoPE of one vector (fp64 copy returned)."""
    v = np.array(x, np.float64, copy=True)
    _load().ora_rope_row(_ptr(v), len(v), float(pos), float(base))
    return v


def step(q, k_cache, v_cache, k_cur, v_cur, *, G, L, S, k, rope_base,
         sel=None, c_list=None, want_scores=True):
    """The whole step.  Returns dict(out [B,Hq,C,d] fp64, sel [B,Hkv,k] int32,
    win_len [B,Hkv] int64, scores [B,Hkv,NS] fp64 or None).

    sel: use this selection instead of scoring (attention-only check).
    c_list: compute only these query positions (others stay 0 in out)."""
    q, dt = _raw(q)
    k_cache, _ = _raw(k_cache)
    v_cache, _ = _raw(v_cache)
    k_cur, _ = _raw(k_cur)
    v_cur, _ = _raw(v_cur)
    B, Hq, C, d = q.shape
    _, Hkv, T, _ = k_cache.shape
    NS = partition(T, G, L, S)[3]
    out = np.zeros((B, Hq, C, d), np.float64)
    sel_out = np.zeros((B, Hkv, max(k, 1)), np.int32)[..., :k].copy()
    win = np.zeros((B, Hkv), np.int64)
    scores = np.zeros((B, Hkv, NS), np.float64) if (want_scores and sel is None) else None
    sel_in = None if sel is None else np.ascontiguousarray(sel, np.int32)
    cl = None if c_list is None else np.ascontiguousarray(c_list, np.int32)
    _load().ora_step(B, Hq, Hkv, d, C, T, G, L, S, k, float(rope_base), dt,
                     _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_cur), _ptr(v_cur),
                     _ptr(sel_in), _ptr(sel_out), _ptr(win), _ptr(scores),
                     _ptr(cl), 0 if cl is None else len(cl), _ptr(out))
    return {"out": out, "sel": sel_out, "win_len": win, "scores": scores}
