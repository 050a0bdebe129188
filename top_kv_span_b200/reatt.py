"""Thin ctypes binding of ``libreatt.so`` (the C ABI in ``include/reatt.h``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Functions keep the C names; tensors are passed as device pointers,
the stream defaults to torch's current stream.  Missing library -> ImportError
(there is no fallback of any kind).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libreatt.so")

OK, EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT = 0, 1, 2, 3, 4
F32, BF16 = 0, 1

EXPORTS = ["reatt_status_string", "reatt_num_spans", "reatt_window_max", "reatt_workspace_bytes",
           "reatt_workspace_status", "reatt_score_spans", "reatt_topk", "reatt_gather_rope",
           "reatt_attend", "reatt_step", "reatt_append_kv", "reatt_selftest_bounded_wait",
           "reatt_step_fixed_scratch", "reatt_fixed_scratch_address", "reatt_shard_plan", "reatt_shard_workspace_bytes",
           "reatt_shard_candidates", "reatt_shard_select", "reatt_shard_attend",
           "reatt_merge_partials"]


class reatt_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("C", ctypes.c_int32), ("G", ctypes.c_int32),
                ("L", ctypes.c_int32), ("S", ctypes.c_int32), ("k", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("T", ctypes.c_int64), ("rope_base", ctypes.c_double),
                ("T_cap", ctypes.c_int64)]


class reatt_shard(ctypes.Structure):
    _fields_ = [("t_begin", ctypes.c_int64), ("t_end", ctypes.c_int64),
                ("rows_cap", ctypes.c_int64), ("owns_current", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class ReattError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m top_kv_span_b200.build` "
                      "(nvcc, sm_100a); there is no fallback path")

lib = ctypes.CDLL(LIB_PATH)
_vp, _dp = ctypes.c_void_p, ctypes.POINTER(reatt_dims)
lib.reatt_status_string.restype = ctypes.c_char_p
lib.reatt_status_string.argtypes = [ctypes.c_int]
lib.reatt_num_spans.argtypes = [_dp, ctypes.POINTER(ctypes.c_int64)]
lib.reatt_window_max.argtypes = [_dp, ctypes.POINTER(ctypes.c_int64)]
lib.reatt_workspace_bytes.argtypes = [_dp, ctypes.POINTER(ctypes.c_size_t)]
lib.reatt_workspace_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_int), _vp]
lib.reatt_score_spans.argtypes = [_dp, _vp, _vp, _vp, _vp, _vp]
lib.reatt_topk.argtypes = [_dp, _vp, _vp, _vp, _vp]
lib.reatt_gather_rope.argtypes = [_dp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.reatt_attend.argtypes = [_dp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.reatt_step.argtypes = [_dp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.reatt_step_fixed_scratch.argtypes = [_dp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.reatt_selftest_bounded_wait.argtypes = [_vp, ctypes.c_int64, _vp]
lib.reatt_append_kv.argtypes = [_dp, _vp, _vp, _vp, _vp, _vp]
_sp = ctypes.POINTER(reatt_shard)
lib.reatt_shard_plan.argtypes = [_dp, ctypes.c_int32, _sp]
lib.reatt_shard_workspace_bytes.argtypes = [_dp, _sp, ctypes.c_int32,
                                            ctypes.POINTER(ctypes.c_size_t)]
lib.reatt_shard_candidates.argtypes = [_dp, _sp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.reatt_shard_select.argtypes = [_dp, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp]
lib.reatt_shard_attend.argtypes = [_dp, _sp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.reatt_merge_partials.argtypes = [_dp, ctypes.c_int32, _vp, _vp, _vp, _vp]
for _name in EXPORTS[1:]:
    getattr(lib, _name).restype = ctypes.c_int


def status_string(code: int) -> str:
    return lib.reatt_status_string(int(code)).decode()


def make_dims(B, Hq, Hkv, d, C, T, G, L, S, k, dtype, rope_base, T_cap=0) -> reatt_dims:
    if isinstance(dtype, str):
        dtype = F32 if dtype == "f32" else BF16
    elif isinstance(dtype, torch.dtype):
        dtype = F32 if dtype == torch.float32 else BF16
    return reatt_dims(int(B), int(Hq), int(Hkv), int(d), int(C), int(G), int(L), int(S), int(k),
                      int(dtype), int(T), float(rope_base), int(T_cap))


def dims_of(w, **override) -> reatt_dims:
    """Dims of a ``workloads.Workload`` (fields may be overridden)."""
    f = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, C=w.C, T=w.T, G=w.G, L=w.L, S=w.S, k=w.k,
             dtype=w.dtype, rope_base=w.rope_base)
    f.update(override)
    return make_dims(**f)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc, where):
    if rc != OK:
        raise ReattError(rc, where)


def reatt_num_spans(dims) -> int:
    v = ctypes.c_int64()
    _check(lib.reatt_num_spans(ctypes.byref(dims), ctypes.byref(v)), "reatt_num_spans")
    return v.value


def reatt_window_max(dims) -> int:
    v = ctypes.c_int64()
    _check(lib.reatt_window_max(ctypes.byref(dims), ctypes.byref(v)), "reatt_window_max")
    return v.value


def reatt_workspace_bytes(dims) -> int:
    v = ctypes.c_size_t()
    _check(lib.reatt_workspace_bytes(ctypes.byref(dims), ctypes.byref(v)),
           "reatt_workspace_bytes")
    return v.value


def reatt_workspace_status(ws, stream=None) -> int:
    v = ctypes.c_int()
    _check(lib.reatt_workspace_status(_ptr(ws), ctypes.byref(v), _stream(stream)),
           "reatt_workspace_status")
    return v.value


def reatt_score_spans(dims, q, k_cache, span_scores, ws, stream=None, check=True):
    rc = lib.reatt_score_spans(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(span_scores),
                               _ptr(ws), _stream(stream))
    if check:
        _check(rc, "reatt_score_spans")
    return rc


def reatt_topk(dims, span_scores, sel, ws, stream=None, check=True):
    rc = lib.reatt_topk(ctypes.byref(dims), _ptr(span_scores), _ptr(sel), _ptr(ws),
                        _stream(stream))
    if check:
        _check(rc, "reatt_topk")
    return rc


def reatt_gather_rope(dims, k_cache, v_cache, k_cur, v_cur, sel, k_win, v_win, win_len,
                      stream=None, check=True):
    rc = lib.reatt_gather_rope(ctypes.byref(dims), _ptr(k_cache), _ptr(v_cache), _ptr(k_cur),
                               _ptr(v_cur), _ptr(sel), _ptr(k_win), _ptr(v_win), _ptr(win_len),
                               _stream(stream))
    if check:
        _check(rc, "reatt_gather_rope")
    return rc


def reatt_attend(dims, q, k_win, v_win, win_len, out, ws, stream=None, check=True):
    rc = lib.reatt_attend(ctypes.byref(dims), _ptr(q), _ptr(k_win), _ptr(v_win), _ptr(win_len),
                          _ptr(out), _ptr(ws), _stream(stream))
    if check:
        _check(rc, "reatt_attend")
    return rc


def reatt_step(dims, q, k_cache, v_cache, k_cur, v_cur, sel_out, out, ws, stream=None,
               check=True):
    rc = lib.reatt_step(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_cur),
                        _ptr(v_cur), _ptr(sel_out), _ptr(out), _ptr(ws), _stream(stream))
    if check:
        _check(rc, "reatt_step")
    return rc


def reatt_append_kv(dims, k_cache, v_cache, k_cur, v_cur, stream=None, check=True):
    rc = lib.reatt_append_kv(ctypes.byref(dims), _ptr(k_cache), _ptr(v_cache), _ptr(k_cur),
                             _ptr(v_cur), _stream(stream))
    if check:
        _check(rc, "reatt_append_kv")
    return rc


def reatt_selftest_bounded_wait(ws, limit_ns, stream=None, check=True):
    """Run one bounded wait that nothing completes; the timeout lands in the
    workspace status word (read it with reatt_workspace_status)."""
    rc = lib.reatt_selftest_bounded_wait(_ptr(ws), int(limit_ns), _stream(stream))
    if check:
        _check(rc, "reatt_selftest_bounded_wait")
    return rc


def reatt_step_fixed_scratch(dims, q, k_cache, v_cache, k_cur, v_cur, sel_out, out, stream=None,
                             check=True):
    """reatt_step with the library's fixed 16 MiB device scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    rc = lib.reatt_step_fixed_scratch(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(k_cur), _ptr(v_cur), _ptr(sel_out), _ptr(out),
                                      _stream(stream))
    if check:
        _check(rc, "reatt_step_fixed_scratch")
    return rc


def reatt_fixed_scratch_address() -> int:
    """Device address of the fixed scratch on the current device, for
    reatt_workspace_status (its status word) and the bounded-wait selftest."""
    p = ctypes.c_void_p()
    _check(lib.reatt_fixed_scratch_address(ctypes.byref(p)), "reatt_fixed_scratch_address")
    return int(p.value)


def reatt_shard_plan(dims, n):
    """n contiguous shards of the sequence's tokens (list of reatt_shard)."""
    arr = (reatt_shard * int(n))()
    _check(lib.reatt_shard_plan(ctypes.byref(dims), int(n), arr), "reatt_shard_plan")
    return list(arr)


def reatt_shard_workspace_bytes(dims, shard, n_shards) -> int:
    v = ctypes.c_size_t()
    _check(lib.reatt_shard_workspace_bytes(ctypes.byref(dims), ctypes.byref(shard),
                                           int(n_shards), ctypes.byref(v)),
           "reatt_shard_workspace_bytes")
    return v.value


def reatt_shard_candidates(dims, shard, q, k_cache, cand_score, cand_id, ws, stream=None,
                           check=True):
    rc = lib.reatt_shard_candidates(ctypes.byref(dims), ctypes.byref(shard), _ptr(q),
                                    _ptr(k_cache), _ptr(cand_score), _ptr(cand_id), _ptr(ws),
                                    _stream(stream))
    if check:
        _check(rc, "reatt_shard_candidates")
    return rc


def reatt_shard_select(dims, n_shards, cand_score_all, cand_id_all, sel, ws, stream=None,
                       check=True):
    rc = lib.reatt_shard_select(ctypes.byref(dims), int(n_shards), _ptr(cand_score_all),
                                _ptr(cand_id_all), _ptr(sel), _ptr(ws), _stream(stream))
    if check:
        _check(rc, "reatt_shard_select")
    return rc


def reatt_shard_attend(dims, shard, q, k_cache, v_cache, k_cur, v_cur, sel, part_ml, part_acc,
                       ws, stream=None, check=True):
    rc = lib.reatt_shard_attend(ctypes.byref(dims), ctypes.byref(shard), _ptr(q), _ptr(k_cache),
                                _ptr(v_cache), _ptr(k_cur), _ptr(v_cur), _ptr(sel),
                                _ptr(part_ml), _ptr(part_acc), _ptr(ws), _stream(stream))
    if check:
        _check(rc, "reatt_shard_attend")
    return rc


def reatt_merge_partials(dims, n_parts, part_ml_all, part_acc_all, out, stream=None,
                         check=True):
    rc = lib.reatt_merge_partials(ctypes.byref(dims), int(n_parts), _ptr(part_ml_all),
                                  _ptr(part_acc_all), _ptr(out), _stream(stream))
    if check:
        _check(rc, "reatt_merge_partials")
    return rc


# ----------------------------------------------------------------- convenience
def alloc_outputs(dims, device="cuda"):
    """Caller-side buffers for one call of every entry point (torch allocates)."""
    NS = reatt_num_spans(dims)
    Wmax = reatt_window_max(dims)
    BH = dims.B * dims.Hkv
    ws_bytes = reatt_workspace_bytes(dims)
    return dict(
        span_scores=torch.empty((dims.B, dims.Hkv, NS), dtype=torch.float32, device=device),
        sel=torch.empty((dims.B, dims.Hkv, dims.k), dtype=torch.int32, device=device),
        k_win=torch.zeros((dims.B, dims.Hkv, Wmax, dims.d), dtype=torch.float32, device=device),
        v_win=torch.zeros((dims.B, dims.Hkv, Wmax, dims.d), dtype=torch.float32, device=device),
        win_len=torch.empty((dims.B, dims.Hkv), dtype=torch.int32, device=device),
        out=torch.empty((dims.B, dims.Hq, dims.C, dims.d), dtype=torch.float32, device=device),
        ws=torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=device),
    )
