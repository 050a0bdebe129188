"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, computes sizes on the host, and rejects bad arguments with
status codes before anything is launched (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def R():
    from top_kv_span_b200 import build
    build.build()
    from top_kv_span_b200 import reatt
    return reatt


def header_functions():
    src = open(os.path.join(ROOT, "include", "reatt.h")).read()
    return sorted(set(re.findall(r"REATT_API\s+[^;(]*?\b(reatt_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(R):
    declared = header_functions()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(R.lib, name), name
    assert sorted(R.EXPORTS) == declared


def test_dims_struct_layout_matches_header(R):
    # int32 x 10, int64 T, double rope_base, int64 T_cap -> 64 bytes
    assert ctypes.sizeof(R.reatt_dims) == 64
    assert R.reatt_dims.T.offset == 40 and R.reatt_dims.rope_base.offset == 48
    assert R.reatt_dims.T_cap.offset == 56


def test_cache_capacity_checks(R):
    # T_cap below T is rejected everywhere; 0 means dense caches (T rows)
    nbytes = ctypes.c_size_t()
    bad = R.make_dims(B=1, Hq=8, Hkv=2, d=128, C=1, T=1000, G=4, L=16, S=8, k=4, dtype="bf16",
                      rope_base=1e4, T_cap=999)
    assert R.lib.reatt_workspace_bytes(ctypes.byref(bad), ctypes.byref(nbytes)) == R.EINVAL
    ok = R.make_dims(B=1, Hq=8, Hkv=2, d=128, C=1, T=1000, G=4, L=16, S=8, k=4, dtype="bf16",
                     rope_base=1e4, T_cap=4096)
    assert R.lib.reatt_workspace_bytes(ctypes.byref(ok), ctypes.byref(nbytes)) == R.OK
    # appending needs room for C rows past T, and every pointer
    dense = R.make_dims(B=1, Hq=8, Hkv=2, d=128, C=1, T=1000, G=4, L=16, S=8, k=4, dtype="bf16",
                        rope_base=1e4)
    fake = 1 << 20   # never dereferenced: the checks fail first
    assert R.reatt_append_kv(dense, fake, fake, fake, fake, stream=0, check=False) == R.EINVAL
    full = R.make_dims(B=1, Hq=8, Hkv=2, d=128, C=2, T=1000, G=4, L=16, S=8, k=4, dtype="bf16",
                       rope_base=1e4, T_cap=1001)
    assert R.reatt_append_kv(full, fake, fake, fake, fake, stream=0, check=False) == R.EINVAL
    assert R.reatt_append_kv(ok, None, fake, fake, fake, stream=0, check=False) == R.EINVAL
    assert R.reatt_append_kv(ok, fake + 8, fake, fake, fake, stream=0, check=False) == R.EINVAL


def test_status_strings(R):
    for code in range(5):
        assert R.status_string(code)
    assert R.status_string(99) == "unknown status"


def dims(R, **kw):
    base = dict(B=1, Hq=32, Hkv=8, d=128, C=1, T=131072, G=32, L=4096, S=32, k=64, dtype="bf16",
                rope_base=5e5)
    base.update(kw)
    return R.make_dims(**base)


@pytest.mark.parametrize("T,G,L,S,k,C,NS,Wmax", [
    (131072, 32, 4096, 32, 64, 1, 3967, 32 + 64 * 32 + 4096 + 1),
    (4096, 4, 256, 32, 8, 1, 120, 4 + 256 + 256 + 1),
    (100, 32, 4096, 32, 64, 2048, 0, 32 + 2048 + 4096 + 2048),
    (0, 4, 4, 3, 2, 1, 0, 4 + 6 + 4 + 1),
])
def test_host_sizes(R, ora, T, G, L, S, k, C, NS, Wmax):
    d = dims(R, T=T, G=G, L=L, S=S, k=k, C=C)
    assert R.reatt_num_spans(d) == NS == ora.partition(T, G, L, S)[3]
    assert R.reatt_window_max(d) == Wmax
    ws = R.reatt_workspace_bytes(d)
    assert ws % 256 == 0 and ws >= 256


def test_workspace_grows_with_spans(R):
    a = R.reatt_workspace_bytes(dims(R, T=1 << 20))
    b = R.reatt_workspace_bytes(dims(R, T=1 << 22))
    assert b > a


@pytest.mark.parametrize("bad,code", [
    (dict(Hq=30), 1), (dict(B=0), 1), (dict(Hkv=0), 1), (dict(C=0), 1), (dict(S=0), 1),
    (dict(k=-1), 1), (dict(T=-5), 1), (dict(G=-1), 1), (dict(L=-1), 1),
    (dict(rope_base=0.0), 1), (dict(rope_base=float("inf")), 1), (dict(rope_base=float("nan")), 1),
    (dict(d=96), 2), (dict(d=256), 2), (dict(dtype=7), 2), (dict(k=70000), 2),
    (dict(T=1 << 31), 2),
    # window positions past 2^24 are not exact fp32 integers in the RoPE angle
    (dict(S=1 << 14, k=1 << 10), 2),
])
def test_bad_dims_rejected_everywhere(R, bad, code):
    d = dims(R, **bad)
    fake = 0x10000   # never dereferenced: validation fails first
    v = ctypes.c_int64()
    assert R.lib.reatt_num_spans(ctypes.byref(d), ctypes.byref(v)) == code
    assert R.lib.reatt_window_max(ctypes.byref(d), ctypes.byref(v)) == code
    sz = ctypes.c_size_t()
    assert R.lib.reatt_workspace_bytes(ctypes.byref(d), ctypes.byref(sz)) == code
    assert R.reatt_score_spans(d, fake, fake, fake, fake, stream=0, check=False) == code
    assert R.reatt_topk(d, fake, fake, fake, stream=0, check=False) == code
    assert R.reatt_gather_rope(d, fake, fake, fake, fake, fake, fake, fake, fake, stream=0,
                               check=False) == code
    assert R.reatt_attend(d, fake, fake, fake, fake, fake, fake, stream=0, check=False) == code
    assert R.reatt_step(d, fake, fake, fake, fake, fake, fake, fake, fake, stream=0,
                        check=False) == code


def test_null_dims_and_outputs(R):
    assert R.lib.reatt_num_spans(None, None) == 1
    assert R.lib.reatt_num_spans(ctypes.byref(dims(R)), None) == 1
    assert R.lib.reatt_workspace_bytes(ctypes.byref(dims(R)), None) == 1
    st = ctypes.c_int()
    assert R.lib.reatt_workspace_status(None, ctypes.byref(st), None) == 1
    assert R.lib.reatt_fixed_scratch_address(None) == 1


def test_null_and_misaligned_pointers(R):
    d = dims(R)
    A, M = 0x10000, 0x10008   # aligned / misaligned fakes, never dereferenced
    # null required pointers
    assert R.reatt_score_spans(d, None, A, A, A, stream=0, check=False) == 1
    assert R.reatt_score_spans(d, A, None, A, A, stream=0, check=False) == 1
    assert R.reatt_score_spans(d, A, A, None, A, stream=0, check=False) == 1
    assert R.reatt_score_spans(d, A, A, A, None, stream=0, check=False) == 1
    assert R.reatt_topk(d, None, A, A, stream=0, check=False) == 1
    assert R.reatt_topk(d, A, None, A, stream=0, check=False) == 1
    assert R.reatt_topk(d, A, A, None, stream=0, check=False) == 1
    assert R.reatt_attend(d, A, A, A, A, None, A, stream=0, check=False) == 1
    assert R.reatt_step(d, A, A, A, A, A, None, None, A, stream=0, check=False) == 1
    assert R.reatt_step(d, A, A, A, A, A, None, A, None, stream=0, check=False) == 1
    assert R.reatt_gather_rope(d, A, A, A, A, None, A, A, A, stream=0, check=False) == 1
    # misaligned pointers
    assert R.reatt_score_spans(d, M, A, A, A, stream=0, check=False) == 1
    assert R.reatt_score_spans(d, A, M, A, A, stream=0, check=False) == 1
    assert R.reatt_topk(d, A, M, A, stream=0, check=False) == 1
    assert R.reatt_gather_rope(d, A, A, A, A, A, M, A, A, stream=0, check=False) == 1
    assert R.reatt_attend(d, A, A, A, A, M, A, stream=0, check=False) == 1
    assert R.reatt_step(d, A, A, A, A, A, M, A, A, stream=0, check=False) == 1
    assert R.reatt_step(d, A, A, A, A, A, None, A, M, stream=0, check=False) == 1


def test_window_limit_is_two_to_the_24(R):
    # Wmax = G + k*S + L + C: exactly 2^24 is accepted, one more is not
    v = ctypes.c_int64()
    ok = dims(R, G=0, L=0, C=1, S=(1 << 24) - 1, k=1)
    assert R.lib.reatt_window_max(ctypes.byref(ok), ctypes.byref(v)) == R.OK
    assert v.value == 1 << 24
    bad = dims(R, G=0, L=0, C=2, S=(1 << 24) - 1, k=1)
    assert R.lib.reatt_window_max(ctypes.byref(bad), ctypes.byref(v)) == R.EUNSUPPORTED
