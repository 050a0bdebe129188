"""Host side of the sharded step, without a GPU: the shard planner's splits
and the argument checks of the shard calls (nothing is launched)."""
import ctypes

import pytest

import oracle


@pytest.fixture(scope="module")
def R():
    from top_kv_span_b200 import build
    build.build()
    from top_kv_span_b200 import reatt
    return reatt


def dims(R, **kw):
    base = dict(B=1, Hq=32, Hkv=8, d=128, C=1, T=131072, G=32, L=4096, S=32, k=64,
                dtype="bf16", rope_base=5e5)
    base.update(kw)
    return R.make_dims(**base)


@pytest.mark.parametrize("T,G,L,S,n", [
    (131072, 32, 4096, 32, 2), (131072, 32, 4096, 32, 8), (4194304, 32, 4096, 32, 4),
    (20003, 32, 512, 32, 3), (1003, 3, 17, 7, 5), (100, 32, 4096, 32, 3), (0, 4, 4, 3, 2),
    (5000, 0, 0, 1, 7), (700, 4, 64, 16, 64),
])
def test_plan_covers_tokens_on_span_boundaries(R, T, G, L, S, n):
    d = dims(R, T=T, G=G, L=L, S=S)
    shards = R.reatt_shard_plan(d, n)
    assert len(shards) == n
    _, _, M, NS = oracle.partition(T, G, L, S)
    prev = 0
    counts = []
    for r, sh in enumerate(shards):
        assert sh.t_begin == prev and sh.t_end >= sh.t_begin
        assert sh.owns_current == (1 if r == n - 1 else 0) and sh.reserved == 0
        for t in (sh.t_begin, sh.t_end):   # boundaries inside the middle sit on span edges
            assert t <= G or t >= G + M or (t - G) % S == 0
        lo = 0 if sh.t_begin <= G else (NS if sh.t_begin >= G + M else (sh.t_begin - G) // S)
        hi = 0 if sh.t_end <= G else (NS if sh.t_end >= G + M else (sh.t_end - G) // S)
        counts.append(max(0, hi - lo))
        prev = sh.t_end
    assert prev == T
    assert sum(counts) == NS
    assert max(counts) - min(counts) <= 1   # spans spread evenly
    assert shards[0].t_begin == 0 and shards[0].t_end >= min(G, T) or n == 1


def test_shard_arguments_are_checked(R):
    d = dims(R, T=20000, L=512, k=16, Hq=8, Hkv=2)
    fake = 0x10000   # never dereferenced: the checks fail first
    sz = ctypes.c_size_t()

    def mk(t0, t1, cap=0, owns=0, res=0):
        s = R.reatt_shard()
        s.t_begin, s.t_end, s.rows_cap, s.owns_current, s.reserved = t0, t1, cap, owns, res
        return s

    good = mk(0, 32 + 32 * 100, owns=1)
    assert R.lib.reatt_shard_workspace_bytes(ctypes.byref(d), ctypes.byref(good), 2,
                                             ctypes.byref(sz)) == R.OK
    assert sz.value % 256 == 0
    bad = [
        mk(0, 32 + 32 * 100 + 5),     # boundary inside a span
        mk(-1, 100), mk(50, 40), mk(0, 20001),
        mk(0, 100, cap=99), mk(0, 100, owns=2), mk(0, 100, res=1),
    ]
    for s in bad:
        assert R.lib.reatt_shard_workspace_bytes(ctypes.byref(d), ctypes.byref(s), 2,
                                                 ctypes.byref(sz)) == R.EINVAL
        assert R.reatt_shard_candidates(d, s, fake, fake, fake, fake, fake, stream=0,
                                        check=False) == R.EINVAL
        assert R.reatt_shard_attend(d, s, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                    stream=0, check=False) == R.EINVAL
    # boundaries inside the global and local parts are allowed
    for s in (mk(16, 32 + 32 * 10), mk(20000 - 100, 20000, owns=1)):
        assert R.lib.reatt_shard_workspace_bytes(ctypes.byref(d), ctypes.byref(s), 2,
                                                 ctypes.byref(sz)) == R.OK
    # null and misaligned pointers, bad shard counts
    M8 = fake + 8
    assert R.reatt_shard_candidates(d, good, None, fake, fake, fake, fake, stream=0,
                                    check=False) == R.EINVAL
    assert R.reatt_shard_candidates(d, good, fake, fake, M8, fake, fake, stream=0,
                                    check=False) == R.EINVAL
    assert R.reatt_shard_select(d, 0, fake, fake, fake, fake, stream=0, check=False) == R.EINVAL
    assert R.reatt_shard_select(d, 2, None, fake, fake, fake, stream=0, check=False) == R.EINVAL
    assert R.reatt_shard_select(d, 2, fake, fake, M8, fake, stream=0, check=False) == R.EINVAL
    assert R.reatt_shard_attend(d, good, fake, fake, fake, None, fake, fake, fake, fake, fake,
                                stream=0, check=False) == R.EINVAL   # owner needs k_cur
    assert R.reatt_merge_partials(d, 0, fake, fake, fake, stream=0, check=False) == R.EINVAL
    assert R.reatt_merge_partials(d, 2, fake, None, fake, stream=0, check=False) == R.EINVAL
    assert R.reatt_merge_partials(d, 2, fake, fake, M8, stream=0, check=False) == R.EINVAL
    assert R.lib.reatt_shard_plan(ctypes.byref(d), 0, None) == R.EINVAL
    # bad dims reach every shard call as the same status as elsewhere
    bd = dims(R, d=96)
    assert R.reatt_merge_partials(bd, 2, fake, fake, fake, stream=0, check=False) == \
        R.EUNSUPPORTED
    assert R.reatt_shard_select(bd, 2, fake, fake, fake, fake, stream=0, check=False) == \
        R.EUNSUPPORTED


def test_workspace_does_not_depend_on_the_shard(R):
    d = dims(R, T=1 << 20)
    shards = R.reatt_shard_plan(d, 4)
    sizes = {R.reatt_shard_workspace_bytes(d, s, 4) for s in shards}
    assert len(sizes) == 1
    assert R.reatt_shard_workspace_bytes(d, shards[0], 8) > sizes.pop()
