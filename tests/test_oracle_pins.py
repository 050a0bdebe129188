"""Pins for the CPU oracle (no GPU): the oracle is checked against things other
than itself -- closed forms, brute force, an independent NumPy textbook, the
pages' window arithmetic and the method's invariants."""
import json
import os

import numpy as np
import pytest

from tests import textbook as tb

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(rng, B, Hq, Hkv, d, C, T, dtype="f32", scale=1.0):
    def draw(*shape):
        x = (rng.standard_normal(shape) * scale).astype(np.float32)
        if dtype == "bf16":
            # round-to-nearest-even to bf16 bits
            u = x.view(np.uint32).astype(np.uint64)
            u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
            return u.astype(np.uint16)
        return x
    return dict(q=draw(B, Hq, C, d), k_cache=draw(B, Hkv, T, d), v_cache=draw(B, Hkv, T, d),
                k_cur=draw(B, Hkv, C, d), v_cur=draw(B, Hkv, C, d))


def f64(x):
    return tb.bits_to_f64(x)


# ---------------------------------------------------------------- partition
@pytest.mark.parametrize("T,G,L,S,expect", [
    (4096, 4, 256, 32, (4, 3840, 3836, 120)),
    (131072, 32, 4096, 32, (32, 126976, 126944, 3967)),
    (1048576, 32, 4096, 32, (32, 1044480, 1044448, 32639)),
    (262144, 32, 4096, 32, (32, 258048, 258016, 8063)),
    (4194304, 32, 4096, 32, (32, 4190208, 4190176, 130943)),
    (10, 4, 8, 3, (4, 4, 0, 0)),        # T < G+L: no middle, local = [G, T)
    (3, 4, 8, 3, (3, 4, 0, 0)),         # T < G: everything is global
    (12, 4, 8, 3, (4, 4, 0, 0)),        # T == G+L
    (13, 4, 8, 3, (4, 5, 1, 1)),        # one-token middle
])
def test_partition_closed_form(ora, T, G, L, S, expect):
    assert ora.partition(T, G, L, S) == expect


def test_window_arithmetic_from_pages(ora):
    """The pages' ReAttention NIAH settings give a cached window of exactly the
    pre-trained length of LLaMA3-8B-8K (golden fixture)."""
    with open(os.path.join(GOLDEN, "niah_settings_window.json")) as f:
        gold = json.load(f)
    G, L, S, k = gold["global_size"], gold["local_size"], gold["seg_size"], gold["num_seg"]
    T = 1 << 20
    NS = ora.partition(T, G, L, S)[3]
    scores = np.random.default_rng(0).standard_normal(NS)
    sel = ora.topk(scores, k)
    src = ora.window(T, G, L, S, 0, sel)
    assert len(src) == gold["cached_window_rows"]


# ---------------------------------------------------------------- scoring
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [43, 40, 12, 13])
def test_span_scores_match_matrix_form(ora, dtype, T):
    """Oracle (per-head double sum, loops) == (sum_j Q_j) K_mid^T, span max."""
    rng = np.random.default_rng(T)
    x = rand_inputs(rng, B=2, Hq=6, Hkv=2, d=8, C=3, T=T, dtype=dtype)
    G, L, S = 3, 5, 4
    got = ora.span_scores(x["q"], x["k_cache"], G, L, S)
    ref = tb.span_scores(f64(x["q"]), f64(x["k_cache"]), G, L, S)
    assert got.shape == ref.shape
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_span_scores_brute_force_single_token(ora):
    """Hand brute force on a 1-token-span case with C=2: one scalar at a time."""
    rng = np.random.default_rng(7)
    x = rand_inputs(rng, B=1, Hq=2, Hkv=1, d=4, C=2, T=9)
    G, L, S = 2, 3, 1
    got = ora.span_scores(x["q"], x["k_cache"], G, L, S)[0, 0]
    q, k = f64(x["q"]), f64(x["k_cache"])
    for sp in range(4):
        t = G + sp
        vals = [sum(q[0, j, c] @ k[0, 0, t] for j in range(2)) for c in range(2)]
        assert got[sp] == pytest.approx(max(vals), rel=1e-13)


def test_span_scores_list_matches_full(ora):
    rng = np.random.default_rng(3)
    x = rand_inputs(rng, B=2, Hq=4, Hkv=2, d=16, C=1, T=100)
    full = ora.span_scores(x["q"], x["k_cache"], 4, 8, 5)
    pairs = np.array([[0, 0], [1, 17], [3, 5], [2, 17]])
    got = ora.span_scores_list(x["q"], x["k_cache"], 4, 8, 5, pairs)
    np.testing.assert_array_equal(got, full.reshape(4, -1)[pairs[:, 0], pairs[:, 1]])


# ---------------------------------------------------------------- top-k
@pytest.mark.parametrize("NS,k", [(50, 8), (50, 50), (7, 12), (1, 1), (64, 0), (333, 64)])
def test_topk_matches_stable_sort(ora, NS, k):
    rng = np.random.default_rng(NS * 100 + k)
    scores = rng.integers(0, 6, NS).astype(np.float64)      # many ties
    sel = ora.topk(scores, k)
    order = np.lexsort((np.arange(NS), -scores))             # score desc, index asc
    keff = min(k, NS)
    expect = np.sort(order[:keff])
    assert list(sel[:keff]) == list(expect)
    assert all(v == -1 for v in sel[keff:])
    if 0 < keff < NS:
        chosen = set(expect)
        lo = min(scores[i] for i in chosen)
        hi = max(scores[i] for i in range(NS) if i not in chosen)
        assert lo >= hi


def test_topk_ties_prefer_lower_index(ora):
    sel = ora.topk(np.array([1.0, 2.0, 2.0, 2.0, 0.5]), 2)
    assert list(sel) == [1, 2]


# ---------------------------------------------------------------- window
def test_window_order_by_hand(ora):
    # T=20, G=2, L=3, S=4: middle [2,17) = spans [2,6) [6,10) [10,14) [14,17)(short)
    src = ora.window(20, 2, 3, 4, 2, np.array([1, 3], np.int32))
    assert list(src) == [0, 1, 6, 7, 8, 9, 14, 15, 16, 17, 18, 19, -1, -2]
    src = ora.window(20, 2, 3, 4, 1, np.array([0, -1], np.int32))
    assert list(src) == [0, 1, 2, 3, 4, 5, 17, 18, 19, -1]


# ---------------------------------------------------------------- RoPE
def test_rope_d2_is_rotation_matrix(ora):
    for pos in [0, 1, 7, 1234.0]:
        x = np.array([0.3, -1.7])
        got = ora.rope_row(x, pos, 10000.0)
        R = np.array([[np.cos(pos), -np.sin(pos)], [np.sin(pos), np.cos(pos)]])
        np.testing.assert_allclose(got, R @ x, atol=1e-12)


def test_rope_frequencies_d4(ora):
    base, pos = 100.0, 5.0
    x = np.array([1.0, 0.0, 0.0, 0.0])        # pair 0 = (x0, x2)
    got = ora.rope_row(x, pos, base)
    np.testing.assert_allclose(got, [np.cos(pos), 0, np.sin(pos), 0], atol=1e-12)
    x = np.array([0.0, 1.0, 0.0, 0.0])        # pair 1 = (x1, x3), freq base^(-1/2)
    a = pos * base ** -0.5
    np.testing.assert_allclose(ora.rope_row(x, pos, base), [0, np.cos(a), 0, np.sin(a)],
                               atol=1e-12)


def test_rope_norm_and_relative_position(ora):
    rng = np.random.default_rng(11)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for base in [1e4, 5e5]:
        qr = ora.rope_row(q, 37, base)
        assert np.linalg.norm(qr) == pytest.approx(np.linalg.norm(q), rel=1e-13)
        ref = qr @ ora.rope_row(k, 12, base)
        for delta in [1, 100, 4000]:
            got = ora.rope_row(q, 37 + delta, base) @ ora.rope_row(k, 12 + delta, base)
            assert got == pytest.approx(ref, abs=1e-10)
        np.testing.assert_allclose(qr, tb.rope(q[None], [37], base)[0], atol=1e-12)


# ---------------------------------------------------------------- whole step
def _rows_full(B, Hkv, T):
    return [[list(range(T)) for _ in range(Hkv)] for _ in range(B)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("C,Hq,Hkv", [(1, 4, 1), (3, 4, 2), (2, 2, 2)])
def test_step_reduces_to_full_attention(ora, dtype, C, Hq, Hkv):
    """Invariant 1: when every middle span fits (k >= NS), the step is textbook
    causal RoPE attention over the whole cache ++ current tokens."""
    rng = np.random.default_rng(C * 10 + Hq)
    T, G, L, S, k, base = 45, 3, 6, 4, 9, 1e4          # M = 36, NS = 9
    x = rand_inputs(rng, B=2, Hq=Hq, Hkv=Hkv, d=16, C=C, T=T, dtype=dtype)
    res = ora.step(**x, G=G, L=L, S=S, k=k, rope_base=base)
    assert (res["win_len"] == T + C).all()
    ref = tb.window_attention(f64(x["q"]), f64(x["k_cache"]), f64(x["v_cache"]),
                              f64(x["k_cur"]), f64(x["v_cur"]), _rows_full(2, Hkv, T), base)
    np.testing.assert_allclose(res["out"], ref, atol=1e-12)


def test_step_short_cache_is_full_attention(ora):
    """T < G+L: no middle at all; still full attention."""
    rng = np.random.default_rng(5)
    x = rand_inputs(rng, B=1, Hq=2, Hkv=1, d=8, C=2, T=7)
    res = ora.step(**x, G=4, L=8, S=3, k=2, rope_base=500.0)
    assert list(res["sel"][0, 0]) == [-1, -1]
    ref = tb.window_attention(f64(x["q"]), f64(x["k_cache"]), f64(x["v_cache"]),
                              f64(x["k_cur"]), f64(x["v_cur"]), _rows_full(1, 1, 7), 500.0)
    np.testing.assert_allclose(res["out"], ref, atol=1e-12)


def test_step_k0_is_streaming(ora):
    """k = 0 reduces the method to global ++ local ++ current (StreamingLLM)."""
    rng = np.random.default_rng(9)
    T, G, L = 60, 4, 10
    x = rand_inputs(rng, B=1, Hq=4, Hkv=2, d=8, C=1, T=T)
    res = ora.step(**x, G=G, L=L, S=5, k=0, rope_base=1e4)
    rows = [[list(range(G)) + list(range(T - L, T)) for _ in range(2)]]
    ref = tb.window_attention(f64(x["q"]), f64(x["k_cache"]), f64(x["v_cache"]),
                              f64(x["k_cur"]), f64(x["v_cur"]), rows, 1e4)
    np.testing.assert_allclose(res["out"], ref, atol=1e-12)
    assert (res["win_len"] == G + L + 1).all()


def test_step_token_level_s1(ora):
    """S = 1 is the token-level selection of the decoding pseudocode."""
    rng = np.random.default_rng(13)
    T, G, L, k = 80, 4, 8, 10
    x = rand_inputs(rng, B=1, Hq=4, Hkv=2, d=16, C=1, T=T)
    res = ora.step(**x, G=G, L=L, S=1, k=k, rope_base=1e4)
    q, kc = f64(x["q"]), f64(x["k_cache"])
    rows = [[]]
    for h in range(2):
        tok = q[0, 2 * h:2 * h + 2, 0].sum(0) @ kc[0, h, G:T - L].T
        order = np.lexsort((np.arange(len(tok)), -tok))[:k]
        chosen = sorted(int(G + i) for i in order)
        assert list(res["sel"][0, h]) == [c - G for c in chosen]
        rows[0].append(list(range(G)) + chosen + list(range(T - L, T)))
    ref = tb.window_attention(q, kc, f64(x["v_cache"]), f64(x["k_cur"]), f64(x["v_cur"]),
                              rows, 1e4)
    np.testing.assert_allclose(res["out"], ref, atol=1e-12)


def test_step_ragged_selection_matches_textbook(ora):
    """General case with a short last span that gets chosen."""
    rng = np.random.default_rng(21)
    T, G, L, S, k = 50, 3, 4, 5, 3        # M = 43: 8 full spans + one of 3 tokens
    x = rand_inputs(rng, B=1, Hq=2, Hkv=1, d=8, C=2, T=T)
    x["k_cache"][0, 0, G + 40:G + 43] *= 6.0  # make the short span win
    res = ora.step(**x, G=G, L=L, S=S, k=k, rope_base=1e4)
    sel = list(res["sel"][0, 0])
    assert 8 in sel and sel == sorted(sel)
    rows = list(range(G))
    for sp in sel:
        rows += list(range(G + sp * S, min(G + (sp + 1) * S, T - L)))
    rows += list(range(T - L, T))
    ref = tb.window_attention(f64(x["q"]), f64(x["k_cache"]), f64(x["v_cache"]),
                              f64(x["k_cur"]), f64(x["v_cur"]), [[rows]], 1e4)
    np.testing.assert_allclose(res["out"], ref, atol=1e-12)
    assert res["win_len"][0, 0] == len(rows) + 2


def test_step_zero_query_gives_mean_of_values(ora):
    rng = np.random.default_rng(2)
    x = rand_inputs(rng, B=1, Hq=2, Hkv=1, d=8, C=1, T=40)
    x["q"][:] = 0
    res = ora.step(**x, G=2, L=4, S=4, k=3, rope_base=1e4)
    src = ora.window(40, 2, 4, 4, 1, res["sel"][0, 0])
    v = np.concatenate([x["v_cache"][0, 0, src[:-1]], x["v_cur"][0, 0]], 0).astype(np.float64)
    np.testing.assert_allclose(res["out"][0, 0, 0], v.mean(0), atol=1e-12)


def test_step_explicit_selection_and_query_subset(ora):
    rng = np.random.default_rng(4)
    x = rand_inputs(rng, B=1, Hq=2, Hkv=1, d=8, C=4, T=60)
    full = ora.step(**x, G=2, L=4, S=4, k=3, rope_base=1e4)
    again = ora.step(**x, G=2, L=4, S=4, k=3, rope_base=1e4, sel=full["sel"], c_list=[1, 3])
    np.testing.assert_array_equal(again["out"][:, :, [1, 3]], full["out"][:, :, [1, 3]])
    assert not again["out"][:, :, [0, 2]].any()


# ---------------------------------------------------------------- invariants
def test_needle_always_selected(ora):
    """Invariant 2 on the tiny fp32 workload and a scaled-down per-channel one."""
    from top_kv_span_b200 import workloads as wl
    for w in [wl.WORKLOADS["tiny_f32_4k"],
              wl.WORKLOADS["llama3_8b_128k"].replace(T=8192, Hq=8, Hkv=2, L=512, G=8, k=8,
                                                     n_needles=3)]:
        x = wl.make_inputs(w)
        xs = {n: wl.to_oracle(x[n]) for n in ("q", "k_cache", "v_cache", "k_cur", "v_cur")}
        res = ora.step(**xs, G=w.G, L=w.L, S=w.S, k=w.k, rope_base=w.rope_base)
        for h in range(w.Hkv):
            sc = res["scores"][0, h]
            needles = x["needles"][0]
            assert set(needles) <= set(res["sel"][0, h].tolist())
            others = np.delete(sc, needles)
            assert sc[needles].min() > others.max()


def test_position_agnostic_selection(ora):
    """Invariant 3: shuffling full middle spans permutes span identities but not
    which spans are chosen; moving only unchosen spans leaves the output as is."""
    rng = np.random.default_rng(17)
    T, G, L, S, k = 4 + 30 * 8 + 5 + 8, 4, 8, 8, 6    # 30 full spans + one of 5
    x = rand_inputs(rng, B=1, Hq=4, Hkv=1, d=16, C=1, T=T)
    base = ora.step(**x, G=G, L=L, S=S, k=k, rope_base=1e4)
    chosen = [int(s) for s in base["sel"][0, 0]]
    nfull = 30

    def permuted(perm):
        y = {n: v.copy() for n, v in x.items()}
        for new, old in enumerate(perm):
            for key in ("k_cache", "v_cache"):
                y[key][0, 0, G + new * S:G + (new + 1) * S] = x[key][0, 0, G + old * S:G + (old + 1) * S]
        return y

    perm = rng.permutation(nfull)                       # arbitrary shuffle
    res = ora.step(**permuted(perm), G=G, L=L, S=S, k=k, rope_base=1e4)
    ident = {int(perm[s]) if s < nfull else s for s in res["sel"][0, 0]}
    assert ident == set(chosen)

    unchosen = [s for s in range(nfull) if s not in chosen]
    perm2 = np.arange(nfull)
    perm2[unchosen] = rng.permutation(unchosen)          # only unchosen spans move
    res2 = ora.step(**permuted(perm2), G=G, L=L, S=S, k=k, rope_base=1e4)
    assert list(res2["sel"][0, 0]) == chosen
    np.testing.assert_allclose(res2["out"], base["out"], atol=1e-12)
