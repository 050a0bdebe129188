"""GPU parity of every C-ABI call against the CPU oracle, at sizes the oracle
finishes in seconds: the tiny fp32 workload, scaled-down bf16 LLaMA/Qwen
shapes, ragged spans, and the degenerate cases of the method."""
import numpy as np
import pytest
import torch

from tests import parity
from top_kv_span_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    from top_kv_span_b200 import build
    build.build()
    from top_kv_span_b200 import reatt
    assert torch.cuda.is_available()
    return reatt


TINY = wl.WORKLOADS["tiny_f32_4k"]
LLAMA = wl.WORKLOADS["llama3_8b_128k"]

CASES = {
    "tiny_f32_4k": TINY,
    # ragged: M = 983 = 140*7 + 3, two sequences, GQA 3
    "odd_f32_d64": TINY.replace(name="odd", B=2, Hq=6, Hkv=2, T=1003, G=3, L=17, S=7, k=5,
                                n_needles=2, seed=11),
    # middle a whole number of spans (M = 987 = 141*7): the window length is
    # known before the selection, so the decode attention starts early
    "early_f32_gqa3": TINY.replace(name="early", B=2, Hq=6, Hkv=2, T=1007, G=3, L=17, S=7, k=5,
                                   n_needles=2, seed=27),
    "bf16_d128_20k": LLAMA.replace(name="bf16_20k", Hq=8, Hkv=2, T=20000, L=512, k=16,
                                   n_needles=3, seed=12),
    # decode on the tensor cores with a few current tokens (causal among them)
    # and with one query head per KV head
    "decode_tc_c3": LLAMA.replace(name="dtc_c3", Hq=4, Hkv=2, C=3, T=32 + 256 + 32 * 210,
                                  L=256, k=10, n_needles=1, seed=28),
    "decode_tc_g1": LLAMA.replace(name="dtc_g1", Hq=2, Hkv=2, T=8 + 200 + 16 * 550, G=8, L=200,
                                  S=16, k=12, n_needles=2, seed=29),
    # bf16, d = 128, ragged last span: the CUDA-core staged decode kernel
    "bf16_d128_ragged_staged": LLAMA.replace(name="bf16_rg", Hq=8, Hkv=2, T=20003, L=512, k=16,
                                             n_needles=2, seed=30),
    "bf16_d64_ragged": LLAMA.replace(name="bf16_d64", Hq=4, Hkv=2, d=64, T=9001, G=5, L=300,
                                     S=32, k=12, n_needles=2, seed=13),
    "k_ge_ns_full_attention": LLAMA.replace(name="kge", Hq=8, Hkv=2, T=300, G=16, L=128, k=8,
                                            n_needles=0, seed=14),
    "no_middle": LLAMA.replace(name="nomid", Hq=8, Hkv=2, T=100, G=32, L=128, k=8, n_needles=0,
                               seed=15),
    "shorter_than_global": TINY.replace(name="tiny_t", T=3, G=4, L=8, S=3, k=2, n_needles=0,
                                        seed=16),
    "token_level_s1": TINY.replace(name="s1", Hq=4, Hkv=2, T=700, G=4, L=32, S=1, k=40,
                                   n_needles=0, seed=17),
    "streaming_k0": LLAMA.replace(name="k0", Hq=8, Hkv=2, T=5000, L=256, k=0, n_needles=0,
                                  seed=18),
    "prefill_f32_c5": TINY.replace(name="c5", Hq=6, Hkv=2, C=5, T=2000, G=4, L=64, S=16, k=6,
                                   n_needles=0, seed=19),
    "prefill_bf16_c7": LLAMA.replace(name="c7", Hq=8, Hkv=2, C=7, T=6000, L=256, k=10,
                                     n_needles=0, seed=20),
    "prefill_bf16_c70": LLAMA.replace(name="c70", Hq=4, Hkv=1, C=70, T=3000, G=8, L=64, S=32,
                                      k=5, n_needles=0, seed=23),
    "prefill_bf16_g2_d64_c300": LLAMA.replace(name="c300", Hq=4, Hkv=2, d=64, C=300, T=5000,
                                              G=8, L=100, S=16, k=20, n_needles=0, seed=24),
    "prefill_bf16_g1_c130_s8": LLAMA.replace(name="c130", Hq=2, Hkv=2, C=130, T=2600, G=8,
                                             L=64, S=8, k=30, n_needles=0, seed=25),
    "prefill_bf16_s64_fallback": LLAMA.replace(name="s64", Hq=4, Hkv=1, C=9, T=3000, G=8, L=64,
                                               S=64, k=5, n_needles=0, seed=26),
    # query-resident tensor-core scan (S = 32): d = 64; one raw query head per KV
    # head (one term); two raw heads and an odd number of query tiles (an item
    # with one query slot); several key chunks per head with a 3-token last key
    # tile and a 3-token last span
    "prefill_bf16_d64_s32_c200": LLAMA.replace(name="c200", Hq=8, Hkv=2, d=64, C=200, T=7000,
                                               G=8, L=100, S=32, k=12, n_needles=2, seed=31),
    "prefill_bf16_g1_s32_c260": LLAMA.replace(name="c260", Hq=2, Hkv=2, C=260, T=6003, G=8,
                                              L=64, S=32, k=10, n_needles=2, seed=32),
    "prefill_bf16_g2_s32_c300": LLAMA.replace(name="c300s32", Hq=4, Hkv=2, C=300, T=5000, G=8,
                                              L=100, S=32, k=12, n_needles=1, seed=34),
    "prefill_bf16_chunks_c130": LLAMA.replace(name="c130k", Hq=8, Hkv=2, C=130, T=20003, G=32,
                                              L=256, S=32, k=16, n_needles=3, seed=33),
    "prefill_bf16_b2_c150": LLAMA.replace(name="b2c150", B=2, Hq=4, Hkv=2, C=150, T=4000, G=8,
                                          L=100, S=32, k=8, n_needles=2, seed=35),
    # GQA 4 with hi/lo query terms and 8 query tiles (four query-slot pairs),
    # two sequences, and k a large share of the spans
    "prefill_bf16_b2_g4_c1000": LLAMA.replace(name="b2g4c1000", B=2, Hq=4, Hkv=1, C=1000,
                                              T=4000, G=8, L=100, S=32, k=8, n_needles=2,
                                              seed=36),
    "prefill_bf16_g4_k40_c1000": LLAMA.replace(name="g4k40", Hq=8, Hkv=2, C=1000, T=3000, G=8,
                                               L=64, S=32, k=40, n_needles=0, seed=37),
    "two_level_topk": LLAMA.replace(name="big_ns", Hq=2, Hkv=1, d=64, T=200000, G=32, L=256,
                                    S=8, k=100, n_needles=4, seed=21),
    "batch3_large_s": TINY.replace(name="b3", B=3, Hq=2, Hkv=1, T=5000, G=2, L=40, S=100, k=3,
                                   n_needles=1, seed=22),
}


@pytest.mark.parametrize("name", list(CASES))
def test_all_entry_points_match_oracle(R, ora, name):
    w = CASES[name]
    info = parity.full_check(R, ora, w)
    print(name, info)


def test_empty_cache(R, ora):
    """T = 0: the window is just the current tokens."""
    w = TINY.replace(name="t0", T=0, n_needles=0, C=3, seed=30)
    info = parity.full_check(R, ora, w)
    assert info["swaps"] == 0


def test_repeat_calls_are_deterministic(R):
    """Same inputs, same workspace, two calls: bit-identical results (tickets reset)."""
    w = CASES["bf16_d128_20k"]
    x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
    d = R.dims_of(w)
    b = R.alloc_outputs(d)
    outs = []
    for _ in range(3):
        R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                     b["out"], b["ws"])
        torch.cuda.synchronize()
        outs.append((b["sel"].clone(), b["out"].clone()))
    for s, o in outs[1:]:
        assert torch.equal(s, outs[0][0]) and torch.equal(o, outs[0][1])


def test_runs_on_a_side_stream(R, ora):
    w = CASES["odd_f32_d64"]
    x = wl.make_inputs(w)
    xd = {n: x[n].cuda() for n in parity.NAMES}
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gpu = parity.run_all(R, R.dims_of(w), xd, stream=s)
    ref = ora.step(**parity.host_inputs(x), G=w.G, L=w.L, S=w.S, k=w.k, rope_base=w.rope_base)
    parity.check_selection(ref["scores"], ref["sel"], gpu["sel_step"], w.k)
    parity.check_outputs(ora, parity.host_inputs(x), gpu["sel_step"], gpu["out_step"], w, ref=ref)


def test_topk_ties_prefer_lower_index(R):
    """Exact ties in the scores: the lower span id wins, output ascending."""
    w = LLAMA.replace(Hq=2, Hkv=1, d=64, T=32 + 4096 + 32 * 9000, G=32, L=4096, S=32, k=50)
    d = R.dims_of(w)
    NS = R.reatt_num_spans(d)
    rng = np.random.default_rng(5)
    sc = rng.integers(0, 7, NS).astype(np.float32)     # many ties, NS > one slice
    scores = torch.tensor(sc).reshape(1, 1, NS).cuda()
    sel = torch.empty((1, 1, w.k), dtype=torch.int32, device="cuda")
    ws = torch.zeros(R.reatt_workspace_bytes(d), dtype=torch.uint8, device="cuda")
    R.reatt_topk(d, scores, sel, ws)
    torch.cuda.synchronize()
    order = np.lexsort((np.arange(NS), -sc.astype(np.float64)))
    assert sel.cpu().numpy()[0, 0].tolist() == sorted(order[:w.k].tolist())


def test_topk_negative_and_infinite_scores(R):
    w = LLAMA.replace(Hq=2, Hkv=1, d=64, T=32 + 4096 + 32 * 40, G=32, L=4096, S=32, k=7)
    d = R.dims_of(w)
    NS = R.reatt_num_spans(d)
    sc = np.linspace(-5, 5, NS).astype(np.float32)
    sc[3] = np.inf
    sc[4] = -np.inf
    sc[10] = -0.0
    sc[11] = 0.0
    scores = torch.tensor(sc).reshape(1, 1, NS).cuda()
    sel = torch.empty((1, 1, w.k), dtype=torch.int32, device="cuda")
    ws = torch.zeros(R.reatt_workspace_bytes(d), dtype=torch.uint8, device="cuda")
    R.reatt_topk(d, scores, sel, ws)
    torch.cuda.synchronize()
    order = np.lexsort((np.arange(NS), -sc.astype(np.float64)))
    assert sel.cpu().numpy()[0, 0].tolist() == sorted(order[:w.k].tolist())


@pytest.mark.parametrize("dist", ["normal", "ties", "narrow", "equal", "wide"])
def test_topk_sizes_and_value_spreads(R, dist):
    """The selection against its definition (score descending, ties to the lower
    span id, the first k_eff ids, ascending) over one-slice and multi-slice span
    counts, k around and above the span count, and several heads at once."""
    rng = np.random.default_rng(["normal", "ties", "narrow", "equal", "wide"].index(dist) + 40)
    for NS, k in [(1, 1), (7, 3), (7, 9), (100, 64), (3967, 64), (4096, 64), (4097, 64),
                  (5000, 1), (8192, 64), (8193, 64), (9000, 200), (20000, 64), (2048, 2048)]:
        w = LLAMA.replace(B=2, Hq=4, Hkv=2, d=64, T=32 + 4096 + 32 * NS, G=32, L=4096, S=32, k=k)
        d = R.dims_of(w)
        assert R.reatt_num_spans(d) == NS
        shape = (w.B, w.Hkv, NS)
        if dist == "normal":
            sc = rng.standard_normal(shape)
        elif dist == "ties":
            sc = rng.integers(0, 5, shape)
        elif dist == "narrow":
            sc = 100.0 + 1e-4 * rng.standard_normal(shape)
        elif dist == "equal":
            sc = np.full(shape, 3.5)
        else:
            sc = rng.standard_normal(shape) * 10.0 ** rng.integers(-30, 30, shape)
        sc = sc.astype(np.float32)
        scores = torch.tensor(sc).cuda()
        sel = torch.full((w.B, w.Hkv, k), 12345, dtype=torch.int32, device="cuda")
        ws = torch.empty(R.reatt_workspace_bytes(d), dtype=torch.uint8, device="cuda")
        R.reatt_topk(d, scores, sel, ws)
        torch.cuda.synchronize()
        got = sel.cpu().numpy()
        keff = min(k, NS)
        for b in range(w.B):
            for h in range(w.Hkv):
                s = sc[b, h].astype(np.float64)
                order = np.lexsort((np.arange(NS), -s))
                want = sorted(order[:keff].tolist()) + [-1] * (k - keff)
                assert got[b, h].tolist() == want, (dist, NS, k, b, h)
