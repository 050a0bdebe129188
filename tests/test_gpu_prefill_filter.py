"""The fused prefill step's two-pass span filter against the one-pass scan.

For chunks of at least 8 query tiles with hi/lo query terms, reatt_step scores
the spans with a hi-only pass, rules out the spans whose bound cannot reach the
k-th lower bound, and rescores only the rest with hi + lo (ReAttention
OpenReview discussion, "Prefilling Phase" pseudocode: the top-k of the chunk's
span scores).  The selection must be exactly the top-k of the one-pass scores
that reatt_score_spans returns: the k largest scores, ties to the lower span
id, in ascending span order.  No oracle is involved, so the full-size 64K
chunk is checked in every head."""
import pytest
import torch

from top_kv_span_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LLAMA = wl.WORKLOADS["llama3_8b_128k"]

CASES = {
    # 2048 queries over 64K: 1,919 spans per KV head, k = 64
    "llama3_8b_prefill_64k": wl.WORKLOADS["llama3_8b_prefill_64k"],
    # k a large share of the spans, so most key tiles are rescored
    "g4_k40_c1000": LLAMA.replace(name="g4k40", Hq=8, Hkv=2, C=1000, T=3000, G=8, L=64, S=32,
                                  k=40, n_needles=0, seed=37),
    # two sequences, needles
    "b2_g4_c1024": LLAMA.replace(name="b2g4", B=2, Hq=8, Hkv=2, C=1024, T=40000, G=32, L=512,
                                 S=32, k=32, n_needles=3, seed=38),
}


@pytest.fixture(scope="module")
def R():
    from top_kv_span_b200 import build
    build.build()
    from top_kv_span_b200 import reatt
    assert torch.cuda.is_available()
    return reatt


def expected_selection(scores, k):
    """Top-k of one head's scores: largest first, ties to the lower id, then ascending."""
    ns = scores.shape[0]
    ids = torch.arange(ns, device=scores.device)
    order = torch.sort(-scores, stable=True).indices   # ties keep the lower id first
    chosen = ids[order[:min(k, ns)]]
    return torch.sort(chosen).values


@pytest.mark.parametrize("name", list(CASES))
def test_step_selection_equals_one_pass_top_k(R, name):
    w = CASES[name]
    g = w.Hq // w.Hkv
    assert g > 2 and w.S == 32 and (w.C + 127) // 128 >= 8, "the case must take the filter"
    x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
    d = R.dims_of(w)
    b = R.alloc_outputs(d)
    R.reatt_score_spans(d, x["q"], x["k_cache"], b["span_scores"], b["ws"])
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                 b["out"], b["ws"])
    torch.cuda.synchronize()
    assert R.reatt_workspace_status(b["ws"]) == 0
    scores = b["span_scores"]
    ns = scores.shape[-1]
    assert w.k < ns
    for bi in range(w.B):
        for h in range(w.Hkv):
            want = expected_selection(scores[bi, h], w.k).to(torch.int32)
            got = b["sel"][bi, h]
            assert torch.equal(got, want), (bi, h, got.tolist(), want.tolist())
