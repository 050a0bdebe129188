"""The fused prefill step's two-pass span filter against the one-pass scan.

For long prefill chunks with hi/lo query terms (a 2048-query chunk over 256K),
reatt_step scores the spans with a hi-only pass, rules out the spans whose
bound cannot reach the k-th lower bound, and rescores only the rest with
hi + lo (ReAttention OpenReview discussion, "Prefilling Phase" pseudocode: the
top-k of the chunk's span scores).  The selection must be exactly the top-k of
the one-pass scores that reatt_score_spans returns: the k largest scores, ties
to the lower span id, in ascending span order.  No oracle is involved, so the
full-size chunk is checked in every head."""
import pytest
import torch

from top_kv_span_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CASES = {
    # 2048 queries over 256K: 8,063 spans per KV head, k = 64
    "llama3_8b_prefill_256k": wl.WORKLOADS["llama3_8b_prefill_256k"],
    # the same chunk with k = 128: more spans near the k-th score
    "llama3_8b_prefill_256k_k128": wl.WORKLOADS["llama3_8b_prefill_256k"].replace(
        name="p256k128", k=128, seed=1007),
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
    x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
    d = R.dims_of(w)
    b = R.alloc_outputs(d)
    R.reatt_score_spans(d, x["q"], x["k_cache"], b["span_scores"], b["ws"])
    torch.cuda.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                     b["out"], b["ws"])
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
    # the step took the filter: two scan passes and the candidate selection
    assert sum("scan_prefill_tcq_kernel" in n for n in names) == 2, names
    assert any("prefill_candidates_kernel" in n for n in names), names
    assert R.reatt_workspace_status(b["ws"]) == 0
    scores = b["span_scores"]
    ns = scores.shape[-1]
    assert w.k < ns
    for bi in range(w.B):
        for h in range(w.Hkv):
            want = expected_selection(scores[bi, h], w.k).to(torch.int32)
            got = b["sel"][bi, h]
            assert torch.equal(got, want), (bi, h, got.tolist(), want.tolist())
