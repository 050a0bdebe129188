"""One sequence's cache split over token-range shards, run on one GPU: every
shard's calls go through the C ABI in one process, and the two exchanges
(candidates, partials) are plain stacks.  The merged result is checked
against the oracle on the whole sequence (selection up to the swap rule,
outputs within the workload's tolerance) and against reatt_step on the
whole cache (the same selection, outputs to fp32 rounding)."""
import numpy as np
import pytest
import torch

from tests import parity
from top_kv_span_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LLAMA = wl.WORKLOADS["llama3_8b_128k"]
TINY = wl.WORKLOADS["tiny_f32_4k"]


@pytest.fixture(scope="module")
def R():
    from top_kv_span_b200 import build
    build.build()
    from top_kv_span_b200 import reatt
    return reatt


def make_shard(R, t0, t1, owns, cap=0):
    s = R.reatt_shard()
    s.t_begin, s.t_end, s.rows_cap, s.owns_current, s.reserved = t0, t1, cap, owns, 0
    return s


def run_sharded(R, w, x, shards, extra_rows=0):
    """Phases of every shard in turn; returns (sel, out, per-shard candidates)."""
    from top_kv_span_b200.sharded import ShardedStep
    d = R.dims_of(w)
    n = len(shards)
    steps, caches = [], []
    for sh in shards:
        rows = sh.t_end - sh.t_begin
        cap = rows + extra_rows
        if extra_rows:
            sh.rows_cap = cap
        kc = torch.full((w.B, w.Hkv, cap, w.d), float("nan"), dtype=w.torch_dtype, device="cuda")
        vc = torch.full_like(kc, float("nan"))
        kc[:, :, :rows] = x["k_cache"][:, :, sh.t_begin:sh.t_end]
        vc[:, :, :rows] = x["v_cache"][:, :, sh.t_begin:sh.t_end]
        caches.append((kc, vc))
        steps.append(ShardedStep(d, sh, n))
    for st, (kc, _) in zip(steps, caches):
        st.candidates(x["q"], kc)
    cs = torch.stack([st.cand_score for st in steps])
    ci = torch.stack([st.cand_id for st in steps])
    for st in steps:
        st.cand_score_all.copy_(cs)
        st.cand_id_all.copy_(ci)
        st.select()
    for st, (kc, vc) in zip(steps, caches):
        st.attend(x["q"], kc, vc, x["k_cur"], x["v_cur"])
    ml = torch.stack([st.part_ml for st in steps])
    acc = torch.stack([st.part_acc for st in steps])
    out = torch.full((w.B, w.Hq, w.C, w.d), float("nan"), dtype=torch.float32, device="cuda")
    steps[-1].part_ml_all.copy_(ml)
    steps[-1].part_acc_all.copy_(acc)
    steps[-1].merge(out)
    torch.cuda.synchronize()
    for st in steps:
        assert R.reatt_workspace_status(st.ws) == R.OK
        assert torch.equal(st.sel, steps[0].sel)   # every shard selects the same
    cands = [(c.cpu().numpy(), i.cpu().numpy()) for c, i in zip(cs, ci)]
    return steps[0].sel.cpu().numpy(), out.cpu().numpy(), cands


def check_against_oracle_and_step(R, ora, w, x, shards, extra_rows=0):
    sel, out, cands = run_sharded(R, w, x, shards, extra_rows)
    xh = parity.host_inputs(x)
    ref = ora.step(**xh, G=w.G, L=w.L, S=w.S, k=w.k, rope_base=w.rope_base)
    swaps = parity.check_selection(ref["scores"], ref["sel"], sel, w.k)
    err = parity.check_outputs(ora, xh, sel, out, w, ref=ref)
    # each shard's candidates: the top-k of its own spans, ascending, with
    # their scores (swaps only among near-ties of the slice's k-th score)
    d = R.dims_of(w)
    NS = ref["scores"].shape[-1]
    M = max(0, w.T - w.G - w.L)

    def span_at(t):
        return 0 if t <= w.G else (NS if t >= w.G + M else (t - w.G) // w.S)

    for sh, (cs, ci) in zip(shards, cands):
        lo, hi = span_at(sh.t_begin), max(span_at(sh.t_begin), span_at(sh.t_end))
        for b in range(w.B):
            for h in range(w.Hkv):
                local = ref["scores"][b, h, lo:hi]
                keff = min(w.k, local.size)
                got = ci[b, h]
                assert (got[keff:] == -1).all() and np.isneginf(cs[b, h, keff:]).all()
                assert (np.diff(got[:keff]) > 0).all()
                assert ((got[:keff] >= lo) & (got[:keff] < hi)).all()
                if not keff:
                    continue
                scale = max(1.0, float(np.abs(local).max()))
                assert np.abs(cs[b, h, :keff] - ref["scores"][b, h, got[:keff]]).max() <= \
                    parity.SCORE_RTOL * scale
                want = set((ora.topk(local, w.k)[:keff] + lo).tolist())
                kth = np.sort(local)[::-1][keff - 1]
                for sp in want ^ set(got[:keff].tolist()):
                    assert abs(ref["scores"][b, h, sp] - kth) <= parity.SWAP_REL * abs(kth)
    # the unsharded step on the whole cache: same kernels' scores, same selection
    b = R.alloc_outputs(d)
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                 b["out"], b["ws"])
    torch.cuda.synchronize()
    assert np.array_equal(b["sel"].cpu().numpy(), sel)
    diff = float(np.abs(b["out"].cpu().numpy().astype(np.float64) - out).max())
    assert diff <= parity.OUT_TOL[w.dtype]
    return swaps, err, diff


CASES = [
    # bf16 GQA decode, shards from the planner
    (LLAMA.replace(name="sh_dec", Hq=8, Hkv=2, T=20000, L=512, k=16, n_needles=2, seed=80), 2),
    (LLAMA.replace(name="sh_dec3", Hq=8, Hkv=2, T=20000, L=512, k=16, n_needles=3, seed=81), 3),
    # ragged last span, batch of 2
    (LLAMA.replace(name="sh_rag", B=2, Hq=8, Hkv=2, T=20003, L=512, k=16, n_needles=2, seed=82), 2),
    # fp32, d=64, odd sizes, more shards than some shards have spans
    (TINY.replace(name="sh_f32", B=2, Hq=6, Hkv=2, T=1003, G=3, L=17, S=7, k=5, n_needles=1,
                  seed=83), 5),
    # prefill chunk (CUDA-core span scan on each shard)
    (LLAMA.replace(name="sh_pre", Hq=8, Hkv=2, C=40, T=9000, L=256, k=10, n_needles=0, seed=84), 2),
    # everything selected (k >= NS): full attention split over shards
    (TINY.replace(name="sh_all", Hq=4, Hkv=1, T=600, G=4, L=64, S=32, k=64, n_needles=0,
                  seed=85), 3),
]


@pytest.mark.parametrize("w,n", CASES, ids=[c[0].name for c in CASES])
def test_planned_shards_match_oracle(R, ora, w, n):
    x = {k: v.cuda() if torch.is_tensor(v) else v for k, v in wl.make_inputs(w).items()}
    shards = R.reatt_shard_plan(R.dims_of(w), n)
    assert shards[0].t_begin == 0 and shards[-1].t_end == w.T
    assert sum(s.owns_current for s in shards) == 1
    swaps, err, diff = check_against_oracle_and_step(R, ora, w, x, shards)
    print(w.name, n, "swaps", swaps, "max-abs", err, "vs step", diff)


def test_hand_made_shards_split_global_and_local(R, ora):
    """Boundaries inside the global part and inside the local part, a shard
    without middle spans, strided shard caches, and the current tokens owned
    by the first shard."""
    w = LLAMA.replace(name="sh_hand", Hq=8, Hkv=2, T=12000, G=32, L=512, k=12, n_needles=2,
                      seed=86)
    M = w.T - w.G - w.L
    mid = w.G + (M // w.S // 2) * w.S
    cuts = [0, 16, mid, w.T - 200, w.T]
    shards = [make_shard(R, a, b, 1 if i == 0 else 0) for i, (a, b) in enumerate(zip(cuts, cuts[1:]))]
    x = {k: v.cuda() if torch.is_tensor(v) else v for k, v in wl.make_inputs(w).items()}
    check_against_oracle_and_step(R, ora, w, x, shards, extra_rows=37)


def test_llama3_8b_128k_two_shards(R, ora):
    """The 128K LLaMA3-8B-shaped decode split over two shards."""
    w = LLAMA
    x = {k: v for k, v in wl.make_inputs(w, "cuda").items()}
    shards = R.reatt_shard_plan(R.dims_of(w), 2)
    swaps, err, diff = check_against_oracle_and_step(R, ora, w, x, shards)
    print("128K two shards: swaps", swaps, "max-abs", err, "vs step", diff)
