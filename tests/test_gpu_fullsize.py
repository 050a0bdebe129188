"""Parity at the full workload sizes, in the launch configuration the
benchmark times.  Where the oracle cannot afford every output (the 1M x 4
batch, the 2048-query prefill chunk) it checks whole sequences or whole KV
heads in full and samples the rest (spans, queries), plus properties that
hold at any size."""
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
    return reatt


def _device_inputs(w):
    x = wl.make_inputs(w, "cuda")
    torch.cuda.synchronize()
    return x


def _seq(x, b):
    return {n: x[n][b:b + 1] for n in parity.NAMES}


def test_llama3_8b_128k(R, ora):
    w = wl.WORKLOADS["llama3_8b_128k"]
    info = parity.full_check(R, ora, w, x=wl.make_inputs(w, "cpu"))
    print(info)


@pytest.mark.parametrize("name", ["qwen2_1p5b_4m", "llama3_8b_1m_x4"])
def test_long_decode(R, ora, name):
    """4M single sequence: every span scored by the oracle.  1M x 4: the whole
    batch runs on the GPU; sequences 0 and 3 are checked in full."""
    w = wl.WORKLOADS[name]
    x = _device_inputs(w)
    d = R.dims_of(w)
    gpu = parity.run_all(R, d, {n: x[n] for n in parity.NAMES})
    for b in ([0] if w.B == 1 else [0, w.B - 1]):
        wb = w.replace(B=1)
        xh = parity.host_inputs(_seq(x, b))
        ref = ora.step(**xh, G=w.G, L=w.L, S=w.S, k=w.k, rope_base=w.rope_base)
        parity.check_scores(gpu["span_scores"][b:b + 1], ref["scores"])
        swaps = parity.check_selection(ref["scores"], ref["sel"], gpu["sel_step"][b:b + 1], w.k)
        parity.check_selection(ref["scores"], ref["sel"], gpu["sel"][b:b + 1], w.k)
        err = parity.check_outputs(ora, xh, gpu["sel_step"][b:b + 1], gpu["out_step"][b:b + 1],
                                   wb, ref=ref)
        parity.check_outputs(ora, xh, gpu["sel"][b:b + 1], gpu["out"][b:b + 1], wb, ref=ref)
        for h in range(w.Hkv):
            assert set(x["needles"][b]) <= set(gpu["sel_step"][b, h].tolist())
        print(name, b, "swaps", swaps, "max-abs", err)
        del xh, ref


def test_llama3_8b_prefill_chunk(R, ora):
    """2048-query chunk over a 256K cache.

    * KV heads 0 and 5: the oracle scores every one of their 8,063 spans
      (max over the whole chunk's queries, the pages' prefill score), and the
      GPU's scores and selection of those heads meet the full bars: scores
      within 2e-5 of the head's max |score|, selection exact up to the swap
      rule.
    * The other heads: sampled spans (the lowest chosen and highest unchosen
      by GPU score, plus random ones) and the selection property on them.
    * Outputs of 64 queries touching all 16 query tiles of 128 (the first
      and last query of every tile plus 32 random ones), all 32 query heads."""
    w = wl.WORKLOADS["llama3_8b_prefill_256k"]
    x = _device_inputs(w)
    d = R.dims_of(w)
    gpu = parity.run_all(R, d, {n: x[n] for n in parity.NAMES})
    xh = parity.host_inputs(x)
    g = w.Hq // w.Hkv
    full_heads = (0, 5)
    for h in full_heads:
        sub = {"q": xh["q"][:, h * g:(h + 1) * g], "k_cache": xh["k_cache"][:, h:h + 1]}
        oscore = ora.span_scores(sub["q"], sub["k_cache"], w.G, w.L, w.S)   # [1, 1, NS]
        osel = ora.topk(oscore[0, 0], w.k)[None, None]
        parity.check_scores(gpu["span_scores"][:, h:h + 1], oscore)
        for key in ("sel_step", "sel"):
            swaps = parity.check_selection(oscore, osel, gpu[key][:, h:h + 1], w.k)
            print("head", h, key, "swaps", swaps)
    rng = np.random.default_rng(1)
    NS = gpu["span_scores"].shape[-1]
    pairs, groups = [], []
    for h in range(w.Hkv):
        if h in full_heads:
            continue
        sc = gpu["span_scores"][0, h]
        chosen = gpu["sel_step"][0, h]
        mask = np.zeros(NS, bool)
        mask[chosen] = True
        ch = np.flatnonzero(mask)
        un = np.flatnonzero(~mask)
        lo_ch = ch[np.argsort(sc[ch])[:6]]
        hi_un = un[np.argsort(sc[un])[::-1][:6]]
        rnd = rng.choice(NS, 6, replace=False)
        for sp in np.concatenate([lo_ch, hi_un, rnd]):
            pairs.append((h, int(sp)))
            groups.append(bool(mask[sp]))
    pairs = np.array(pairs, np.int64)
    oscore = ora.span_scores_list(xh["q"], xh["k_cache"], w.G, w.L, w.S, pairs)
    gscore = gpu["span_scores"][0][pairs[:, 0], pairs[:, 1]].astype(np.float64)
    scale = np.abs(oscore).max()
    assert np.abs(gscore - oscore).max() <= parity.SCORE_RTOL * scale
    groups = np.array(groups)
    for h in range(w.Hkv):
        if h in full_heads:
            continue
        m = pairs[:, 0] == h
        lo = oscore[m & groups].min()
        hi = oscore[m & ~groups].max()
        assert hi <= lo + parity.SWAP_REL * abs(lo), (h, lo, hi)
    tiles = np.arange(0, w.C, 128)
    edges = np.concatenate([tiles, tiles + 127])
    rest = np.setdiff1d(np.arange(w.C), edges)
    c_list = np.sort(np.concatenate([edges, rng.choice(rest, 32, replace=False)])).tolist()
    assert len(c_list) == 64 and len({c // 128 for c in c_list}) == w.C // 128
    for key in ("sel_step", "sel"):
        out_key = "out_step" if key == "sel_step" else "out"
        err = parity.check_outputs(ora, xh, gpu[key], gpu[out_key], w, c_list=c_list)
        print(key, "max-abs", err)
