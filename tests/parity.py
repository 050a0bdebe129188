"""Shared parity checks: CUDA path (through the C ABI) against the CPU oracle.

Acceptance bars:
  * selection: the chosen span sets match the oracle's exactly, except swaps
    among spans whose oracle score lies within 1e-3 relative of the oracle's
    k-th score; the number of such swaps is reported;
  * outputs: max-abs 1e-4 (fp32 inputs) / 2e-2 (bf16 inputs) against the oracle
    run on the same input bits (with the GPU's selection when a tolerated swap
    happened);
  * span scores: fp32 accumulation against fp64, relative to the head's
    largest |score| (2e-5).
"""
import numpy as np
import torch

from top_kv_span_b200 import workloads as wl

OUT_TOL = {"f32": 1e-4, "bf16": 2e-2}
SCORE_RTOL = 2e-5
SWAP_REL = 1e-3
NAMES = ("q", "k_cache", "v_cache", "k_cur", "v_cur")


def host_inputs(x):
    return {n: wl.to_oracle(x[n]) for n in NAMES}


def run_all(R, d, x, stream=None):
    """Every entry point on device inputs x; returns host numpy results."""
    b = R.alloc_outputs(d)
    R.reatt_score_spans(d, x["q"], x["k_cache"], b["span_scores"], b["ws"], stream)
    R.reatt_topk(d, b["span_scores"], b["sel"], b["ws"], stream)
    R.reatt_gather_rope(d, x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                        b["k_win"], b["v_win"], b["win_len"], stream)
    R.reatt_attend(d, x["q"], b["k_win"], b["v_win"], b["win_len"], b["out"], b["ws"], stream)
    sel_step = torch.full_like(b["sel"], -7)
    out_step = torch.full_like(b["out"], float("nan"))
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], sel_step,
                 out_step, b["ws"], stream)
    torch.cuda.synchronize()
    assert R.reatt_workspace_status(b["ws"]) == 0
    res = {k: v.cpu().numpy() for k, v in b.items() if k != "ws"}
    res["sel_step"] = sel_step.cpu().numpy()
    res["out_step"] = out_step.cpu().numpy()
    return res


def check_scores(gpu, ora):
    assert gpu.shape == ora.shape
    for idx in np.ndindex(ora.shape[:2]):
        o, g = ora[idx], gpu[idx].astype(np.float64)
        if o.size == 0:
            continue
        scale = max(1.0, float(np.abs(o).max()))
        err = float(np.abs(g - o).max())
        assert err <= SCORE_RTOL * scale, f"scores {idx}: err {err} scale {scale}"


def kth_score(scores, keff):
    return np.sort(scores)[::-1][keff - 1]


def check_selection(ora_scores, ora_sel, gpu_sel, k):
    """Swap rule; returns the number of tolerated swaps."""
    swaps = 0
    NS = ora_scores.shape[-1]
    keff = min(k, NS)
    for idx in np.ndindex(ora_sel.shape[:2]):
        g = gpu_sel[idx]
        assert (g[keff:] == -1).all(), f"padding {idx}: {g[keff:]}"
        gv = g[:keff]
        assert (np.diff(gv) > 0).all(), f"not ascending {idx}"
        assert ((gv >= 0) & (gv < NS)).all()
        O, Gs = set(ora_sel[idx][:keff].tolist()), set(gv.tolist())
        if O == Gs:
            continue
        sk = kth_score(ora_scores[idx], keff)
        for sp in O ^ Gs:
            assert abs(ora_scores[idx][sp] - sk) <= SWAP_REL * abs(sk), \
                f"{idx}: span {sp} score {ora_scores[idx][sp]} vs k-th {sk}"
        swaps += len(O - Gs)
    return swaps


def check_outputs(ora, xh, gpu_sel, gpu_out, w, c_list=None, ref=None):
    """Compare outputs against the oracle; when the selection differs, the
    oracle is re-run on the GPU's selection (attention-only check)."""
    tol = OUT_TOL[w.dtype]
    if ref is None or not np.array_equal(ref["sel"], gpu_sel):
        ref = ora.step(**xh, G=w.G, L=w.L, S=w.S, k=w.k, rope_base=w.rope_base,
                       sel=gpu_sel, c_list=c_list)
    o = ref["out"]
    g = gpu_out.astype(np.float64)
    if c_list is not None:
        o, g = o[:, :, c_list], g[:, :, c_list]
    assert np.isfinite(g).all()
    err = float(np.abs(g - o).max())
    assert err <= tol, f"max-abs {err} > {tol}"
    return err


def full_check(R, ora, w, x=None, dims=None):
    """All entry points vs the oracle on one workload (sizes the oracle finishes fast)."""
    if x is None:
        x = wl.make_inputs(w, "cpu")
    xd = {n: x[n].cuda() for n in NAMES}
    d = dims or R.dims_of(w)
    gpu = run_all(R, d, xd)
    xh = host_inputs(x)
    ref = ora.step(**xh, G=w.G, L=w.L, S=w.S, k=w.k, rope_base=w.rope_base)
    check_scores(gpu["span_scores"], ref["scores"])
    swaps = check_selection(ref["scores"], ref["sel"], gpu["sel"], w.k)
    # reatt_step's selection must equal the standalone top-k of the same scores
    # only up to the same tolerance (its scores come from the same kernel)
    swaps_step = check_selection(ref["scores"], ref["sel"], gpu["sel_step"], w.k)
    assert (gpu["win_len"] == ref["win_len"]).all() or not np.array_equal(gpu["sel"], ref["sel"])
    err_split = check_outputs(ora, xh, gpu["sel"], gpu["out"], w, ref=ref)
    err_step = check_outputs(ora, xh, gpu["sel_step"], gpu["out_step"], w, ref=ref)
    check_window(ora, xh, w, gpu)
    for needles, b in zip(x["needles"], range(w.B)):
        for h in range(w.Hkv):
            assert set(needles) <= set(gpu["sel_step"][b, h].tolist())
    return dict(swaps=swaps, swaps_step=swaps_step, err_split=err_split, err_step=err_step)


def check_window(ora, xh, w, gpu, max_rows=64):
    """Materialised window rows: K rotated at its window position, V copied."""
    rng = np.random.default_rng(0)
    tol = 2e-5
    for b in range(w.B):
        for h in range(w.Hkv):
            src = ora.window(w.T, w.G, w.L, w.S, w.C, gpu["sel"][b, h])
            W = len(src)
            assert gpu["win_len"][b, h] == W
            rows = np.arange(W) if W <= max_rows else np.unique(
                np.concatenate([[0, W - 1], rng.choice(W, max_rows, replace=False)]))
            for p in rows:
                s = src[p]
                if s >= 0:
                    kr, vr = xh["k_cache"][b, h, s], xh["v_cache"][b, h, s]
                else:
                    kr, vr = xh["k_cur"][b, h, -s - 1], xh["v_cur"][b, h, -s - 1]
                from tests.textbook import bits_to_f64
                kf, vf = bits_to_f64(kr), bits_to_f64(vr)
                want = ora.rope_row(kf, p, w.rope_base)
                got = gpu["k_win"][b, h, p].astype(np.float64)
                assert np.abs(got - want).max() <= tol * max(1.0, np.abs(kf).max()), (b, h, p)
                assert np.array_equal(gpu["v_win"][b, h, p].astype(np.float64), vf)
