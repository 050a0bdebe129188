"""Caches allocated with room to grow (T_cap rows per KV head) and the append
of the current tokens' K/V: the strided caches give exactly the dense
results; a chunked prefill (first chunk G+L tokens, then fixed chunks, each
followed by its append) and a decoding loop captured in one CUDA graph both
match the oracle run on the dense caches of each step."""
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


def _strided(t, cap):
    """[B,H,T,d] -> [B,H,cap,d] with the T rows first and NaN after them."""
    B, H, T, d = t.shape
    out = torch.full((B, H, cap, d), float("nan"), dtype=t.dtype, device=t.device)
    out[:, :, :T] = t
    return out


@pytest.mark.parametrize("w", [
    LLAMA.replace(name="s_dec", Hq=8, Hkv=2, T=20000, L=512, k=16, n_needles=2, seed=60),
    LLAMA.replace(name="s_rag", Hq=8, Hkv=2, T=20003, L=512, k=16, n_needles=2, seed=61),
    LLAMA.replace(name="s_pre", Hq=8, Hkv=2, C=40, T=9000, L=256, k=10, n_needles=0, seed=62),
    TINY.replace(name="s_f32", B=2, Hq=6, Hkv=2, T=1003, G=3, L=17, S=7, k=5, n_needles=1,
                 seed=63),
], ids=lambda w: w.name)
def test_strided_caches_match_dense(R, w):
    x = {n: t.cuda() for n, t in wl.make_inputs(w).items() if n != "needles"}
    d = R.dims_of(w)
    b = R.alloc_outputs(d)
    R.reatt_step(d, x["q"], x["k_cache"], x["v_cache"], x["k_cur"], x["v_cur"], b["sel"],
                 b["out"], b["ws"])
    cap = w.T + 777
    ks, vs = _strided(x["k_cache"], cap), _strided(x["v_cache"], cap)
    ds = R.dims_of(w, T_cap=cap)
    bs = R.alloc_outputs(ds)
    R.reatt_step(ds, x["q"], ks, vs, x["k_cur"], x["v_cur"], bs["sel"], bs["out"], bs["ws"])
    torch.cuda.synchronize()
    assert torch.equal(bs["sel"], b["sel"])
    assert torch.equal(bs["out"], b["out"])


def _rand(shape, gen, dtype=torch.bfloat16, scale=1.0):
    return (torch.randn(shape, generator=gen) * scale).to(dtype)


def test_chunked_prefill_with_append(R, ora):
    """The pages' prefill: a first chunk of G+L tokens, then chunks of 512
    tokens (chunk_size=512 in the OpenReview discussion's NIAH settings) and
    a shorter last one; each chunk attends over the cache built so far (span
    selection on its middle) and is then appended."""
    B, Hq, Hkv, dh, G, L, S, k, base = 1, 8, 2, 128, 32, 256, 32, 8, 5e5
    chunks = [G + L] + [512] * 4 + [300]
    P = sum(chunks)
    gen = torch.Generator().manual_seed(70)
    q_all = _rand((B, Hq, P, dh), gen)
    sig = torch.rand((1, Hkv, 1, dh), generator=gen) * 3.5 + 0.5
    k_all = (_rand((B, Hkv, P, dh), gen, torch.float32) * sig).to(torch.bfloat16)
    v_all = (_rand((B, Hkv, P, dh), gen, torch.float32) * sig).to(torch.bfloat16)
    kc = torch.zeros((B, Hkv, P, dh), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    w = LLAMA.replace(name="chunked", B=B, Hq=Hq, Hkv=Hkv, d=dh, G=G, L=L, S=S, k=k,
                      rope_base=base)
    ws = torch.zeros(max(R.reatt_workspace_bytes(R.dims_of(w, T=P, C=max(chunks), T_cap=P)), 256),
                     dtype=torch.uint8, device="cuda")
    t = 0
    for c in chunks:
        d = R.dims_of(w, T=t, C=c, T_cap=P)
        qc = q_all[:, :, t:t + c].contiguous()
        kcur = k_all[:, :, t:t + c].contiguous()
        vcur = v_all[:, :, t:t + c].contiguous()
        qd, kd, vd = qc.cuda(), kcur.cuda(), vcur.cuda()
        sel = torch.empty((B, Hkv, k), dtype=torch.int32, device="cuda")
        out = torch.empty((B, Hq, c, dh), dtype=torch.float32, device="cuda")
        R.reatt_step(d, qd, kc, vc, kd, vd, sel, out, ws)
        R.reatt_append_kv(d, kc, vc, kd, vd)
        torch.cuda.synchronize()
        assert R.reatt_workspace_status(ws) == R.OK
        # oracle on the dense cache of this chunk
        xh = {"q": wl.to_oracle(qc), "k_cache": wl.to_oracle(k_all[:, :, :t].contiguous()),
              "v_cache": wl.to_oracle(v_all[:, :, :t].contiguous()),
              "k_cur": wl.to_oracle(kcur), "v_cur": wl.to_oracle(vcur)}
        wc = w.replace(T=t, C=c)
        ref = ora.step(**xh, G=G, L=L, S=S, k=k, rope_base=base)
        gsel = sel.cpu().numpy()
        if t > G + L:
            parity.check_selection(ref["scores"], ref["sel"], gsel, k)
        parity.check_outputs(ora, xh, gsel, out.cpu().numpy(), wc, ref=ref)
        t += c
    assert torch.equal(kc.cpu(), k_all) and torch.equal(vc.cpu(), v_all)


def test_decode_loop_in_one_graph(R, ora):
    """Several decode steps, each followed by its append, captured once in a
    CUDA graph: the replay equals the eager loop, and the steps match the
    oracle on the dense caches."""
    w = LLAMA.replace(name="loop", Hq=8, Hkv=2, T=6000, L=512, k=16, n_needles=1, seed=71)
    N = 5
    cap = w.T + N
    x = wl.make_inputs(w)
    gen = torch.Generator().manual_seed(72)
    qs = [_rand((w.B, w.Hq, 1, w.d), gen).cuda() for _ in range(N)]
    kn = [_rand((w.B, w.Hkv, 1, w.d), gen).cuda() for _ in range(N)]
    vn = [_rand((w.B, w.Hkv, 1, w.d), gen).cuda() for _ in range(N)]
    k0 = _strided(x["k_cache"].cuda(), cap)
    v0 = _strided(x["v_cache"].cuda(), cap)
    dims = [R.dims_of(w, T=w.T + i, T_cap=cap) for i in range(N)]
    ws = torch.zeros(max(R.reatt_workspace_bytes(d) for d in dims), dtype=torch.uint8,
                     device="cuda")
    outs = [torch.empty((w.B, w.Hq, 1, w.d), dtype=torch.float32, device="cuda") for _ in range(N)]
    sels = [torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda") for _ in range(N)]

    def loop(kc, vc, stream=None):
        for i in range(N):
            R.reatt_step(dims[i], qs[i], kc, vc, kn[i], vn[i], sels[i], outs[i], ws, stream=stream)
            R.reatt_append_kv(dims[i], kc, vc, kn[i], vn[i], stream=stream)

    ke, ve = k0.clone(), v0.clone()
    loop(ke, ve)
    torch.cuda.synchronize()
    eager = [(s.clone(), o.clone()) for s, o in zip(sels, outs)]
    kg, vg = k0.clone(), v0.clone()
    st = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=st):
        loop(kg, vg, stream=st)
    for _ in range(2):
        kg.copy_(k0)
        vg.copy_(v0)
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for (es, eo), s, o in zip(eager, sels, outs):
            assert torch.equal(s, es) and torch.equal(o, eo)
        assert torch.equal(kg[:, :, :cap], ke[:, :, :cap])
    # oracle on the dense caches of the first and the last step
    kd = ke[:, :, :cap].cpu()
    vd = ve[:, :, :cap].cpu()
    for i in (0, N - 1):
        T = w.T + i
        xh = {"q": wl.to_oracle(qs[i]), "k_cache": wl.to_oracle(kd[:, :, :T].contiguous()),
              "v_cache": wl.to_oracle(vd[:, :, :T].contiguous()),
              "k_cur": wl.to_oracle(kn[i]), "v_cur": wl.to_oracle(vn[i])}
        ref = ora.step(**xh, G=w.G, L=w.L, S=w.S, k=w.k, rope_base=w.rope_base)
        gsel = eager[i][0].cpu().numpy()
        parity.check_selection(ref["scores"], ref["sel"], gsel, w.k)
        parity.check_outputs(ora, xh, gsel, eager[i][1].cpu().numpy(), w.replace(T=T), ref=ref)
