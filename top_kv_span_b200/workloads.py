"""Seeded synthetic workloads for the top-k span attention step.

This module only *describes and draws inputs*: shapes, value distributions and
planted needle spans.  It computes no scores, no selection, no RoPE and no
attention, so both the CUDA path and the CPU oracle can be fed from it without
sharing any of the method's arithmetic.

Shapes follow the head geometry of the models the ReAttention pages evaluate
(LLaMA3-8B: 32 query / 8 KV heads of width 128; Qwen2-1.5B: 12 / 2) and the
window hyper-parameters of the OpenReview discussion's NIAH settings
(global 32, local 4096, span 32), with k = 64 spans.  The pages' own datasets
(LongBench, NIAH, InfiniteBench) need trained weights and are not used; these
caches stand in for them.

Distributions
-------------
* ``unit``:    q, K, V and the current-token K/V ~ N(0, 1).
* ``channel``: q ~ N(0, 1); K and V ~ N(0, sigma_c^2) with one sigma_c ~ U[0.5, 4]
  per (sequence, KV head, channel), drawn separately for K and V and shared by
  the cached and the current tokens.
* Needles: ``n_needles`` distinct full middle spans per sequence, chosen
  uniformly.  For KV head h every token of a needle span gets
  K = A * u_h + noise, where u_h is the unit vector along the sum of the
  group's query vectors (query position 0), A = 3 * sqrt(d) * sigma_rms
  (sigma_rms = rms of that head's K sigma_c, 1 for ``unit``) and the noise has
  per-channel std 0.1 * sigma_c.  V is left random.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    C: int
    T: int
    G: int
    L: int
    S: int
    k: int
    dtype: str          # "f32" or "bf16": dtype of q, caches and current tokens
    rope_base: float
    seed: int
    n_needles: int
    dist: str           # "unit" or "channel"
    description: str = ""

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self):
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_f32_4k": Workload(
        "tiny_f32_4k", B=1, Hq=4, Hkv=1, d=64, C=1, T=4096, G=4, L=256, S=32, k=8,
        dtype="f32", rope_base=1e4, seed=1000, n_needles=1, dist="unit",
        description="tiny fp32 decode, T=4096"),
    "llama3_8b_128k": Workload(
        "llama3_8b_128k", B=1, Hq=32, Hkv=8, d=128, C=1, T=131072, G=32, L=4096, S=32, k=64,
        dtype="bf16", rope_base=5e5, seed=1001, n_needles=4, dist="channel",
        description="LLaMA3-8B-shaped single-layer bf16 decode at 128K context"),
    "llama3_8b_1m_x4": Workload(
        "llama3_8b_1m_x4", B=4, Hq=32, Hkv=8, d=128, C=1, T=1048576, G=32, L=4096, S=32, k=64,
        dtype="bf16", rope_base=5e5, seed=1002, n_needles=8, dist="channel",
        description="LLaMA3-8B-shaped bf16 decode at 1M context, 4 independent sequences"),
    "llama3_8b_prefill_256k": Workload(
        "llama3_8b_prefill_256k", B=1, Hq=32, Hkv=8, d=128, C=2048, T=262144, G=32, L=4096,
        S=32, k=64, dtype="bf16", rope_base=5e5, seed=1003, n_needles=0, dist="channel",
        description="LLaMA3-8B-shaped bf16 chunked prefill: 2048-query chunk over 256K cache"),
    "llama3_8b_prefill_64k": Workload(
        "llama3_8b_prefill_64k", B=1, Hq=32, Hkv=8, d=128, C=2048, T=65536, G=32, L=4096,
        S=32, k=64, dtype="bf16", rope_base=5e5, seed=1005, n_needles=0, dist="channel",
        description="the 2048-query prefill chunk over a 64K cache: K+V 268 MB (more than "
                    "L2), the size full profiler captures of the prefill kernels run on"),
    "llama3_8b_1m": Workload(
        "llama3_8b_1m", B=1, Hq=32, Hkv=8, d=128, C=1, T=1048576, G=32, L=4096, S=32, k=64,
        dtype="bf16", rope_base=5e5, seed=1006, n_needles=8, dist="channel",
        description="one sequence of the 1M x 4 decode (K+V 4.3 GB): the size profiler "
                    "captures of its scan run on"),
    "qwen2_1p5b_4m": Workload(
        "qwen2_1p5b_4m", B=1, Hq=12, Hkv=2, d=128, C=1, T=4194304, G=32, L=4096, S=32, k=64,
        dtype="bf16", rope_base=1e6, seed=1004, n_needles=5, dist="channel",
        description="Qwen2-1.5B-shaped single-layer bf16 decode at 4M context"),
}

ORDER = ["tiny_f32_4k", "llama3_8b_128k", "llama3_8b_1m_x4", "llama3_8b_prefill_256k",
         "qwen2_1p5b_4m"]


def middle_span_rows(T: int, G: int, L: int, S: int):
    """Number of complete middle spans (the input recipe plants needles only there)."""
    M = max(0, T - G - L)
    return M // S


def _one_sequence(w: Workload, seed: int, device):
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    f32 = dict(dtype=torch.float32, device=device)
    Hq, Hkv, d, C, T = w.Hq, w.Hkv, w.d, w.C, w.T

    q = torch.randn((Hq, C, d), generator=gen, **f32)
    if w.dist == "channel":
        sk = torch.rand((Hkv, 1, d), generator=gen, **f32) * 3.5 + 0.5
        sv = torch.rand((Hkv, 1, d), generator=gen, **f32) * 3.5 + 0.5
    elif w.dist == "unit":
        sk = torch.ones((Hkv, 1, d), **f32)
        sv = torch.ones((Hkv, 1, d), **f32)
    else:
        raise ValueError(w.dist)

    kc = torch.empty((Hkv, T, d), dtype=w.torch_dtype, device=device)
    vc = torch.empty((Hkv, T, d), dtype=w.torch_dtype, device=device)
    for h in range(Hkv):  # one head at a time keeps the fp32 temporaries small
        kc[h] = (torch.randn((T, d), generator=gen, **f32) * sk[h]).to(w.torch_dtype)
        vc[h] = (torch.randn((T, d), generator=gen, **f32) * sv[h]).to(w.torch_dtype)
    kcur = (torch.randn((Hkv, C, d), generator=gen, **f32) * sk).to(w.torch_dtype)
    vcur = (torch.randn((Hkv, C, d), generator=gen, **f32) * sv).to(w.torch_dtype)

    needles = []
    nfull = middle_span_rows(T, w.G, w.L, w.S)
    n = min(w.n_needles, nfull)
    if n > 0:
        perm = torch.randperm(nfull, generator=gen, device=device)[:n]
        needles = sorted(int(v) for v in perm.cpu())
        g = Hq // Hkv
        for h in range(Hkv):
            qsum = q[h * g:(h + 1) * g, 0, :].sum(0)
            u = qsum / qsum.norm()
            sig = sk[h, 0]
            amp = 3.0 * math.sqrt(d) * float(sig.pow(2).mean().sqrt())
            for sp in needles:
                t0 = w.G + sp * w.S
                noise = torch.randn((w.S, d), generator=gen, **f32) * (0.1 * sig)
                kc[h, t0:t0 + w.S] = (amp * u + noise).to(w.torch_dtype)
    return q.to(w.torch_dtype), kc, vc, kcur, vcur, needles


def make_inputs(w: Workload, device="cpu"):
    """Draw one batch: dict of q [B,Hq,C,d], k_cache/v_cache [B,Hkv,T,d],
    k_cur/v_cur [B,Hkv,C,d] (all in the workload dtype on ``device``) and
    ``needles`` (list per sequence of planted span ids).  Sequence b uses seed
    ``w.seed + b``."""
    out = {name: [] for name in ("q", "k_cache", "v_cache", "k_cur", "v_cur", "needles")}
    for b in range(w.B):
        parts = _one_sequence(w, w.seed + b, device)
        for name, val in zip(("q", "k_cache", "v_cache", "k_cur", "v_cur", "needles"), parts):
            out[name].append(val)
    res = {name: torch.stack(out[name]) for name in ("q", "k_cache", "v_cache", "k_cur", "v_cur")}
    res["needles"] = out["needles"]
    return res


def to_oracle(t: torch.Tensor):
    """Host numpy view the oracle reads: float32 as is, bf16 as raw uint16 bits."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    raise TypeError(t.dtype)
