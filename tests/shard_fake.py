"""CPU stand-in for the library's shard calls, built from the oracle's pinned
pieces (span scoring, top-k, window order, RoPE of a row) and written out in
numpy: it lets the sharded step's orchestration and its exchanges run on CPU
gloo ranks.  Test infrastructure only."""
import math

import numpy as np
import torch

from top_kv_span_b200 import reatt as R


def _np(t):
    return t.detach().cpu().numpy()


class FakeShardOps:
    """Same signatures as the binding's reatt_shard_* / reatt_merge_partials
    (fp32 inputs, CPU tensors)."""

    def __init__(self, ora):
        self.ora = ora

    # host-only size query: the library's own
    def reatt_shard_workspace_bytes(self, dims, shard, n):
        return R.reatt_shard_workspace_bytes(dims, shard, n)

    def _span_range(self, dims, shard):
        M = max(0, dims.T - dims.G - dims.L)
        NS = (M + dims.S - 1) // dims.S

        def at(t):
            return 0 if t <= dims.G else (NS if t >= dims.G + M else (t - dims.G) // dims.S)
        lo = at(shard.t_begin)
        return lo, max(lo, at(shard.t_end)), M, NS

    def reatt_shard_candidates(self, dims, shard, q, k_cache, cand_score, cand_id, ws,
                               stream=None):
        lo, hi, M, NS = self._span_range(dims, shard)
        cand_score.fill_(-math.inf)
        cand_id.fill_(-1)
        if hi <= lo:
            return
        # the shard's rows as a cache of their own whose middle is its spans
        t0 = shard.t_begin
        G_sub = dims.G + lo * dims.S - t0
        end = dims.G + min(M, hi * dims.S)
        kc = _np(k_cache)[:, :, :shard.t_end - t0]
        L_sub = (shard.t_end - t0) - (end - t0)
        sc = self.ora.span_scores(_np(q), np.ascontiguousarray(kc), G_sub, L_sub, dims.S)
        for b in range(dims.B):
            for h in range(dims.Hkv):
                sel = self.ora.topk(sc[b, h], dims.k)
                for i, s in enumerate(sel):
                    if s >= 0:
                        cand_id[b, h, i] = int(s) + lo
                        cand_score[b, h, i] = float(sc[b, h, s])

    def reatt_shard_select(self, dims, n, cand_score_all, cand_id_all, sel, ws, stream=None):
        cs, ci = _np(cand_score_all), _np(cand_id_all)
        NS = self._span_range(dims, R.reatt_shard(0, dims.T, 0, 1, 0))[3]
        keff = min(dims.k, NS)
        sel.fill_(-1)
        for b in range(dims.B):
            for h in range(dims.Hkv):
                pool = [(-float(cs[r, b, h, i]), int(ci[r, b, h, i]))
                        for r in range(n) for i in range(dims.k) if ci[r, b, h, i] >= 0]
                chosen = sorted(i for _, i in sorted(pool)[:keff])
                sel[b, h, :len(chosen)] = torch.tensor(chosen, dtype=torch.int32)

    def reatt_shard_attend(self, dims, shard, q, k_cache, v_cache, k_cur, v_cur, sel, part_ml,
                           part_acc, ws, stream=None):
        qn, kn, vn = _np(q).astype(np.float64), _np(k_cache), _np(v_cache)
        kcn, vcn, sn = _np(k_cur), _np(v_cur), _np(sel)
        g = dims.Hq // dims.Hkv
        log2e = 1.0 / math.log(2.0)
        ml = np.zeros((dims.B, dims.Hq, dims.C, 2))
        acc = np.zeros((dims.B, dims.Hq, dims.C, dims.d))
        for b in range(dims.B):
            for h in range(dims.Hkv):
                src = self.ora.window(dims.T, dims.G, dims.L, dims.S, dims.C, sn[b, h])
                W = len(src)
                held = [(p, s) for p, s in enumerate(src)
                        if (s >= 0 and shard.t_begin <= s < shard.t_end) or
                        (s < 0 and shard.owns_current)]
                keys, vals, pos = [], [], []
                for p, s in held:
                    if s >= 0:
                        kr, vr = kn[b, h, s - shard.t_begin], vn[b, h, s - shard.t_begin]
                    else:
                        kr, vr = kcn[b, h, -s - 1], vcn[b, h, -s - 1]
                    keys.append(self.ora.rope_row(kr, p, dims.rope_base))
                    vals.append(vr.astype(np.float64))
                    pos.append(p)
                for jj in range(g):
                    j = h * g + jj
                    for c in range(dims.C):
                        qp = W - dims.C + c
                        qr = self.ora.rope_row(qn[b, j, c], qp, dims.rope_base)
                        vis = [i for i, p in enumerate(pos) if p <= qp]
                        if not vis:
                            ml[b, j, c] = (-math.inf, 0.0)
                            continue
                        z = np.array([qr @ keys[i] for i in vis]) / math.sqrt(dims.d) * log2e
                        m = z.max()
                        w = np.exp2(z - m)
                        ml[b, j, c] = (m, w.sum())
                        acc[b, j, c] = sum(wi * vals[i] for wi, i in zip(w, vis))
        part_ml.copy_(torch.from_numpy(ml).to(part_ml.dtype))
        part_acc.copy_(torch.from_numpy(acc).to(part_acc.dtype))

    def reatt_merge_partials(self, dims, n, part_ml_all, part_acc_all, out, stream=None):
        ml, acc = _np(part_ml_all).astype(np.float64), _np(part_acc_all).astype(np.float64)
        m = ml[..., 0]
        M = m.max(0)
        f = np.where(np.isneginf(m), 0.0, np.exp2(m - M))
        den = (f * ml[..., 1]).sum(0)
        num = (f[..., None] * acc).sum(0)
        out.copy_(torch.from_numpy(num / den[..., None]).to(out.dtype))
