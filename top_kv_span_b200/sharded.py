"""One sequence's KV cache split by token ranges over several GPUs.

The research-map summary ("Limitations") and the OpenReview discussion
(reply on W4, "memory overhead tradeoff") name memory as the method's bound:
a long enough sequence outgrows one GPU.  ``ShardedStep`` runs the step of
one rank that holds a contiguous token range of every (batch, KV head) of
the cache, through the C ABI's shard calls (``include/reatt.h``):

  1. ``reatt_shard_candidates``  this rank's own top-k (score, span id);
  2. exchange                    every rank receives every rank's candidates;
  3. ``reatt_shard_select``      the global top-k (the same on every rank);
  4. ``reatt_shard_attend``      partial attention over the window rows held
                                 here, at their positions in the whole window;
  5. exchange                    every rank receives every rank's partial;
  6. ``reatt_merge_partials``    the log-sum-exp merge into the output.

The two exchanges are all-gathers of a few KB (k candidates per (b, h);
d + 2 floats per query row) through ``torch.distributed`` (NCCL between GPUs);
``dist_all_gather`` makes one for a process group.  Every step of the path
itself runs in the library's kernels; this module only allocates buffers and
orders the calls.
"""
from __future__ import annotations

import torch

from . import reatt as R


def dist_all_gather(group=None):
    """All-gather over a torch.distributed group: gather(dst [n, ...], src)."""
    import torch.distributed as dist

    def gather(dst, src):
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(dst, src.contiguous(), group=group)
        else:   # gloo: list form
            parts = list(dst.unbind(0))
            dist.all_gather(parts, src.contiguous(), group=group)
    return gather


class ShardedStep:
    """Buffers and call order of one rank's sharded step.

    dims: the whole sequence's dims (T = all cached tokens); shard: this
    rank's ``reatt_shard``; n_shards: ranks in the group, in token order."""

    def __init__(self, dims, shard, n_shards, device="cuda", ops=R):
        self.dims, self.shard, self.n = dims, shard, int(n_shards)
        self.ops = ops
        B, Hq, Hkv, C, d, k = dims.B, dims.Hq, dims.Hkv, dims.C, dims.d, dims.k
        f32, i32 = torch.float32, torch.int32
        ws = ops.reatt_shard_workspace_bytes(dims, shard, self.n)
        self.ws = torch.zeros(max(ws, 256), dtype=torch.uint8, device=device)
        self.cand_score = torch.empty((B, Hkv, k), dtype=f32, device=device)
        self.cand_id = torch.empty((B, Hkv, k), dtype=i32, device=device)
        self.cand_score_all = torch.empty((self.n, B, Hkv, k), dtype=f32, device=device)
        self.cand_id_all = torch.empty((self.n, B, Hkv, k), dtype=i32, device=device)
        self.sel = torch.empty((B, Hkv, k), dtype=i32, device=device)
        self.part_ml = torch.empty((B, Hq, C, 2), dtype=f32, device=device)
        self.part_acc = torch.empty((B, Hq, C, d), dtype=f32, device=device)
        self.part_ml_all = torch.empty((self.n, B, Hq, C, 2), dtype=f32, device=device)
        self.part_acc_all = torch.empty((self.n, B, Hq, C, d), dtype=f32, device=device)

    # the phases, for callers that exchange by other means
    def candidates(self, q, k_cache, stream=None):
        self.ops.reatt_shard_candidates(self.dims, self.shard, q, k_cache, self.cand_score,
                                        self.cand_id, self.ws, stream)

    def select(self, stream=None):
        self.ops.reatt_shard_select(self.dims, self.n, self.cand_score_all, self.cand_id_all,
                                    self.sel, self.ws, stream)

    def attend(self, q, k_cache, v_cache, k_cur, v_cur, stream=None):
        self.ops.reatt_shard_attend(self.dims, self.shard, q, k_cache, v_cache, k_cur, v_cur,
                                    self.sel, self.part_ml, self.part_acc, self.ws, stream)

    def merge(self, out, stream=None):
        self.ops.reatt_merge_partials(self.dims, self.n, self.part_ml_all, self.part_acc_all,
                                      out, stream)

    def __call__(self, q, k_cache, v_cache, k_cur, v_cur, out, gather, stream=None):
        """The whole step on this rank; `gather(dst, src)` is the all-gather
        of the group (every rank calls it in the same order).  Returns out."""
        self.candidates(q, k_cache, stream)
        gather(self.cand_score_all, self.cand_score)
        gather(self.cand_id_all, self.cand_id)
        self.select(stream)
        self.attend(q, k_cache, v_cache, k_cur, v_cur, stream)
        gather(self.part_ml_all, self.part_ml)
        gather(self.part_acc_all, self.part_acc)
        self.merge(out, stream)
        return out


def shard_rows(t, shard):
    """This shard's rows [t_begin, t_end) of a whole-sequence cache [B,Hkv,T,d]."""
    return t[:, :, shard.t_begin:shard.t_end].contiguous()
