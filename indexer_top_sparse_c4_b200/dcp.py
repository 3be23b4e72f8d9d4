"""Sequence-sharded decode (decode context parallelism) over R shards, each
holding a contiguous range of every request's pages.

Plumbing only: buffers, the shard bounds, the all-gathers between ranks and
the order of the library calls.  Every step of the computation is a libqsa
call (see include/qsa.h, "Sequence-sharded decode"):

    per shard: qsa_dcp_shard_positions -> qsa_index_scores -> qsa_topk_groups
               -> qsa_dcp_candidates                         (records [T, K])
    all-gather of the records                                ([R, T, K])
    qsa_dcp_merge_topk                                       (global sel)
    per shard: qsa_dcp_expand -> qsa_sparse_attn_decode      (partial o, lse)
    all-gather of the partials; qsa_dcp_merge_attn          (out, lse)

With a torch.distributed process group, rank r runs shard r and the
all-gathers are collectives (NCCL on GPUs); without one, a single device runs
every shard in turn over the shared cache and the gathered tensors are simply
the stacked per-shard buffers.
"""
from __future__ import annotations

from typing import List, Tuple

import torch

from . import qsa
from .workloads import GROUP_TOKENS, PAGE_GROUPS, Workload


def shard_bounds(pages_per_req: int, shards: int) -> List[Tuple[int, int]]:
    """Contiguous page ranges [lo, hi) of the shards: as equal as whole pages
    allow, the first shards taking the extra page."""
    base, extra = divmod(pages_per_req, shards)
    out, lo = [], 0
    for r in range(shards):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def gather(x: torch.Tensor, group=None) -> torch.Tensor:
    """[R, *x.shape] of every rank's x, in rank order (an all-gather; NCCL on
    GPUs, gloo on the host)."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    parts = [torch.empty_like(x) for _ in range(R)]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


class QSADcpDecode:
    def __init__(self, w: Workload, shards: int, group=None):
        import torch.distributed as dist
        self.w, self.R, self.group = w, shards, group
        if group is not None and dist.get_world_size(group) != shards:
            raise ValueError("one shard per rank")
        self.mine = [dist.get_rank(group)] if group is not None else list(range(shards))
        dev = w.q.device
        T, K = w.T, w.K
        P = w.page_table.shape[1]
        self.bounds = shard_bounds(P, shards)
        self.W = GROUP_TOKENS * K + GROUP_TOKENS        # every selected group on one shard, plus the block
        self.status = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.cand_score = torch.empty((shards, T, K), dtype=torch.float32, device=dev)
        self.cand_id = torch.empty((shards, T, K), dtype=torch.int32, device=dev)
        self.o_parts = torch.empty((shards, T, w.Hq, w.D), dtype=torch.float32, device=dev)
        self.lse_parts = torch.empty((shards, T, w.Hq), dtype=torch.float32, device=dev)
        self.sel = torch.empty((T, K), dtype=torch.int32, device=dev)
        self.n_sel = torch.empty((T,), dtype=torch.int32, device=dev)
        out_dtype = torch.float32 if w.q.dtype == torch.float32 else torch.bfloat16
        self.out = torch.empty((T, w.Hq, w.D), dtype=out_dtype, device=dev)
        self.lse = torch.empty((T, w.Hq), dtype=torch.float32, device=dev)
        self.sh = {}
        for r in self.mine:
            lo, hi = self.bounds[r]
            groups = (hi - lo) * PAGE_GROUPS
            stride = max(4, -(-groups // 4) * 4)
            ws = qsa.qsa_sparse_attn_decode_workspace_size(T, w.Hq, w.Hkv, w.D, self.W, w.k_pages.dtype)
            self.sh[r] = dict(
                g_lo=lo * PAGE_GROUPS, g_hi=hi * PAGE_GROUPS,
                pt=w.page_table[:, lo:hi].contiguous(),
                q_pos=torch.empty((T,), dtype=torch.int32, device=dev),
                scores=torch.empty((T, stride), dtype=torch.float32, device=dev),
                hist=torch.zeros((T, qsa.QSA_PREFIX_HIST_BINS), dtype=torch.int32, device=dev),
                sel=torch.empty((T, K), dtype=torch.int32, device=dev),
                n_sel=torch.empty((T,), dtype=torch.int32, device=dev),
                tok=torch.empty((T, self.W), dtype=torch.int32, device=dev),
                n_tok=torch.empty((T,), dtype=torch.int32, device=dev),
                ws=torch.empty((max(ws, 16),), dtype=torch.uint8, device=dev))

    def select(self, stream=None):
        """Stages 1 and 2 on every owned shard, the records, their gather and merge."""
        w = self.w
        for r in self.mine:
            s = self.sh[r]
            qsa.qsa_dcp_shard_positions(w.q_pos, s["g_lo"], s["g_hi"], s["q_pos"], stream=stream)
            qsa.qsa_index_scores(w.q_idx, w.w_idx, w.k_idx_pages, s["pt"], s["q_pos"], s["scores"], q_req=w.q_req,
                                 dev_status=self.status, stream=stream, prefix_hist=s["hist"])
            qsa.qsa_topk_groups(s["scores"], s["q_pos"], w.K, s["sel"], s["n_sel"], dev_status=self.status,
                                stream=stream, prefix_hist=s["hist"])
            qsa.qsa_dcp_candidates(s["scores"], s["sel"], s["n_sel"], s["g_lo"], self.cand_score[r], self.cand_id[r],
                                   dev_status=self.status, stream=stream)
        if self.group is not None:
            r = self.mine[0]
            self.cand_score.copy_(gather(self.cand_score[r], self.group))
            self.cand_id.copy_(gather(self.cand_id[r], self.group))
        qsa.qsa_dcp_merge_topk(self.cand_score, self.cand_id, self.sel, self.n_sel, stream=stream)

    def attend(self, stream=None, sm_scale=0.0):
        """Stages 3 and 4 on every owned shard, the partials' gather and merge."""
        w = self.w
        for r in self.mine:
            s = self.sh[r]
            qsa.qsa_dcp_expand(self.sel, self.n_sel, w.q_pos, s["g_lo"], s["g_hi"], s["tok"], s["n_tok"],
                               dev_status=self.status, stream=stream)
            qsa.qsa_sparse_attn_decode(w.q, w.k_pages, w.v_pages, s["pt"], s["tok"], s["n_tok"], self.o_parts[r],
                                       workspace=s["ws"], k_scale=w.k_scale, v_scale=w.v_scale, q_req=w.q_req,
                                       sm_scale=sm_scale, lse=self.lse_parts[r], dev_status=self.status,
                                       stream=stream)
        if self.group is not None:
            r = self.mine[0]
            self.o_parts.copy_(gather(self.o_parts[r], self.group))
            self.lse_parts.copy_(gather(self.lse_parts[r], self.group))
        qsa.qsa_dcp_merge_attn(self.o_parts, self.lse_parts, self.out, self.lse, stream=stream)

    def run(self, stream=None, sm_scale=0.0):
        self.select(stream)
        self.attend(stream, sm_scale)
        return self.out
