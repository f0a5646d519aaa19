"""The DSA decode layer-step with each sequence's context split over the
ranks of a process group: rank r holds positions [offset_r, offset_r + len_r)
in its own caches.  The steps run in libdsa's kernels (see include/dsa.h,
"Context-sharded decode"); this module only enqueues them and the two
exchanges, which are all-gathers over the process group (NCCL on GPUs):

  local selection  indexer + top-k over the rank's slice
  exchange 1       all-gather of (score, global position), top_k per row
  merge            the global top-k, identical on every rank
  local attention  over the rank's share of the selection, no sink
  exchange 2       all-gather of (O_r, lse_r)
  combine          log-sum-exp merge, the sink added once

`ops` carries the per-rank operations: the library's by default; tests on
hosts without a GPU pass stand-ins with the same signatures to exercise the
exchange protocol over gloo.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist


@dataclass
class Shard:
    offset: int          # first position of this rank's slice
    length: int          # positions in the slice
    Lmax_local: int      # scores buffer length of the local indexer (>= visible positions of the slice)


class LibOps:
    """The library's kernels (a CUDA device)."""

    def __init__(self):
        from . import (OP_INDEXER, OP_PRODUCE, OP_SPARSE_ATTN, OP_TOPK, alloc_workspace, dsa_indexer_scores,
                       dsa_shard_candidates, dsa_shard_combine, dsa_shard_merge, dsa_shard_positions,
                       dsa_topk_select, sparse_gqa_attn_decode)
        self._f = dict(ws=alloc_workspace, positions=dsa_shard_positions, indexer=dsa_indexer_scores,
                       topk=dsa_topk_select, candidates=dsa_shard_candidates, merge=dsa_shard_merge,
                       attention=sparse_gqa_attn_decode, combine=dsa_shard_combine)
        self.OP = dict(indexer=OP_INDEXER, produce=OP_PRODUCE, attn=OP_SPARSE_ATTN, topk=OP_TOPK)
        self._ws = {}

    def _workspace(self, op, B, T, L, k, device):
        key = (op, B, T, L, k, str(device))
        if key not in self._ws:
            self._ws[key] = self._f["ws"](self.OP[op], B, T, L, k, device=device)
        return self._ws[key]

    def local_select(self, q8, q_scale, w, kv, q_pos, shard: Shard, top_k):
        B, T = q_pos.shape
        dev = q_pos.device
        q_local = torch.empty_like(q_pos)
        self._f["positions"](q_pos, shard.offset, shard.length, q_local, self._workspace("produce", B, T, 1, 1, dev))
        L = shard.Lmax_local
        scores = torch.empty((B, T, L), dtype=torch.float32, device=dev)
        self._f["indexer"](q8, q_scale, w, kv, q_local, L, scores, self._workspace("indexer", B, T, L, 1, dev))
        idx = torch.empty((B, T, top_k), dtype=torch.int32, device=dev)
        cnt = torch.empty((B, T), dtype=torch.int32, device=dev)
        self._f["topk"](scores, q_local, L, top_k, idx, cnt, self._workspace("topk", B, T, L, top_k, dev))
        cs = torch.empty((B, T, top_k), dtype=torch.float32, device=dev)
        cp = torch.empty((B, T, top_k), dtype=torch.int32, device=dev)
        self._f["candidates"](scores, idx, top_k, shard.offset, cs, cp)
        return cs, cp

    def merge(self, cs_all, cp_all, top_k, shard: Shard):
        N, B, T = cp_all.shape[:3]
        dev = cp_all.device
        idx = torch.empty((B, T, top_k), dtype=torch.int32, device=dev)
        cnt = torch.empty((B, T), dtype=torch.int32, device=dev)
        lidx = torch.empty_like(idx)
        lcnt = torch.empty_like(cnt)
        self._f["merge"](cs_all, cp_all, top_k, shard.offset, shard.length, idx, cnt, lidx, lcnt)
        return idx, cnt, lidx, lcnt

    def local_attention(self, Q, kv, lidx, lcnt, top_k, sm_scale):
        B, T = lcnt.shape
        dev = Q.device
        O = torch.empty((B, T, 64, 128), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, T, 64), dtype=torch.float32, device=dev)
        self._f["attention"](Q, kv, lidx, lcnt, top_k, None, sm_scale, O, lse,
                             self._workspace("attn", B, T, 1, top_k, dev))
        return O, lse

    def combine(self, O_all, lse_all, sink, O, lse):
        self._f["combine"](O_all, lse_all, sink, O, lse)


def sharded_layer_decode(q8, q_scale, w, Q, kv, q_pos, shard: Shard, top_k: int, sink, sm_scale: float, O,
                         lse=None, group: Optional[dist.ProcessGroup] = None, ops=None):
    """This rank's part of the layer-step; every rank of `group` calls it with
    the same q8 / q_scale / w / Q / q_pos / sink (the query side is
    replicated) and its own `kv` slice.  Writes the full O (and lse) on every
    rank; returns (idx, count) of the merged selection (global positions)."""
    ops = ops or LibOps()
    N = dist.get_world_size(group) if dist.is_initialized() else 1
    cs, cp = ops.local_select(q8, q_scale, w, kv, q_pos, shard, top_k)
    cs_all, cp_all = _gather(cs, N, group), _gather(cp, N, group)
    idx, cnt, lidx, lcnt = ops.merge(cs_all, cp_all, top_k, shard)
    O_r, lse_r = ops.local_attention(Q, kv, lidx, lcnt, top_k, sm_scale)
    ops.combine(_gather(O_r, N, group), _gather(lse_r, N, group), sink, O, lse)
    return idx, cnt


def _gather(x: torch.Tensor, N: int, group) -> torch.Tensor:
    """[N, *x.shape]: every rank's x in rank order (an all-gather into one
    buffer, concatenated along the first dimension)."""
    x = x.contiguous()
    out = torch.empty((N * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    if N > 1:
        dist.all_gather_into_tensor(out, x, group=group)
    else:
        out.copy_(x)
    return out.view((N,) + tuple(x.shape))
