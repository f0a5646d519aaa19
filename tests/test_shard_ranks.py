"""The context-sharded decode protocol on CPU: two `gloo` ranks, each holding
half of one sequence's context, exchange their local top-k candidates and
their attention outputs through local_attention_decode_b200.sharded; the
result is the one-process layer-step over the whole context.

The per-rank operations are CPU stand-ins written here from the oracle (the
kernels need a GPU); what is tested is the exchange protocol: rank order of
the gathered tensors, global positions, the owner split of the selection, and
the sink added once in the combine.  The kernels themselves are compared with
the one-GPU layer-step in tests/test_gpu_shard.py.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from workloads import bits16, make_decode_workload

L, TOP_K, SM = 6000, 256, 1.0 / math.sqrt(192)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """Per-rank operations in plain numpy on the oracle."""

    def __init__(self, wl):
        self.wl = wl

    def local_select(self, q8, q_scale, w, kv, q_pos, shard, top_k):
        k8, ks = kv
        p = int(q_pos[0, 0]) - shard.offset
        p = min(p, shard.length - 1)
        s = oracle.indexer_scores(q8[0].numpy(), q_scale[0].numpy(), w[0].numpy(), k8, ks, np.array([p], np.int32))[0]
        idx, c = oracle.topk(s[:p + 1], top_k)
        idx = np.sort(idx[:c])
        cs = np.full(top_k, -np.inf, np.float32)
        cp = np.full(top_k, -1, np.int32)
        cs[:c] = s[idx]
        cp[:c] = idx + shard.offset
        return torch.from_numpy(cs).view(1, 1, top_k), torch.from_numpy(cp).view(1, 1, top_k)

    def merge(self, cs_all, cp_all, top_k, shard):
        cs, cp = cs_all.reshape(-1).numpy(), cp_all.reshape(-1).numpy()
        ok = cp >= 0
        order = sorted(zip(-cs[ok].astype(np.float64), cp[ok]))[:top_k]
        sel = np.sort(np.array([p for _, p in order], np.int32))
        mine = sel[(sel >= shard.offset) & (sel < shard.offset + shard.length)] - shard.offset
        return (torch.from_numpy(sel).view(1, 1, -1), torch.tensor([[len(sel)]]),
                torch.from_numpy(mine.astype(np.int32)).view(1, 1, -1), torch.tensor([[len(mine)]]))

    def local_attention(self, Q, kv, lidx, lcnt, top_k, sm_scale):
        rows = lidx.reshape(-1).numpy()
        o, l = oracle.gqa_attention(bits16(Q[0, 0]), self.K_local, self.V_local, rows, None, sm_scale)
        return torch.from_numpy(o).view(1, 1, 64, 128), torch.from_numpy(l).view(1, 1, 64)

    def combine(self, O_all, lse_all, sink, O, lse):
        l = lse_all.numpy()[:, 0, 0]                            # [N, 64]
        s = sink.numpy().astype(np.float64)
        M = np.maximum(l.max(0), s)
        wts = np.exp(l - M)                                     # [N, 64]
        den = wts.sum(0) + np.exp(s - M)
        o = (wts[:, :, None] * O_all.numpy()[:, 0, 0]).sum(0) / den[:, None]
        O.copy_(torch.from_numpy(o).view(O.shape))
        lse.copy_(torch.from_numpy(M + np.log(den)).view(lse.shape))


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from local_attention_decode_b200.sharded import Shard, sharded_layer_decode
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = make_decode_workload(seed=140, seq_lens=[L], T=1, n_needles=8)
        half = L // world
        shard = Shard(offset=rank * half, length=half if rank < world - 1 else L - rank * half, Lmax_local=0)
        sl = slice(shard.offset, shard.offset + shard.length)
        ops = OracleOps(wl)
        ops.K_local, ops.V_local = bits16(wl.K[sl]), bits16(wl.V[sl])
        kv = (wl.k8[sl].numpy(), wl.k_scale[sl].numpy())
        O = torch.zeros((1, 1, 64, 128), dtype=torch.float64)
        lse = torch.zeros((1, 1, 64), dtype=torch.float64)
        idx, cnt = sharded_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, shard, TOP_K, wl.sink, SM, O,
                                        lse, ops=ops)
        out.put((rank, idx.numpy(), O.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reproduce_the_one_process_layer_step():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((out.get(timeout=240) for _ in procs), key=lambda g: g[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the one-process reference over the whole context
    wl = make_decode_workload(seed=140, seq_lens=[L], T=1, n_needles=8)
    s = oracle.indexer_scores(wl.q8[0].numpy(), wl.q_scale[0].numpy(), wl.w[0].numpy(), wl.k8.numpy(),
                              wl.k_scale.numpy(), wl.q_pos[0].numpy())[0]
    ref_idx, c = oracle.topk(s, TOP_K)
    ref_sel = np.sort(ref_idx[:c])
    ref_o, ref_l = oracle.gqa_attention(bits16(wl.Q[0, 0]), bits16(wl.K), bits16(wl.V), ref_sel, wl.sink.numpy(), SM)
    for rank, idx, O, lse in got:
        assert np.array_equal(idx.reshape(-1), ref_sel)                 # every rank: the same merged selection
        assert np.allclose(O.reshape(64, 128), ref_o, rtol=1e-10, atol=1e-13)
        assert np.allclose(lse.reshape(64), ref_l, rtol=1e-12, atol=1e-12)
