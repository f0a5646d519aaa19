"""The context-sharded decode kernels on one GPU: N ranks emulated in one
process (each rank's slice a view of one cache; the all-gathers are
concatenations).  The merged selection equals the one-GPU layer-step's
selection bit for bit; the combined output matches the oracle over it."""
import math

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import local_attention_decode_b200 as dsa  # noqa: E402
from local_attention_decode_b200.sharded import LibOps, Shard  # noqa: E402
from workloads import make_decode_workload  # noqa: E402
from parity import kv_for, oracle_attention_rows, assert_attn_close  # noqa: E402

DEV = "cuda"
SM = 1.0 / math.sqrt(192)


@pytest.mark.parametrize("N,L,top_k", [(2, 60000, 2048), (4, 131072, 2048), (3, 9000, 100)])
def test_sharded_layer_step_equals_one_gpu(N, L, top_k):
    wl = make_decode_workload(seed=150 + N, seq_lens=[L], T=1, device=DEV, n_needles=16, needle_mode="zipf")
    # the one-GPU layer-step
    O1 = torch.empty((1, 1, 64, 128), dtype=torch.bfloat16, device=DEV)
    idx1 = torch.empty((1, 1, top_k), dtype=torch.int32, device=DEV)
    cnt1 = torch.empty((1, 1), dtype=torch.int32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_LAYER, 1, 1, L, top_k)
    dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv_for(wl), wl.q_pos, L, top_k, wl.sink, SM, O1, None, idx1,
                         cnt1, ws)
    # N ranks, contiguous slices (offsets multiples of 128)
    step = (L // N + 127) // 128 * 128
    shards = [Shard(offset=r * step, length=min(step, L - r * step), Lmax_local=min(step, L - r * step))
              for r in range(N)]
    ops = LibOps()
    kvs = []
    for sh in shards:
        sl = slice(sh.offset, sh.offset + sh.length)
        kvs.append(dsa.KV(k=wl.K[sl], v=wl.V[sl], index_k=wl.k8[sl], index_k_scale=wl.k_scale[sl], num_kv_heads=4,
                          seq_stride=sh.length, num_rows=sh.length))
    cands = [ops.local_select(wl.q8, wl.q_scale, wl.w, kv, wl.q_pos, sh, top_k) for kv, sh in zip(kvs, shards)]
    cs_all = torch.stack([c[0] for c in cands])
    cp_all = torch.stack([c[1] for c in cands])
    outs, merged = [], []
    for kv, sh in zip(kvs, shards):
        idx, cnt, lidx, lcnt = ops.merge(cs_all, cp_all, top_k, sh)
        merged.append((idx, cnt))
        outs.append(ops.local_attention(wl.Q, kv, lidx, lcnt, top_k, SM))
    for idx, cnt in merged:   # every rank has the same selection, the one-GPU one
        assert torch.equal(cnt, cnt1) and torch.equal(idx, idx1)
    O = torch.empty_like(O1)
    lse = torch.empty((1, 1, 64), dtype=torch.float32, device=DEV)
    ops.combine(torch.stack([o for o, _ in outs]), torch.stack([l for _, l in outs]), wl.sink, O, lse)
    c = int(cnt1[0, 0])
    ref_o, ref_l = oracle_attention_rows(wl, 0, 0, idx1[0, 0, :c].cpu().numpy(), wl.sink, SM)
    assert_attn_close(O[0, 0], ref_o, lse[0, 0], ref_l)
