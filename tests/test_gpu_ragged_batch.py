"""The ragged serving batch at full size: 64 sequences with contexts
log-uniform in [4,096, 262,144] (5.0M cached positions in all), paged caches
with 64-position pages, one query token each.  One DSA layer-step over the
whole batch (64 rows: the separate-kernel path of dsa_layer_decode) and the
SWA layer-steps over window-only paged caches, checked against the oracle:
every row's selection bit-exact against the oracle's top-k over the GPU
scores, scores and attention of sampled rows against the oracle end to end,
and every row of the SWA step."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import local_attention_decode_b200 as dsa  # noqa: E402
import oracle  # noqa: E402
from parity import (assert_attn_close, assert_scores_close, kv_for, oracle_attention_rows,  # noqa: E402
                    oracle_scores)
from test_gpu_parity import SM, run_indexer, run_layer, run_topk  # noqa: E402
from workloads import CONFIGS, make_decode_workload, make_swa_window_workload  # noqa: E402

DEV = "cuda"


@pytest.fixture(scope="module")
def batch():
    wl = make_decode_workload(device=DEV, **CONFIGS["ragged_b64"])
    yield wl
    del wl
    torch.cuda.empty_cache()


def test_ragged_b64_dsa_layer_step(batch):
    wl = batch
    lens = wl.layout.seq_lens
    O, lse, idx, cnt = run_layer(wl)
    scores = run_indexer(wl)
    idx2, cnt2 = run_topk(scores, wl.q_pos, 2048)
    assert torch.equal(cnt, cnt2) and torch.equal(idx, idx2)
    assert torch.equal(cnt[:, 0].cpu(), torch.tensor([min(L, 2048) for L in lens], dtype=torch.int32))
    for b, L in enumerate(lens):   # every row: the oracle's top-k over the same scores
        ref_idx, _ = oracle.topk(scores[b, 0, :L].cpu().numpy(), 2048)
        assert np.array_equal(idx[b, 0].cpu().numpy(), np.sort(ref_idx)), f"row {b}"
    order = np.argsort(lens)
    for b in sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2]), 7}):
        L = lens[b]
        assert_scores_close(scores[b, :, :L].cpu().numpy(), oracle_scores(wl, b))
        ref_o, ref_l = oracle_attention_rows(wl, b, 0, idx[b, 0].cpu().numpy(), wl.sink, SM)
        assert_attn_close(O[b, 0], ref_o, lse[b, 0], ref_l)
        assert set(wl.needles[b].tolist()) <= set(idx[b, 0].cpu().numpy().tolist())


def test_ragged_b64_swa_layer_step():
    lens = CONFIGS["ragged_b64"]["seq_lens"]
    wl = make_swa_window_workload(33, lens, device=DEV)
    O = torch.empty((wl.B, 1, 64, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((wl.B, 1, 64), dtype=torch.float32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_SWA_ATTN, wl.B, 1, 1, 128)
    dsa.swa_attn_decode(wl.Q, kv_for(wl, with_index=False), wl.q_pos, 128, wl.sink, SM, O, lse, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK
    for b, L in enumerate(lens):
        win = oracle.swa_indices(L - 1, 128)
        ref_o, ref_l = oracle_attention_rows(wl, b, 0, win, wl.sink, SM)
        assert_attn_close(O[b, 0], ref_o, lse[b, 0], ref_l)
