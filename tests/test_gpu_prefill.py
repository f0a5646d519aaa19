"""dsa_prefill: the DSA layer for a block of query tokens of one sequence,
each token attending causally (its visible keys are 0..its position).  It
must compute, token by token, what the decode layer-step computes."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import local_attention_decode_b200 as dsa  # noqa: E402
import oracle  # noqa: E402
from parity import assert_attn_close, kv_for, oracle_attention_rows  # noqa: E402
from test_gpu_parity import SM, _check_layer  # noqa: E402
from workloads import CONFIGS, make_decode_workload  # noqa: E402

DEV = "cuda"


def run_prefill(wl, top_k=2048):
    NQ = wl.T
    Lmax = int(wl.q_pos.max()) + 1
    O = torch.empty((NQ, 64, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((NQ, 64), dtype=torch.float32, device=DEV)
    idx = torch.empty((NQ, top_k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((NQ,), dtype=torch.int32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_PREFILL, 1, NQ, Lmax, top_k)
    dsa.dsa_prefill(wl.q8[0], wl.q_scale[0], wl.w[0], wl.Q[0], kv_for(wl), wl.q_pos[0], Lmax, top_k, wl.sink, SM,
                    O, lse, idx, cnt, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK
    return O, lse, idx, cnt


@pytest.mark.parametrize("L,NQ,page_size", [(8192, 40, 0), (5000, 16, 64), (3000, 3, 0)])
def test_prefill_matches_oracle_token_by_token(L, NQ, page_size):
    wl = make_decode_workload(seed=90 + NQ, seq_lens=[L], T=NQ, device=DEV, page_size=page_size, n_needles=8)
    O, lse, idx, cnt = run_prefill(wl)
    _check_layer(wl, O[None], lse[None], idx[None], cnt[None])


def test_prefill_equals_decode_blocks():
    wl = make_decode_workload(seed=95, seq_lens=[20000], T=37, device=DEV, n_needles=4)
    O, lse, idx, cnt = run_prefill(wl)
    Lmax = 20000
    for t0 in range(0, 37, 16):
        T = min(16, 37 - t0)
        O2 = torch.empty((1, T, 64, 128), dtype=torch.bfloat16, device=DEV)
        lse2 = torch.empty((1, T, 64), dtype=torch.float32, device=DEV)
        idx2 = torch.empty((1, T, 2048), dtype=torch.int32, device=DEV)
        cnt2 = torch.empty((1, T), dtype=torch.int32, device=DEV)
        ws = dsa.alloc_workspace(dsa.OP_LAYER, 1, T, Lmax, 2048)
        sl = slice(t0, t0 + T)
        dsa.dsa_layer_decode(wl.q8[:, sl].contiguous(), wl.q_scale[:, sl].contiguous(), wl.w[:, sl].contiguous(),
                             wl.Q[:, sl].contiguous(), kv_for(wl), wl.q_pos[:, sl].contiguous(), Lmax, 2048, wl.sink,
                             SM, O2, lse2, idx2, cnt2, ws)
        assert torch.equal(idx[sl], idx2[0]) and torch.equal(cnt[sl], cnt2[0])
        assert torch.equal(O[sl].view(torch.int16), O2[0].view(torch.int16))
        assert torch.equal(lse[sl], lse2[0])


def test_prefill_8k_queries_at_1m_context_sampled():
    """The chunked-prefill workload at full size: 8,192 query tokens at
    1,040,384..1,048,575 over a 1,048,576-token cache.  Sampled tokens: the
    selection bit-exact against the oracle's top-k over that token's GPU
    scores, and the attention against the oracle over the selection."""
    wl = make_decode_workload(device=DEV, **CONFIGS["prefill_8k_1m"])
    O, lse, idx, cnt = run_prefill(wl)
    L = wl.layout.seq_lens[0]
    assert torch.equal(cnt, torch.full_like(cnt, 2048))
    for t in (0, 4095, 8191):
        scores = torch.empty((1, 1, L), dtype=torch.float32, device=DEV)
        ws = dsa.alloc_workspace(dsa.OP_INDEXER, 1, 1, L, 1)
        kv = kv_for(wl, with_backbone=False)
        dsa.dsa_indexer_scores(wl.q8[:, t:t + 1].contiguous(), wl.q_scale[:, t:t + 1].contiguous(),
                               wl.w[:, t:t + 1].contiguous(), kv, wl.q_pos[:, t:t + 1].contiguous(), L, scores, ws)
        p = int(wl.q_pos[0, t])
        gs = scores[0, 0, :p + 1].cpu().numpy()
        ref_idx, _ = oracle.topk(gs, 2048)
        assert np.array_equal(idx[t].cpu().numpy(), np.sort(ref_idx)), f"token {t}"
        ref_o, ref_l = oracle_attention_rows(wl, 0, t, idx[t].cpu().numpy(), wl.sink, SM)
        assert_attn_close(O[t], ref_o, lse[t], ref_l)


def _decode_blocks(wl, Lmax, top_k=2048):
    """The same tokens through dsa_layer_decode, 16 at a time."""
    NQ = wl.T
    O = torch.empty((NQ, 64, 128), dtype=torch.bfloat16, device=DEV)
    idx = torch.empty((NQ, top_k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((NQ,), dtype=torch.int32, device=DEV)
    for t0 in range(0, NQ, 16):
        T = min(16, NQ - t0)
        sl = slice(t0, t0 + T)
        ws = dsa.alloc_workspace(dsa.OP_LAYER, 1, T, Lmax, top_k)
        O2 = torch.empty((1, T, 64, 128), dtype=torch.bfloat16, device=DEV)
        idx2 = torch.empty((1, T, top_k), dtype=torch.int32, device=DEV)
        cnt2 = torch.empty((1, T), dtype=torch.int32, device=DEV)
        dsa.dsa_layer_decode(wl.q8[:, sl].contiguous(), wl.q_scale[:, sl].contiguous(), wl.w[:, sl].contiguous(),
                             wl.Q[:, sl].contiguous(), kv_for(wl), wl.q_pos[:, sl].contiguous(), Lmax, top_k,
                             wl.sink, SM, O2, None, idx2, cnt2, ws)
        O[sl], idx[sl], cnt[sl] = O2[0], idx2[0], cnt2[0]
    return O, idx, cnt


@pytest.mark.parametrize("L,NQ,page_size", [(100000, 64, 0), (70000, 96, 64), (40000, 80, 128)])
def test_tensor_core_prefill_equals_decode_blocks(L, NQ, page_size):
    """NQ a multiple of 16 (>= 64): the indexer runs as one contraction with the
    candidate filter; every token's selection and output equal the decode
    layer-step's bit for bit."""
    wl = make_decode_workload(seed=170 + NQ, seq_lens=[L], T=NQ, device=DEV, page_size=page_size, n_needles=16,
                              needle_mode="zipf")
    O, lse, idx, cnt = run_prefill(wl)
    O2, idx2, cnt2 = _decode_blocks(wl, L)
    assert torch.equal(cnt, cnt2) and torch.equal(idx, idx2)
    assert torch.equal(O.view(torch.int16), O2.view(torch.int16))
    for t in (0, NQ // 2, NQ - 1):   # and the attention against the oracle over the selection
        c = int(cnt[t])
        ref_o, ref_l = oracle_attention_rows(wl, 0, t, idx[t, :c].cpu().numpy(), wl.sink, SM)
        assert_attn_close(O[t], ref_o, lse[t], ref_l)


def test_tensor_core_prefill_hands_tied_tokens_to_the_decode_path():
    """Every score tied (zero index queries): the candidate lists overflow, every
    token takes the decode layer-step, and the result is still exact."""
    wl = make_decode_workload(seed=180, seq_lens=[30000], T=64, device=DEV, n_needles=2)
    wl.q8 = torch.zeros_like(wl.q8)
    O, lse, idx, cnt = run_prefill(wl)
    O2, idx2, cnt2 = _decode_blocks(wl, 30000)
    assert torch.equal(cnt, cnt2) and torch.equal(idx, idx2)
    assert torch.equal(idx[0].cpu(), torch.arange(2048, dtype=torch.int32))
    assert torch.equal(O.view(torch.int16), O2.view(torch.int16))
