"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Sizes span several 128-key tiles with ragged tails, contiguous and paged
caches, 1 and 4 query tokens, and the 1,048,576-token context (sampled where
the oracle cannot do the whole thing).  Tolerances are in tests/parity.py.
"""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():   # collected on CPU machines, skipped there by the marker filter
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import local_attention_decode_b200 as dsa  # noqa: E402
from workloads import CONFIGS, bits16, make_decode_workload, logical_rows, ragged_batch_lengths  # noqa: E402
from parity import (kv_for, assert_scores_close, assert_attn_close, oracle_scores,  # noqa: E402
                    oracle_attention_rows, selection_agrees_outside_tie_band)

DEV = "cuda"
SM = 1.0 / math.sqrt(192)


def run_indexer(wl, Lmax=None):
    Lmax = Lmax or int(wl.q_pos.max()) + 1
    scores = torch.full((wl.B, wl.T, Lmax), float("nan"), device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_INDEXER, wl.B, wl.T, Lmax, 1)
    dsa.dsa_indexer_scores(wl.q8, wl.q_scale, wl.w, kv_for(wl, with_backbone=False), wl.q_pos, Lmax, scores, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK
    return scores


def run_topk(scores, q_pos, top_k):
    B, T, Lmax = scores.shape
    idx = torch.full((B, T, top_k), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, T), -7, dtype=torch.int32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_TOPK, B, T, Lmax, top_k)
    dsa.dsa_topk_select(scores, q_pos, Lmax, top_k, idx, cnt, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK
    # the workspace is left zeroed for the next call
    assert int(ws.count_nonzero()) == 0
    return idx, cnt


# ------------------------------------------------------------------ indexer
@pytest.mark.parametrize("case", [
    dict(seq_lens=[8192], T=1),                 # the tiny decode workload
    dict(seq_lens=[3001], T=4),                 # ragged tail, speculative block
    dict(seq_lens=[1, 127, 128, 129, 700], T=1),  # degenerate and boundary lengths
    dict(seq_lens=[5000, 300, 2000], T=2, page_size=64),   # paged, ragged
    dict(seq_lens=[1000, 4100], T=1, page_size=16),
    dict(seq_lens=[3000, 1500], T=3, page_size=256),
])
def test_indexer_matches_oracle(case):
    wl = make_decode_workload(seed=11, device=DEV, n_needles=4, **case)
    scores = run_indexer(wl).cpu().numpy()
    for b in range(wl.B):
        ref = oracle_scores(wl, b)
        assert_scores_close(scores[b, :, :ref.shape[1]], ref)


def test_indexer_t16_and_many_sequences():
    wl = make_decode_workload(seed=12, seq_lens=[700] * 3, T=16, device=DEV)
    scores = run_indexer(wl).cpu().numpy()
    for b in range(wl.B):
        ref = oracle_scores(wl, b)
        assert_scores_close(scores[b], ref)
    lens = [int(x) for x in np.random.default_rng(0).integers(1, 600, 100)]
    wl = make_decode_workload(seed=13, seq_lens=lens, T=1, device=DEV, page_size=64)
    scores = run_indexer(wl).cpu().numpy()
    for b in range(0, wl.B, 7):
        ref = oracle_scores(wl, b)
        assert_scores_close(scores[b, :, :ref.shape[1]], ref)


# -------------------------------------------------------------------- top-k
@pytest.mark.parametrize("n,k", [(1, 2048), (2047, 2048), (2048, 2048), (2049, 2048), (5000, 2048),
                                 (70000, 2048), (70000, 1), (300000, 2048), (1048576, 2048)])
def test_topk_bit_exact_against_oracle(n, k):
    g = torch.Generator(device=DEV).manual_seed(n + k)
    scores = torch.rand((1, 1, n), generator=g, device=DEV) * 10
    q_pos = torch.tensor([[n - 1]], dtype=torch.int32, device=DEV)
    idx, cnt = run_topk(scores, q_pos, k)
    ref_idx, ref_cnt = oracle.topk(scores[0, 0].cpu().numpy(), k)
    assert int(cnt) == ref_cnt
    got = idx[0, 0].cpu().numpy()
    assert np.all(got[ref_cnt:] == -1)
    assert np.all(np.diff(got[:ref_cnt]) > 0)              # increasing position order
    assert np.array_equal(got[:ref_cnt], np.sort(ref_idx[:ref_cnt]))


@pytest.mark.parametrize("kind", ["all_equal", "few_values", "signed_zero", "negative", "heavy_ties_long"])
def test_topk_ties(kind):
    n, k = (200000, 2048) if kind == "heavy_ties_long" else (9000, 2048)
    g = torch.Generator(device=DEV).manual_seed(7)
    if kind == "all_equal":
        s = torch.full((n,), 3.25, device=DEV)
    elif kind == "few_values":
        s = torch.randint(0, 5, (n,), generator=g, device=DEV).float()
    elif kind == "signed_zero":
        s = torch.where(torch.rand(n, generator=g, device=DEV) < 0.5, torch.tensor(-0.0, device=DEV),
                        torch.tensor(0.0, device=DEV))
        s[::97] = 1.0
    elif kind == "negative":
        s = -torch.rand(n, generator=g, device=DEV) - 1
    else:
        s = torch.randint(0, 3, (n,), generator=g, device=DEV).float()
    scores = s.view(1, 1, n).contiguous()
    q_pos = torch.tensor([[n - 1]], dtype=torch.int32, device=DEV)
    idx, cnt = run_topk(scores, q_pos, k)
    ref_idx, ref_cnt = oracle.topk(s.cpu().numpy(), k)
    assert int(cnt) == ref_cnt
    assert np.array_equal(idx[0, 0, :ref_cnt].cpu().numpy(), np.sort(ref_idx[:ref_cnt]))


def test_topk_many_rows_ragged():
    B, T, L = 6, 4, 40000
    g = torch.Generator(device=DEV).manual_seed(3)
    scores = torch.randn((B, T, L), generator=g, device=DEV)
    q_pos = torch.randint(0, L, (B, T), generator=g, device=DEV, dtype=torch.int32)
    q_pos[0, 0] = 0
    q_pos[1, 1] = 2047
    q_pos[2, 2] = L - 1
    idx, cnt = run_topk(scores, q_pos, 2048)
    sc = scores.cpu().numpy()
    for b in range(B):
        for t in range(T):
            n = int(q_pos[b, t]) + 1
            ref_idx, ref_cnt = oracle.topk(sc[b, t, :n], 2048)
            assert int(cnt[b, t]) == ref_cnt
            assert np.array_equal(idx[b, t, :ref_cnt].cpu().numpy(), np.sort(ref_idx[:ref_cnt]))
            assert np.all(idx[b, t, ref_cnt:].cpu().numpy() == -1)


def test_topk_rows_of_very_different_lengths():
    """More than 16 rows: the grid's CTAs go to the rows in proportion to their
    lengths (one row of 250K keys next to rows of a few thousand)."""
    B, T = 10, 4
    L = 250000
    g = torch.Generator(device=DEV).manual_seed(9)
    scores = torch.randn((B, T, L), generator=g, device=DEV)
    lens = np.exp(np.random.default_rng(9).uniform(np.log(3000), np.log(L), B * T)).astype(np.int64)
    lens[0] = L
    lens[1] = 2049
    q_pos = torch.from_numpy(lens - 1).to(torch.int32).view(B, T).to(DEV)
    for _ in range(2):   # run_topk also checks that the call leaves its workspace zeroed
        idx, cnt = run_topk(scores, q_pos, 2048)
    sc = scores.cpu().numpy()
    for b in range(B):
        for t in range(T):
            n = int(q_pos[b, t]) + 1
            ref_idx, ref_cnt = oracle.topk(sc[b, t, :n], 2048)
            assert int(cnt[b, t]) == ref_cnt
            assert np.array_equal(idx[b, t, :ref_cnt].cpu().numpy(), np.sort(ref_idx[:ref_cnt]))


# ---------------------------------------------------------------- attention
def _sparse_case(seed, seq_len, T, count_list, G=4, qk_std=None, page_size=0, sink=True):
    wl = make_decode_workload(seed=seed, seq_lens=[seq_len], T=T, G=G, device=DEV, qk_std=qk_std,
                              page_size=page_size)
    rng = np.random.default_rng(seed)
    top_k = 2048
    idx = np.full((1, T, top_k), -1, np.int32)
    cnt = np.zeros((1, T), np.int32)
    for t, c in enumerate(count_list):
        idx[0, t, :c] = rng.choice(seq_len, c, replace=False)
        cnt[0, t] = c
    idx_t = torch.from_numpy(idx).to(DEV)
    cnt_t = torch.from_numpy(cnt).to(DEV)
    O = torch.empty((1, T, 64, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((1, T, 64), dtype=torch.float32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_SPARSE_ATTN, 1, T, 1, top_k)
    sk = wl.sink if sink else None
    dsa.sparse_gqa_attn_decode(wl.Q, kv_for(wl, with_index=False), idx_t, cnt_t, top_k, sk, SM, O, lse, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK
    for t in range(T):
        ref_o, ref_l = oracle_attention_rows(wl, 0, t, idx[0, t, :cnt[0, t]], sk, SM)
        assert_attn_close(O[0, t], ref_o, lse[0, t], ref_l)


@pytest.mark.parametrize("counts", [[2048], [1], [0], [2047, 64, 65, 1000]])
def test_sparse_attention_matches_oracle(counts):
    _sparse_case(20 + len(counts), 10000, len(counts), counts)


def test_sparse_attention_peaked_and_paged():
    _sparse_case(31, 7000, 2, [2048, 333], qk_std=1.0, page_size=64)
    _sparse_case(32, 7000, 1, [2048], qk_std=1.0, sink=False)


@pytest.mark.parametrize("G", [4, 8, 16])
def test_sparse_attention_other_group_sizes(G):
    _sparse_case(40 + G, 3000, 1, [1500], G=G)


@pytest.mark.parametrize("seq_lens,T,page_size", [([8192], 1, 0), ([100], 1, 0), ([1], 1, 0),
                                                  ([300, 129, 5000], 2, 64)])
def test_swa_attention_matches_oracle(seq_lens, T, page_size):
    wl = make_decode_workload(seed=50, seq_lens=seq_lens, T=T, G=8, device=DEV, page_size=page_size)
    O = torch.empty((wl.B, T, 64, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((wl.B, T, 64), dtype=torch.float32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_SWA_ATTN, wl.B, T, 1, 128)
    dsa.swa_attn_decode(wl.Q, kv_for(wl, with_index=False), wl.q_pos, 128, wl.sink, SM, O, lse, ws)
    for b in range(wl.B):
        for t in range(T):
            p = int(wl.q_pos[b, t])
            win = oracle.swa_indices(p, 128)
            ref_o, ref_l = oracle_attention_rows(wl, b, t, win, wl.sink, SM)
            assert_attn_close(O[b, t], ref_o, lse[b, t], ref_l)


# -------------------------------------------------------- fused layer-step
def run_layer(wl, top_k=2048, sink=True, events=None):
    Lmax = int(wl.q_pos.max()) + 1
    O = torch.empty((wl.B, wl.T, 64, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((wl.B, wl.T, 64), dtype=torch.float32, device=DEV)
    idx = torch.empty((wl.B, wl.T, top_k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((wl.B, wl.T), dtype=torch.int32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_LAYER, wl.B, wl.T, Lmax, top_k)
    dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv_for(wl), wl.q_pos, Lmax, top_k,
                         wl.sink if sink else None, SM, O, lse, idx, cnt, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK
    LAST_PATHS[:] = dsa.dsa_layer_path_counts(ws)
    return O, lse, idx, cnt


# (fast, general) path counts of the one-barrier kernel in the last run_layer call
LAST_PATHS = [0, 0]


def _check_layer(wl, O, lse, idx, cnt, top_k=2048, full_oracle=True, sink=True):
    sk = wl.sink if sink else None
    for b in range(wl.B):
        ref_scores = oracle_scores(wl, b) if full_oracle else None
        for t in range(wl.T):
            n = int(wl.q_pos[b, t]) + 1
            c = int(cnt[b, t])
            assert c == min(n, top_k)
            sel = idx[b, t, :c].cpu().numpy()
            assert np.all(idx[b, t, c:].cpu().numpy() == -1)
            if ref_scores is not None:
                assert selection_agrees_outside_tie_band(sel, ref_scores[t, :n].astype(np.float64), top_k)
            ref_o, ref_l = oracle_attention_rows(wl, b, t, sel, sk, SM)
            assert_attn_close(O[b, t], ref_o, lse[b, t], ref_l)


@pytest.mark.parametrize("name", ["tiny_8k", "verify_64k_t4"])
def test_layer_decode_matches_oracle(name):
    wl = make_decode_workload(device=DEV, **CONFIGS[name])
    O, lse, idx, cnt = run_layer(wl)
    # up to four long rows: the one-barrier kernel, and its sample was good
    assert LAST_PATHS == [1, 0]
    _check_layer(wl, O, lse, idx, cnt)
    # planted needles rank in the oracle's top-2048 and are selected
    sel = set(idx[0, 0].cpu().numpy().tolist())
    assert set(wl.needles[0].tolist()) <= sel


def test_layer_decode_short_contexts_and_pages():
    wl = make_decode_workload(seed=60, seq_lens=[2, 900, 2048, 2049, 4000], T=2, device=DEV, page_size=64,
                              n_needles=2)
    O, lse, idx, cnt = run_layer(wl)
    _check_layer(wl, O, lse, idx, cnt)


def test_layer_decode_is_deterministic():
    wl = make_decode_workload(device=DEV, **CONFIGS["verify_64k_t4"])
    a = run_layer(wl)
    b = run_layer(wl)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.uint8) if y.dtype == torch.bfloat16 else y)


@pytest.mark.parametrize("seq_lens,T,page_size", [([65536], 4, 0), ([3000, 9000], 2, 64), ([20000] * 5, 4, 0),
                                                   ([40000], 3, 0), ([12000, 30000, 9000, 20000], 1, 64)])
def test_layer_decode_equals_separate_calls(seq_lens, T, page_size):
    """dsa_layer_decode (the one-barrier kernel for up to four long rows, one
    fused launch for B*T <= 16 rows, separate kernels above) gives exactly
    what the three separate entry points give: three and four query rows of
    one sequence, and four sequences of one row each, take the one-barrier
    kernel."""
    wl = make_decode_workload(seed=80, seq_lens=seq_lens, T=T, device=DEV, page_size=page_size, n_needles=8)
    O, lse, idx, cnt = run_layer(wl)
    assert sum(LAST_PATHS) == (1 if wl.B * T <= 4 else 0)   # the one-barrier kernel ran once, or not at all
    Lmax = int(wl.q_pos.max()) + 1
    scores = run_indexer(wl, Lmax)
    idx2, cnt2 = run_topk(scores, wl.q_pos, 2048)
    assert torch.equal(cnt, cnt2) and torch.equal(idx, idx2)
    O2 = torch.empty_like(O)
    lse2 = torch.empty_like(lse)
    ws = dsa.alloc_workspace(dsa.OP_SPARSE_ATTN, wl.B, wl.T, 1, 2048)
    dsa.sparse_gqa_attn_decode(wl.Q, kv_for(wl, with_index=False), idx2, cnt2, 2048, wl.sink, SM, O2, lse2, ws)
    assert torch.equal(O.view(torch.int16), O2.view(torch.int16))
    assert torch.equal(lse, lse2)


# ------------------------------------------ layer-step options not in the configs
# Cases for the fused path (B * T <= 16 rows, one cooperative launch) and for
# the separate kernels (B * T > 16 rows).
_LAYER_CASES = {
    "fused": dict(seq_lens=[20000], T=2, page_size=0),
    "separate": dict(seq_lens=[3000, 9000, 20000, 40000, 2500], T=4, page_size=64),
}


@pytest.mark.parametrize("path", ["fused", "separate"])
def test_layer_decode_without_sink(path):
    """sink = NULL, the DSA layers' configuration in the shipped weights
    ([EXPL] "Inside a DSA layer": no attention sink on the DSA layers)."""
    wl = make_decode_workload(seed=90, device=DEV, n_needles=4, **_LAYER_CASES[path])
    O, lse, idx, cnt = run_layer(wl, sink=False)
    _check_layer(wl, O, lse, idx, cnt, sink=False)


@pytest.mark.parametrize("top_k", [1, 100, 2047])
@pytest.mark.parametrize("path", ["fused", "separate"])
def test_layer_decode_other_top_k(path, top_k):
    """top_k below the model's 2,048 through the whole layer-step: the
    selection is bit-exact against the oracle's top-k over the same scores,
    and the attention matches the oracle over it."""
    wl = make_decode_workload(seed=91 + top_k, device=DEV, n_needles=4, **_LAYER_CASES[path])
    O, lse, idx, cnt = run_layer(wl, top_k=top_k)
    scores = run_indexer(wl)
    for b in range(wl.B):
        for t in range(wl.T):
            n = int(wl.q_pos[b, t]) + 1
            ref_idx, ref_cnt = oracle.topk(scores[b, t, :n].cpu().numpy(), top_k)
            assert int(cnt[b, t]) == ref_cnt
            assert np.array_equal(idx[b, t, :ref_cnt].cpu().numpy(), np.sort(ref_idx[:ref_cnt]))
    _check_layer(wl, O, lse, idx, cnt, top_k=top_k)


def test_batched_contiguous_index_cache_needs_aligned_stride():
    """A contiguous cache shared by B > 1 sequences whose seq_stride is not a
    multiple of 16 is rejected on the host, before anything is enqueued."""
    wl = make_decode_workload(seed=92, seq_lens=[1000, 1000], T=1, device=DEV)
    lay = wl.layout
    rows = lay.num_rows
    kv = dsa.KV(k=wl.K, v=wl.V, index_k=wl.k8, index_k_scale=wl.k_scale, num_kv_heads=wl.G,
                seq_stride=1001, num_rows=rows)
    O = torch.empty((2, 1, 64, 128), dtype=torch.bfloat16, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_LAYER, 2, 1, 1000, 2048)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, 1000, 2048, wl.sink, SM, O, ws=ws)
    assert e.value.code == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    scores = torch.empty((2, 1, 1000), device=DEV)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_indexer_scores(wl.q8, wl.q_scale, wl.w, kv, wl.q_pos, 1000, scores,
                               dsa.alloc_workspace(dsa.OP_INDEXER, 2, 1, 1000, 1))
    assert e.value.code == dsa.DSA_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("weights", ["negative", "mixed", "zero_query"])
def test_layer_decode_selection_fallbacks(weights):
    """Rows the fused kernel's one-barrier selection does not take (threshold
    among negative scores; one histogram bin holding every score) go through
    the general selection and still equal the separate calls and the oracle."""
    wl = make_decode_workload(seed=81, seq_lens=[30000], T=2, device=DEV, n_needles=4)
    g = torch.Generator(device=DEV).manual_seed(5)
    if weights == "negative":
        wl.w = -torch.rand(wl.w.shape, generator=g, device=DEV) / 16
    elif weights == "mixed":
        wl.w = (torch.rand(wl.w.shape, generator=g, device=DEV) - 0.5) / 8
    else:   # every score 0: all tied, the lowest positions win
        wl.q8 = torch.zeros_like(wl.q8)
    O, lse, idx, cnt = run_layer(wl)
    scores = run_indexer(wl)
    idx2, cnt2 = run_topk(scores, wl.q_pos, 2048)
    assert torch.equal(cnt, cnt2) and torch.equal(idx, idx2)
    for t in range(wl.T):
        ref_idx, _ = oracle.topk(scores[0, t, :int(wl.q_pos[0, t]) + 1].cpu().numpy(), 2048)
        assert np.array_equal(idx[0, t].cpu().numpy(), np.sort(ref_idx))
    if weights == "zero_query":
        assert np.array_equal(idx[0, 0].cpu().numpy(), np.arange(2048))
    if weights != "mixed":
        # every key at or above the sampled threshold (all negative, or all
        # tied): too many candidates, so the one-barrier kernel's general path
        assert LAST_PATHS == [0, 1]
    _check_layer(wl, O, lse, idx, cnt)


def test_layer_decode_1m_context_sampled():
    """Native 1,048,576-token context: scores at sampled positions and every
    needle against the oracle; the selection bit-exact against the oracle's
    top-k over the GPU scores; attention against the oracle over the selection."""
    wl = make_decode_workload(device=DEV, **CONFIGS["ctx_1m"])
    L = wl.layout.seq_lens[0]
    scores = run_indexer(wl)
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([rng.choice(L, 8192, replace=False), wl.needles[0].numpy(),
                                       np.arange(L - 300, L)]))
    rows = torch.from_numpy(sample).to(DEV)
    ref = oracle.indexer_scores(wl.q8[0].cpu().numpy(), wl.q_scale[0].cpu().numpy(), wl.w[0].cpu().numpy(),
                                wl.k8[rows].cpu().numpy(), wl.k_scale[rows].cpu().numpy(),
                                np.array([len(sample) - 1], np.int32))
    assert_scores_close(scores[0][:, rows].cpu().numpy(), ref)
    O, lse, idx, cnt = run_layer(wl)
    assert LAST_PATHS == [1, 0]   # the one-barrier kernel's fast path at 1M
    gpu_scores = scores[0, 0].cpu().numpy()
    ref_idx, ref_cnt = oracle.topk(gpu_scores, 2048)
    assert int(cnt[0, 0]) == 2048
    assert np.array_equal(idx[0, 0].cpu().numpy(), np.sort(ref_idx))
    ref_o, ref_l = oracle_attention_rows(wl, 0, 0, idx[0, 0].cpu().numpy(), wl.sink, SM)
    assert_attn_close(O[0, 0], ref_o, lse[0, 0], ref_l)


def test_bad_positions_are_flagged_not_faulted():
    wl = make_decode_workload(seed=70, seq_lens=[1000], T=1, device=DEV)
    idx = torch.full((1, 1, 2048), -1, dtype=torch.int32, device=DEV)
    idx[0, 0, :3] = torch.tensor([5, 999999, -3], dtype=torch.int32)
    cnt = torch.tensor([[3]], dtype=torch.int32, device=DEV)
    O = torch.empty((1, 1, 64, 128), dtype=torch.bfloat16, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_SPARSE_ATTN, 1, 1, 1, 2048)
    dsa.sparse_gqa_attn_decode(wl.Q, kv_for(wl, with_index=False), idx, cnt, 2048, wl.sink, SM, O, None, ws)
    st, flags = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_ERR_DEVICE_BAD_INDEX and flags == (1 << dsa.DSA_ERR_DEVICE_BAD_INDEX)
    ref_o, _ = oracle_attention_rows(wl, 0, 0, np.array([5]), wl.sink, SM)   # bad entries are skipped
    assert_attn_close(O[0, 0], ref_o)
    assert dsa.dsa_check_device_status(ws)[0] == dsa.DSA_OK   # reading clears the word


def test_layer_decode_many_tied_top_keys():
    """3,000 keys share the row's highest score (copies of its best key, at
    twice its scale): the bin of the k-th largest key in the one-barrier
    kernel's candidate histogram holds all of them, so its general search runs;
    the selection is the 2,048 lowest positions of the tied keys, as the
    oracle's top-k (ties to the lower position)."""
    wl = make_decode_workload(seed=95, seq_lens=[20000], T=1, device=DEV, n_needles=0)
    scores = run_indexer(wl)
    best = int(torch.argmax(scores[0, 0]))
    assert float(scores[0, 0, best]) > 0
    g = torch.Generator().manual_seed(6)
    tied = torch.randperm(20000, generator=g)[:3000].sort().values.to(DEV)
    key, scale = wl.k8[best].clone(), wl.k_scale[best].clone() * 2
    wl.k8[tied] = key
    wl.k_scale[tied] = scale
    O, lse, idx, cnt = run_layer(wl)
    assert LAST_PATHS == [1, 0]   # the fast path: the general search is inside it
    scores = run_indexer(wl)
    ref_idx, ref_cnt = oracle.topk(scores[0, 0].cpu().numpy(), 2048)
    assert int(cnt[0, 0]) == ref_cnt == 2048
    got = idx[0, 0].cpu().numpy()
    assert np.array_equal(got, np.sort(ref_idx))
    assert np.array_equal(got, np.sort(tied.cpu().numpy())[:2048])
    ref_o, ref_l = oracle_attention_rows(wl, 0, 0, got, wl.sink, SM)
    assert_attn_close(O[0, 0], ref_o, lse[0, 0], ref_l)
