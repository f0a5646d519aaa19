"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources: "Naive-N0.5-Flash: no full-attention layers, and a runtime built by
AI" (explainer) -- property table; "What 'no full-attention layers' means";
"Inside a DSA layer: the lightning indexer"; "How much of this did AI
actually build?".
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from workloads import bits16, make_decode_workload, quantize_e4m3_rows
from conftest import load_golden


def _codes(tokens):
    return np.array([int(x, 16) for x in tokens], dtype=np.uint8)


def _floats(tokens):
    return np.array([float(x) for x in tokens], dtype=np.float32)


# ----------------------------------------------------------------- formats
def test_e4m3_matches_torch_for_every_code():
    mine = oracle.e4m3_to_float64(np.arange(256))
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    # the format definition's landmarks
    assert mine[0x7E] == 448.0 and mine[0xFE] == -448.0
    assert mine[0x38] == 1.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6
    assert nan[0x7F] and nan[0xFF] and nan.sum() == 2


def test_bf16_matches_torch():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(4096, generator=g) * torch.exp(torch.randn(4096, generator=g) * 8)
    b = x.to(torch.bfloat16)
    assert np.array_equal(oracle.bf16_to_float64(bits16(b)), b.to(torch.float64).numpy())


# ----------------------------------------------------------------- indexer
def test_fp8_dot_is_exact():
    """The double-precision e4m3 dot equals the rational-arithmetic sum."""
    rng = np.random.default_rng(0)
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = np.flatnonzero(np.isfinite(table)).astype(np.uint8)
    for trial in range(200):
        a = rng.choice(finite, 128)
        b = rng.choice(finite, 128)
        if trial % 4 == 0:    # extreme magnitudes: the largest and smallest codes
            a[:64] = rng.choice([0x7E, 0xFE, 0x01, 0x81], 64)
            b[:64] = rng.choice([0x7E, 0xFE, 0x01, 0x81], 64)
        exact = sum(Fraction(float(table[x])) * Fraction(float(table[y])) for x, y in zip(a, b))
        assert Fraction(oracle.fp8_dot(a, b)) == exact


def test_indexer_hand_worked_example():
    g = load_golden("indexer_worked_example.txt")
    q8 = np.stack([np.stack([_codes(g[f"q8_t{t}_h{h}"]) for h in range(2)]) for t in range(2)])
    q_scale = np.stack([_floats(g[f"q_scale_t{t}"]) for t in range(2)])
    w = np.stack([_floats(g[f"w_t{t}"]) for t in range(2)])
    k8 = np.stack([_codes(g[f"k8_s{s}"]) for s in range(3)])
    k_scale = _floats(g["k_scale"])
    q_pos = np.array([int(x) for x in g["q_pos"]], dtype=np.int32)
    got = oracle.indexer_scores(q8, q_scale, w, k8, k_scale, q_pos)
    for t in range(2):
        assert np.array_equal(got[t], _floats(g[f"scores_t{t}"]))
        n = q_pos[t] + 1
        idx, cnt = oracle.topk(got[t, :n], 2)
        assert cnt == 2 and list(idx) == [int(x) for x in g[f"top2_t{t}"]]


def _rand_indexer(rng, T, L, nonneg=False):
    q = torch.from_numpy(rng.standard_normal((T, 16, 128)).astype(np.float32))
    k = torch.from_numpy(rng.standard_normal((L, 128)).astype(np.float32))
    if nonneg:
        q, k = q.abs(), k.abs()
    q8, qs = quantize_e4m3_rows(q.reshape(T, 16 * 128))
    q8 = q8.reshape(T, 16, 128).numpy()
    q_scale = np.repeat(qs.numpy()[:, None], 16, axis=1)
    k8, ks = quantize_e4m3_rows(k)
    w = (rng.random((T, 16)) / 16).astype(np.float32)
    return q8, q_scale, w, k8.numpy(), ks.numpy()


def _deq(codes):
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_indexer_relu_free_case_is_a_matvec():
    """With non-negative operands the ReLU is the identity, and with w = 1 the
    score collapses to k_scale[s] * (sum_h q_scale_h q_h) . k_s: a plain
    matrix-vector product (numpy, float64)."""
    rng = np.random.default_rng(1)
    T, L = 2, 300
    q8, q_scale, _, k8, ks = _rand_indexer(rng, T, L, nonneg=True)
    w = np.ones((T, 16), dtype=np.float32)
    q_pos = np.array([L - 1, L - 1], dtype=np.int32)
    got = oracle.indexer_scores(q8, q_scale, w, k8, ks, q_pos)
    qsum = np.einsum("th,thd->td", q_scale.astype(np.float64), _deq(q8))
    ref = (_deq(k8) @ qsum.T).T * ks.astype(np.float64)[None, :]
    np.testing.assert_allclose(got, ref.astype(np.float32), rtol=2e-7, atol=0)


def test_indexer_relu_drops_negative_heads():
    """A head whose dot product is negative contributes nothing; flipping the
    sign of that head's query leaves its term at exactly the flipped value."""
    rng = np.random.default_rng(2)
    q8, q_scale, w, k8, ks = _rand_indexer(rng, 1, 64)
    q_pos = np.array([63], dtype=np.int32)
    base = oracle.indexer_scores(q8, q_scale, w, k8, ks, q_pos)[0].astype(np.float64)
    # per-head terms from the exact dots
    terms = np.zeros((16, 64))
    for h in range(16):
        for s in range(64):
            d = oracle.fp8_dot(q8[0, h], k8[s])
            terms[h, s] = w[0, h] * max(0.0, q_scale[0, h] * ks[s] * d)
    np.testing.assert_allclose(base, terms.sum(0), rtol=1e-6)
    flipped = q8.copy()
    flipped[0, 3] ^= 0x80          # negate head 3 (sign bit of every code)
    got = oracle.indexer_scores(flipped, q_scale, w, k8, ks, q_pos)[0].astype(np.float64)
    neg = np.zeros(64)
    for s in range(64):
        d = -oracle.fp8_dot(q8[0, 3], k8[s])
        neg[s] = w[0, 3] * max(0.0, q_scale[0, 3] * ks[s] * d)
    np.testing.assert_allclose(got, terms.sum(0) - terms[3] + neg, rtol=1e-6)
    assert np.any(terms[3] == 0) and np.any(neg == 0)


def test_indexer_power_of_two_scale_folding_is_exact():
    rng = np.random.default_rng(3)
    q8, q_scale, w, k8, ks = _rand_indexer(rng, 2, 200)
    q_pos = np.array([199, 150], dtype=np.int32)
    base = oracle.indexer_scores(q8, q_scale, w, k8, ks, q_pos)
    twice = oracle.indexer_scores(q8, q_scale * 2, w, k8, ks, q_pos)
    assert np.array_equal(twice, base * 2)
    ks4 = ks.copy()
    ks4[17] *= 4
    four = oracle.indexer_scores(q8, q_scale, w, k8, ks4, q_pos)
    assert four[0, 17] == base[0, 17] * 4 and np.array_equal(np.delete(four, 17, 1), np.delete(base, 17, 1))


def test_indexer_causal_mask_and_key_permutation():
    rng = np.random.default_rng(4)
    q8, q_scale, w, k8, ks = _rand_indexer(rng, 2, 100)
    q_pos = np.array([99, 40], dtype=np.int32)
    s = oracle.indexer_scores(q8, q_scale, w, k8, ks, q_pos)
    assert np.all(np.isneginf(s[1, 41:])) and np.all(np.isfinite(s[1, :41]))
    perm = rng.permutation(100)
    sp = oracle.indexer_scores(q8, q_scale, w, k8[perm], ks[perm], np.array([99, 99], np.int32))
    assert np.array_equal(sp[0], s[0, perm])


def test_indexer_linear_in_head_weights():
    rng = np.random.default_rng(6)
    q8, q_scale, w, k8, ks = _rand_indexer(rng, 1, 128)
    w2 = (rng.random((1, 16)) / 16).astype(np.float32)
    q_pos = np.array([127], np.int32)
    a = oracle.indexer_scores(q8, q_scale, w, k8, ks, q_pos).astype(np.float64)
    b = oracle.indexer_scores(q8, q_scale, w2, k8, ks, q_pos).astype(np.float64)
    c = oracle.indexer_scores(q8, q_scale, (w + w2).astype(np.float32), k8, ks, q_pos).astype(np.float64)
    np.testing.assert_allclose(c, a + b, rtol=1e-6)


# ------------------------------------------------------------------- top-k
@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_sorted_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    for n in range(0, 70):
        vals = rng.choice(np.array([-1.5, -0.0, 0.0, 0.25, 1.0, 2.0, 7.0], np.float32), n)
        for k in (1, 3, 8, 64):
            idx, cnt = oracle.topk(vals, k)
            ref = sorted(range(n), key=lambda i: (-float(vals[i]), i))[:k]
            assert cnt == len(ref) and list(idx[:cnt]) == ref
            assert np.all(idx[cnt:] == -1)


def test_topk_two_implementations_agree_on_large_rows():
    rng = np.random.default_rng(7)
    for n, k in [(5000, 2048), (70000, 2048), (2048, 2048), (2047, 2048), (100000, 10)]:
        vals = rng.standard_normal(n).astype(np.float32)
        vals[rng.integers(0, n, n // 10)] = vals[0]          # force ties
        a, ca = oracle.topk(vals, k)
        b, cb = oracle.topk_select(vals, k)
        assert ca == cb == min(n, k)
        assert np.array_equal(np.sort(a[:ca]), b[:cb])


def test_topk_all_equal_takes_lowest_positions():
    idx, cnt = oracle.topk(np.full(5000, 3.5, np.float32), 2048)
    assert cnt == 2048 and np.array_equal(idx, np.arange(2048))
    idx, cnt = oracle.topk(np.zeros(10, np.float32), 2048)
    assert cnt == 10 and np.array_equal(idx[:10], np.arange(10)) and np.all(idx[10:] == -1)


def test_topk_signed_zero_ties():
    vals = np.array([-0.0, 0.0, -0.0, 0.0], np.float32)
    idx, cnt = oracle.topk(vals, 2)
    assert list(idx) == [0, 1]


def test_needles_are_selected_in_tiny_workload():
    wl = make_decode_workload(seed=0, seq_lens=[8192], T=1, n_needles=16)
    s = oracle.indexer_scores(wl.q8[0].numpy(), wl.q_scale[0].numpy(), wl.w[0].numpy(),
                              wl.k8.numpy(), wl.k_scale.numpy(), wl.q_pos[0].numpy())
    idx, cnt = oracle.topk(s[0], 2048)
    assert cnt == 2048
    assert set(wl.needles[0].tolist()) <= set(idx.tolist())


# --------------------------------------------------------------- attention
def _bf(rng, shape, std=1.0):
    return torch.from_numpy((rng.standard_normal(shape) * std).astype(np.float32)).to(torch.bfloat16)


def _sdpa(Qb, Kb, Vb, idx, scale):
    """Textbook softmax attention via torch's SDPA in float64; GQA by head repeat."""
    H, G = Qb.shape[0], Kb.shape[1]
    q = Qb.double()[:, None, :]                                  # [H,1,D]
    k = Kb[idx].double().permute(1, 0, 2).repeat_interleave(H // G, 0)   # [H,n,D]
    v = Vb[idx].double().permute(1, 0, 2).repeat_interleave(H // G, 0)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)[:, 0].numpy()


@pytest.mark.parametrize("G", [4, 8])
def test_attention_without_sink_is_textbook_softmax(G):
    rng = np.random.default_rng(10 + G)
    L, H = 500, 64
    Qb, Kb, Vb = _bf(rng, (H, 192)), _bf(rng, (L, G, 192)), _bf(rng, (L, G, 128))
    idx = rng.choice(L, 300, replace=False).astype(np.int32)
    scale = 1 / math.sqrt(192)
    out, lse = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), idx, None, scale)
    np.testing.assert_allclose(out, _sdpa(Qb, Kb, Vb, idx, scale), rtol=1e-10, atol=1e-12)
    logits = torch.einsum("hd,nhd->hn", Qb.double(),
                          Kb[idx].double().repeat_interleave(H // G, 1)) * scale
    np.testing.assert_allclose(lse, torch.logsumexp(logits, 1).numpy(), rtol=1e-12)


def test_attention_sink_identity():
    """With a sink the output is the sink-free output times
    sum e^s / (sum e^s + e^sink), and the lse is logaddexp(lse0, sink)."""
    rng = np.random.default_rng(20)
    L, H, G = 300, 64, 4
    Qb, Kb, Vb = _bf(rng, (H, 192)), _bf(rng, (L, G, 192)), _bf(rng, (L, G, 128))
    idx = np.arange(0, L, 3, dtype=np.int32)
    sink = rng.standard_normal(H).astype(np.float32) * 3
    o0, l0 = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), idx, None, 0.1)
    o1, l1 = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), idx, sink, 0.1)
    frac = np.exp(l0) / (np.exp(l0) + np.exp(sink.astype(np.float64)))
    np.testing.assert_allclose(o1, o0 * frac[:, None], rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(l1, np.logaddexp(l0, sink.astype(np.float64)), rtol=1e-12)
    # a very negative sink reduces to no sink
    o2, _ = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), idx,
                                 np.full(H, -1e4, np.float32), 0.1)
    np.testing.assert_allclose(o2, o0, rtol=1e-12)


def test_attention_single_key_closed_form():
    rng = np.random.default_rng(21)
    H, G = 64, 4
    Qb, Kb, Vb = _bf(rng, (H, 192)), _bf(rng, (5, G, 192)), _bf(rng, (5, G, 128))
    sink = rng.standard_normal(H).astype(np.float32)
    out, _ = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), np.array([3], np.int32), sink, 0.2)
    for h in range(H):
        g = h // (H // G)
        s = 0.2 * float(Qb[h].double() @ Kb[3, g].double())
        coef = math.exp(s) / (math.exp(s) + math.exp(float(sink[h])))
        np.testing.assert_allclose(out[h], Vb[3, g].double().numpy() * coef, rtol=1e-12)


def test_attention_two_key_hand_example():
    # H=2, G=1, Dk=Dv=2, sm_scale=1; logits (head 0) 0 and 2; values e0, e1;
    # sink 0 on head 0:   o = [1, e^2] / (1 + e^2 + 1)
    # head 1 query orthogonal to both keys: logits 0, 0; sink -inf (huge negative): o = mean
    Q = torch.tensor([[1.0, 0.0], [0.0, 1.0]]).to(torch.bfloat16)
    K = torch.tensor([[[0.0, 0.0]], [[2.0, 0.0]]]).to(torch.bfloat16)
    V = torch.tensor([[[1.0, 0.0]], [[0.0, 1.0]]]).to(torch.bfloat16)
    sink = np.array([0.0, -1e30], np.float32)
    out, lse = oracle.gqa_attention(bits16(Q), bits16(K), bits16(V), np.array([0, 1], np.int32), sink, 1.0)
    e2 = math.exp(2.0)
    np.testing.assert_allclose(out[0], [1 / (2 + e2), e2 / (2 + e2)], rtol=1e-14)
    np.testing.assert_allclose(out[1], [0.5, 0.5], rtol=1e-14)
    np.testing.assert_allclose(lse[0], math.log(2 + e2), rtol=1e-14)


def test_gqa_equals_mha_with_repeated_heads():
    """KV head h/16 (contiguous groups): repeating each KV head 16 times and
    running 64 KV heads must give the same output; a strided (h % 4) mapping
    would not."""
    rng = np.random.default_rng(22)
    L, H, G = 200, 64, 4
    Qb, Kb, Vb = _bf(rng, (H, 192)), _bf(rng, (L, G, 192)), _bf(rng, (L, G, 128))
    idx = np.arange(L, dtype=np.int32)
    sink = rng.standard_normal(H).astype(np.float32)
    a, _ = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), idx, sink, 0.07)
    K64 = Kb.repeat_interleave(H // G, 1)
    V64 = Vb.repeat_interleave(H // G, 1)
    b, _ = oracle.gqa_attention(bits16(Qb), bits16(K64), bits16(V64), idx, sink, 0.07)
    assert np.array_equal(a, b)
    K64s = Kb.repeat(1, H // G, 1)          # strided mapping, must differ
    c, _ = oracle.gqa_attention(bits16(Qb), bits16(K64s), bits16(Vb.repeat(1, H // G, 1)), idx, sink, 0.07)
    assert not np.allclose(a, c)


def test_dsa_with_topk_covering_context_is_dense_causal_attention():
    wl = make_decode_workload(seed=30, seq_lens=[700], T=3, n_needles=4)
    r = oracle.dsa_layer_decode(wl.q8[0].numpy(), wl.q_scale[0].numpy(), wl.w[0].numpy(),
                                wl.k8.numpy(), wl.k_scale.numpy(), bits16(wl.Q[0]), bits16(wl.K),
                                bits16(wl.V), wl.q_pos[0].numpy(), 2048, wl.sink.numpy(), 0.5)
    for t in range(3):
        p = int(wl.q_pos[0, t])
        assert r["count"][t] == p + 1
        dense, _ = oracle.gqa_attention(bits16(wl.Q[0, t]), bits16(wl.K), bits16(wl.V),
                                        np.arange(p + 1, dtype=np.int32), wl.sink.numpy(), 0.5)
        np.testing.assert_allclose(r["out"][t], dense, rtol=1e-12, atol=1e-15)
    # no sink: equal to torch SDPA with a causal mask over the whole context
    r0 = oracle.dsa_layer_decode(wl.q8[0].numpy(), wl.q_scale[0].numpy(), wl.w[0].numpy(),
                                 wl.k8.numpy(), wl.k_scale.numpy(), bits16(wl.Q[0]), bits16(wl.K),
                                 bits16(wl.V), wl.q_pos[0].numpy(), 4096, None, 0.5)
    for t in range(3):
        p = int(wl.q_pos[0, t])
        ref = _sdpa(wl.Q[0, t], wl.K, wl.V, np.arange(p + 1), 0.5)
        np.testing.assert_allclose(r0["out"][t], ref, rtol=1e-10, atol=1e-13)


def test_swa_window_covering_context_is_full_attention_and_window_bounds():
    rng = np.random.default_rng(40)
    L, H, G = 300, 64, 8
    Qb, Kb, Vb = _bf(rng, (1, H, 192)), _bf(rng, (L, G, 192)), _bf(rng, (L, G, 128))
    sink = rng.standard_normal(H).astype(np.float32)
    full = oracle.swa_layer_decode(bits16(Qb), bits16(Kb), bits16(Vb), [L - 1], 4096, sink, 0.3)
    ref, _ = oracle.gqa_attention(bits16(Qb[0]), bits16(Kb), bits16(Vb), np.arange(L, dtype=np.int32), sink, 0.3)
    np.testing.assert_allclose(full["out"][0], ref, rtol=1e-12)
    # window 128 at p: exactly keys p-127..p (query_offset - key_offset < 128)
    assert list(oracle.swa_indices(200, 128)) == list(range(73, 201))
    assert list(oracle.swa_indices(5, 128)) == list(range(0, 6))
    base = oracle.swa_layer_decode(bits16(Qb), bits16(Kb), bits16(Vb), [200], 128, sink, 0.3)["out"]
    K2 = Kb.clone()
    K2[72] = 0                 # just outside the window: no effect
    same = oracle.swa_layer_decode(bits16(Qb), bits16(K2), bits16(Vb), [200], 128, sink, 0.3)["out"]
    assert np.array_equal(base, same)
    K2[73] = 0                 # inside the window: changes the output
    diff = oracle.swa_layer_decode(bits16(Qb), bits16(K2), bits16(Vb), [200], 128, sink, 0.3)["out"]
    assert not np.array_equal(base, diff)


def test_attention_order_invariance():
    rng = np.random.default_rng(50)
    L, H, G = 400, 64, 4
    Qb, Kb, Vb = _bf(rng, (H, 192)), _bf(rng, (L, G, 192)), _bf(rng, (L, G, 128))
    idx = rng.choice(L, 256, replace=False).astype(np.int32)
    a, _ = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), idx, None, 0.1)
    b, _ = oracle.gqa_attention(bits16(Qb), bits16(Kb), bits16(Vb), idx[::-1].copy(), None, 0.1)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------- stack constants
def test_stack_constants_from_the_pages():
    g = load_golden("stack_constants.txt")
    dsa = [int(x) for x in g["dsa_layers"]]
    n = int(g["num_layers"][0])
    # eight six-layer modules of 5 SWA + 1 DSA, plus layer 0 also DSA
    pattern = [0 if (i == 0 or i % 6 == 5) else 1 for i in range(n)]
    assert [i for i, x in enumerate(pattern) if x == 0] == dsa
    assert sum(pattern) == int(g["swa_layer_count"][0]) and len(dsa) == int(g["dsa_layer_count"][0])
    W, K, Lmax = int(g["sliding_window"][0]), int(g["index_top_k"][0]), int(g["max_position_embeddings"][0])
    assert 39 * W + 9 * K == int(g["backbone_keys_per_token_sparse"][0])
    assert 39 * W + 9 * Lmax == int(g["backbone_keys_per_token_if_dense"][0])


def test_oracle_results_do_not_depend_on_the_thread_count():
    """The all-core timing of the oracle computes the same numbers as one
    thread: each score and each head's output keeps its own summation order."""
    from workloads import bits16, make_decode_workload
    wl = make_decode_workload(seed=5, seq_lens=[5000], T=2, n_needles=4)
    args = (wl.q8[0].numpy(), wl.q_scale[0].numpy(), wl.w[0].numpy(), wl.k8.numpy(), wl.k_scale.numpy(),
            wl.q_pos[0].numpy())
    sel = np.arange(0, 5000, 3, dtype=np.int32)
    try:
        oracle.set_threads(1)
        s1 = oracle.indexer_scores(*args)
        o1, l1 = oracle.gqa_attention(bits16(wl.Q[0, 0]), bits16(wl.K), bits16(wl.V), sel, wl.sink.numpy(), 0.07)
        oracle.set_threads(4)
        s4 = oracle.indexer_scores(*args)
        o4, l4 = oracle.gqa_attention(bits16(wl.Q[0, 0]), bits16(wl.K), bits16(wl.V), sel, wl.sink.numpy(), 0.07)
    finally:
        oracle.set_threads(1)
    assert np.array_equal(s1.view(np.uint32), s4.view(np.uint32))
    assert np.array_equal(o1, o4) and np.array_equal(l1, l4)


# ------------------------------------------------- index-K / index-Q producer
def _bf16_bits(values):
    return bits16(torch.tensor([float(v) for v in values], dtype=torch.float32).to(torch.bfloat16))


def test_index_key_producer_hand_worked_example():
    g = load_golden("index_producer_worked_example.txt")
    k = _bf16_bits(g["k_bf16_values"])
    ones, zeros = np.ones(4, np.float32), np.zeros(4, np.float32)
    codes, scale, y = oracle.index_k_produce(k, ones, zeros, 0.0, int(g["k_rot"][0]), float(g["k_base"][0]),
                                             int(g["k_pos"][0]))
    assert np.allclose(y, _floats(g["k_y"]).astype(np.float64), rtol=0, atol=1e-9 + 1e-6)
    assert scale == np.float32(float(g["k_scale"][0]))
    assert np.array_equal(codes, _codes(g["k_codes"]))


def test_index_query_producer_hand_worked_example():
    g = load_golden("index_producer_worked_example.txt")
    q = _bf16_bits(g["q_bf16_values"]).reshape(2, 4)
    codes, scale, y = oracle.index_q_produce(q, int(g["q_rot"][0]), float(g["q_base"][0]), int(g["q_pos"][0]))
    assert np.allclose(y.reshape(-1), _floats(g["q_y"]).astype(np.float64), atol=1e-6)
    assert scale == np.float32(float(g["q_scale"][0]))
    assert np.array_equal(codes.reshape(-1), _codes(g["q_codes"]))   # includes a tie broken to the even code


def test_e4m3_encode_matches_torch_rounding():
    """Round-to-nearest-even onto the e4m3 grid, checked against torch's
    float8_e4m3fn conversion on random values, every grid point and every
    midpoint between neighbours (within +-448, where torch does not saturate)."""
    grid = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = (grid[1:] + grid[:-1]) / 2
    rng = np.random.default_rng(3)
    vals = np.concatenate([grid, mids, rng.uniform(-448, 448, 3000), rng.normal(0, 1, 3000),
                           rng.normal(0, 1e-3, 1000)]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    mine = oracle.e4m3_encode(vals)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)
    assert list(oracle.e4m3_encode(np.array([448.0, 449.0, 1e6, -1e6], np.float32))) == [0x7E, 0x7E, 0x7E, 0xFE]


def test_layernorm_closed_forms():
    rng = np.random.default_rng(4)
    x = rng.normal(3.0, 2.0, 128)
    ones, zeros = np.ones(128, np.float32), np.zeros(128, np.float32)
    y = oracle.layernorm(x, ones, zeros, 0.0)
    assert abs(y.mean()) < 1e-12 and abs((y * y).mean() - 1.0) < 1e-12
    # invariant under x -> a x + c (a > 0) without eps
    assert np.allclose(oracle.layernorm(2.5 * x - 7.0, ones, zeros, 0.0), y, atol=1e-12)
    # weight and bias act per dimension after the normalisation
    w = rng.uniform(0.5, 2, 128).astype(np.float32)
    b = rng.normal(0, 1, 128).astype(np.float32)
    assert np.allclose(oracle.layernorm(x, w, b, 0.0), y * w + b, atol=1e-12)
    # eps enters as sqrt(var + eps)
    var = x.var()
    assert np.allclose(oracle.layernorm(x, ones, zeros, 0.5), (x - x.mean()) / np.sqrt(var + 0.5), atol=1e-12)


def test_partial_rope_is_a_complex_rotation_of_the_half_pairs():
    """Pairs (i, i + rot/2) as complex numbers x_i + i x_{i+h} multiplied by
    exp(i pos base^(-2i/rot)); the dims past rot unchanged."""
    rng = np.random.default_rng(6)
    D, rot, base = 128, 42, 1e7
    x = rng.normal(0, 1, D)
    for pos in (0, 1, 17, 65535, 1048575):
        y = oracle.rope_partial(x, rot, pos, base)
        h = rot // 2
        z = (x[:h] + 1j * x[h:rot]) * np.exp(1j * pos * base ** (-2.0 * np.arange(h) / rot))
        assert np.allclose(y[:h], z.real, atol=1e-9) and np.allclose(y[h:rot], z.imag, atol=1e-9)
        assert np.array_equal(y[rot:], x[rot:])
    assert np.array_equal(oracle.rope_partial(x, 0, 12345, base), x)


def test_partial_rope_depends_on_relative_position_only():
    rng = np.random.default_rng(7)
    q, k = rng.normal(0, 1, 128), rng.normal(0, 1, 128)
    rot, base = 42, 1e7
    d1 = oracle.rope_partial(q, rot, 1000, base) @ oracle.rope_partial(k, rot, 700, base)
    d2 = oracle.rope_partial(q, rot, 51300, base) @ oracle.rope_partial(k, rot, 51000, base)
    assert abs(d1 - d2) < 1e-9
    back = oracle.rope_partial(oracle.rope_partial(q, rot, 777, base), rot, -777, base)
    assert np.allclose(back, q, atol=1e-12)


def test_producer_scale_maps_the_largest_magnitude_to_448():
    rng = np.random.default_rng(8)
    k = bits16(torch.from_numpy(rng.normal(0, 1, 128).astype(np.float32)).to(torch.bfloat16))
    w = rng.uniform(0.5, 1.5, 128).astype(np.float32)
    b = rng.normal(0, 0.1, 128).astype(np.float32)
    codes, scale, y = oracle.index_k_produce(k, w, b, 1e-5, 42, 1e7, 123456)
    y32 = y.astype(np.float32)
    assert scale == np.float32(np.abs(y32).max()) / np.float32(448.0)
    assert codes[np.argmax(np.abs(y32))] & 0x7F == 0x7E
    # dequantised codes reproduce the values within half an e4m3 step (relative 1/16) or the subnormal step
    deq = oracle.e4m3_to_float64(codes) * scale
    assert np.all(np.abs(deq - y) <= np.maximum(np.abs(y) / 16, scale * 2.0 ** -10) + 1e-7)


# --------------------------------------------- indexer warm-up KL target
def _kl_inputs(seed, n, H=8, G=2, Dk=16, std=1.0):
    rng = np.random.default_rng(seed)
    Q = bits16(torch.from_numpy(rng.normal(0, std, (H, Dk)).astype(np.float32)).to(torch.bfloat16))
    K = bits16(torch.from_numpy(rng.normal(0, std, (n, G, Dk)).astype(np.float32)).to(torch.bfloat16))
    I = rng.normal(0, 2, n).astype(np.float32)
    return Q, K, I


def test_kl_target_is_the_head_mean_of_softmax_attention():
    """The target equals torch's float64 softmax of the scaled logits, averaged
    over heads; each head reads its contiguous KV group."""
    Q, K, I = _kl_inputs(1, 300)
    sm = 0.25
    kl, P = oracle.indexer_kl(Q, K, I, 299, sm)
    q = torch.from_numpy(oracle.bf16_to_float64(Q))
    k = torch.from_numpy(oracle.bf16_to_float64(K))
    H, G = q.shape[0], k.shape[1]
    logits = torch.stack([sm * k[:, h // (H // G)] @ q[h] for h in range(H)])
    ref = torch.softmax(logits, dim=-1).mean(0).numpy()
    assert np.allclose(P, ref, rtol=1e-12, atol=1e-15)
    assert abs(P.sum() - 1.0) < 1e-12
    r = torch.log_softmax(torch.from_numpy(I.astype(np.float64)), 0).numpy()
    assert abs(kl - float((ref * (np.log(ref) - r)).sum())) < 1e-12
    # a strided head -> KV mapping gives a different target
    logits_s = torch.stack([sm * k[:, h % G] @ q[h] for h in range(H)])
    assert not np.allclose(P, torch.softmax(logits_s, dim=-1).mean(0).numpy(), atol=1e-6)


def test_kl_is_zero_when_the_indexer_matches_the_target():
    Q, K, I = _kl_inputs(2, 200)
    _, P = oracle.indexer_kl(Q, K, I, 199, 0.3)
    kl, _ = oracle.indexer_kl(Q, K, (np.log(P) + 5.0).astype(np.float32), 199, 0.3)
    assert abs(kl) < 1e-6                      # float32 rounding of the matched scores only
    kl1, _ = oracle.indexer_kl(Q, K, I, 0, 0.3)   # a single visible key: both distributions are [1]
    assert kl1 == 0.0


def test_kl_closed_form_for_uniform_attention_and_shift_invariance():
    Q, K, I = _kl_inputs(3, 500)
    Qz = np.zeros_like(Q)                      # every logit 0: each head uniform over the keys
    n = 400
    kl, P = oracle.indexer_kl(Qz, K, I, n - 1, 0.1)
    i = I[:n].astype(np.float64)
    lse = i.max() + np.log(np.exp(i - i.max()).sum())
    assert np.allclose(P, 1.0 / n)
    assert abs(kl - (-np.log(n) - i.mean() + lse)) < 1e-10
    kl2, _ = oracle.indexer_kl(Qz, K, I + np.float32(3.0), n - 1, 0.1)
    assert abs(kl2 - kl) < 1e-6
    assert kl > 0
