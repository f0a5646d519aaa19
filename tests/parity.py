"""Shared helpers of the GPU parity tests: KV descriptors of a workload, the
oracle on the same inputs, and the tolerances.

Tolerances (written here once, used by every parity test):
  * indexer scores: |gpu - ref| <= 1e-3 |ref| + 1e-6 max|ref| (the second term
    absorbs scores that are exactly 0 because every head's dot is <= 0);
    entries the query cannot see are -inf on both sides;
  * selected index sets: identical to the oracle's selection over the same
    (GPU-produced) scores -- bit-exact integers;
  * selection from independently computed scores: every selected position's
    oracle score is >= the oracle's top_k-th score minus 1e-3 relative;
  * attention outputs: |gpu - ref| <= 2e-2 + 1e-2 |ref| elementwise, and per
    head ||gpu - ref|| / ||ref|| <= 1e-2 (the relative norm bound matters
    because with N(0,1)/sqrt(192) inputs |O| is ~1e-3, where the absolute bound
    alone would accept zeros); lse within 1e-3 absolute.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import local_attention_decode_b200 as dsa
from workloads import bits16, logical_rows

SCORE_RTOL, SCORE_ATOL_FRAC = 1e-3, 1e-6
ATTN_ATOL, ATTN_RTOL, ATTN_HEAD_REL = 2e-2, 1e-2, 1e-2
LSE_ATOL = 1e-3


def kv_for(wl, with_index=True, with_backbone=True) -> dsa.KV:
    lay = wl.layout
    return dsa.KV(k=wl.K if with_backbone else None, v=wl.V if with_backbone else None,
                  index_k=wl.k8 if with_index else None, index_k_scale=wl.k_scale if with_index else None,
                  num_kv_heads=wl.G, seq_stride=lay.seq_stride, block_table=lay.block_table,
                  page_size=lay.page_size, num_rows=lay.num_rows)


def assert_scores_close(gpu: np.ndarray, ref: np.ndarray):
    assert gpu.shape == ref.shape
    neg = np.isneginf(ref)
    assert np.array_equal(np.isneginf(gpu), neg)
    g, r = gpu[~neg].astype(np.float64), ref[~neg].astype(np.float64)
    if r.size == 0:
        return
    tol = SCORE_RTOL * np.abs(r) + SCORE_ATOL_FRAC * np.abs(r).max()
    bad = np.abs(g - r) > tol
    assert not bad.any(), f"{bad.sum()} scores off; worst {np.max(np.abs(g - r) / np.maximum(tol, 1e-30)):.3g}x tol"


def assert_attn_close(o_gpu: torch.Tensor, o_ref: np.ndarray, lse_gpu=None, lse_ref=None):
    g = o_gpu.float().cpu().numpy().astype(np.float64).reshape(o_ref.shape)
    err = np.abs(g - o_ref)
    assert np.all(err <= ATTN_ATOL + ATTN_RTOL * np.abs(o_ref)), f"max abs err {err.max():.3g}"
    num = np.linalg.norm((g - o_ref).reshape(-1, o_ref.shape[-1]), axis=-1)
    den = np.linalg.norm(o_ref.reshape(-1, o_ref.shape[-1]), axis=-1)
    rel = num[den > 0] / den[den > 0]
    assert rel.size == 0 or rel.max() <= ATTN_HEAD_REL, f"worst per-head rel err {rel.max():.3g}"
    assert np.all(num[den == 0] == 0)
    if lse_gpu is not None:
        lg = lse_gpu.cpu().numpy().astype(np.float64).reshape(lse_ref.shape)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin)
        assert np.all(np.abs(lg[fin] - lse_ref[fin]) <= LSE_ATOL)


def oracle_scores(wl, b: int) -> np.ndarray:
    """Oracle indexer scores [T, L_b] of sequence b (the whole visible history)."""
    L = int(wl.q_pos[b].max()) + 1
    rows = logical_rows(wl, b, L)
    return oracle.indexer_scores(wl.q8[b].cpu().numpy(), wl.q_scale[b].cpu().numpy(), wl.w[b].cpu().numpy(),
                                 wl.k8[rows].cpu().numpy(), wl.k_scale[rows].cpu().numpy(),
                                 wl.q_pos[b].cpu().numpy())


def oracle_attention_rows(wl, b: int, t: int, positions: np.ndarray, sink, sm_scale: float):
    """Oracle attention of query (b, t) over the given positions (gathers only those rows)."""
    positions = np.asarray(positions, dtype=np.int64)
    rows = wl.layout.rows(b, torch.from_numpy(positions).to(wl.K.device))
    Ks = bits16(wl.K[rows])
    Vs = bits16(wl.V[rows])
    s = None if sink is None else sink.cpu().numpy()
    return oracle.gqa_attention(bits16(wl.Q[b, t]), Ks, Vs, np.arange(len(positions), dtype=np.int32), s, sm_scale)


def selection_agrees_outside_tie_band(sel: np.ndarray, ref_scores: np.ndarray, k: int) -> bool:
    """A selection made from independently computed scores, checked against
    the oracle's scores: the tie band is every position whose oracle score is
    within 1e-3 relative of the oracle's k-th score (where rounding of the
    GPU's fp32 scores may reorder keys).  Outside the band the selection must
    equal the oracle's exactly -- every position above the band selected, none
    below it -- so at most |band| positions can differ from the oracle's top-k,
    and only inside the band."""
    n = ref_scores.shape[0]
    if n <= k:
        return np.array_equal(np.sort(sel), np.arange(n))
    if len(np.unique(sel)) != len(sel) or len(sel) != k:
        return False
    kth = np.partition(ref_scores, n - k)[n - k]
    tol = 1e-3 * abs(kth)
    chosen = np.zeros(n, bool)
    chosen[sel] = True
    above = ref_scores > kth + tol
    below = ref_scores < kth - tol
    return bool(np.all(chosen[above]) and not np.any(chosen[below]))
