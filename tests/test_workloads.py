"""The seeded input recipes (CPU): shapes, positions, layouts and
determinism of the workloads the GPU tests and the benchmark run on.  These
hold no arithmetic of the method; they check that each recipe builds what
its description says."""
import math

import numpy as np
import torch

from workloads import (CONFIGS, log_uniform_lengths, make_decode_workload, make_layout,
                       make_swa_window_workload, ragged_batch_lengths)


def test_ragged_batch_lengths_are_log_uniform_in_range_and_seeded():
    lens = CONFIGS["ragged_b64"]["seq_lens"]
    assert lens == ragged_batch_lengths(3, 64) == log_uniform_lengths(3, 64, 4096, 262144)
    assert len(lens) == 64 and min(lens) >= 4096 and max(lens) <= 262144
    # log-uniform: the logs spread over the whole range, about half below the geometric midpoint
    mid = math.sqrt(4096 * 262144)
    assert 16 <= sum(L < mid for L in lens) <= 48
    assert ragged_batch_lengths(4, 64) != lens


def test_paged_layout_is_a_permutation_of_whole_pages():
    lens = [100, 64, 1, 300]
    lay = make_layout(lens, page_size=64, seed=5)
    pages = [math.ceil(L / 64) for L in lens]
    ids = torch.cat([lay.block_table[b, :n] for b, n in enumerate(pages)])
    assert sorted(ids.tolist()) == list(range(sum(pages)))
    assert lay.num_rows == sum(pages) * 64
    rows = torch.cat([lay.rows(b, torch.arange(L)) for b, L in enumerate(lens)])
    assert len(set(rows.tolist())) == sum(lens)          # no two positions share a row
    assert int(rows.max()) < lay.num_rows


def test_contiguous_layout_rows():
    lay = make_layout([1000, 300], page_size=0)
    assert lay.seq_stride % 128 == 0 and lay.seq_stride >= 1000
    assert int(lay.rows(1, torch.tensor([0]))) == lay.seq_stride


def test_swa_window_workload_maps_exactly_the_window_pages():
    lens = [4129, 70000, 130, 64, 200]
    wl = make_swa_window_workload(11, lens, window=128, page_size=64)
    bt = wl.layout.block_table
    for b, L in enumerate(lens):
        need = set(range(max(0, L - 128) // 64, (L - 1) // 64 + 1))
        mapped = set(int(i) for i in torch.nonzero(bt[b] >= 0).flatten())
        assert mapped == need, b
        rows = wl.layout.rows(b, torch.arange(max(0, L - 128), L))
        assert int(rows.min()) >= 0 and int(rows.max()) < wl.layout.num_rows
    assert wl.K.shape == (wl.layout.num_rows, 8, 192) and wl.V.shape == (wl.layout.num_rows, 8, 128)
    assert wl.q_pos[:, 0].tolist() == [L - 1 for L in lens]
    again = make_swa_window_workload(11, lens, window=128, page_size=64)
    assert torch.equal(again.K.view(torch.int16), wl.K.view(torch.int16))


def test_decode_queries_are_the_last_positions():
    wl = make_decode_workload(seed=7, seq_lens=[500, 40], T=3)
    assert wl.q_pos.tolist() == [[497, 498, 499], [37, 38, 39]]
    # the prefill recipe: the last 8,192 positions of the 1M cache, 0-based
    cfg = CONFIGS["prefill_8k_1m"]
    assert cfg["T"] == 8192 and cfg["seq_lens"] == [1048576]
    first, last = cfg["seq_lens"][0] - cfg["T"], cfg["seq_lens"][0] - 1
    assert (first, last) == (1040384, 1048575)


def test_needles_point_along_the_first_query_and_are_seeded():
    wl = make_decode_workload(seed=9, seq_lens=[5000], T=1, n_needles=6)
    pos = wl.needles[0]
    assert len(pos) == 6 and len(set(pos.tolist())) == 6
    k = wl.k8[pos].view(torch.float8_e4m3fn).float() * wl.k_scale[pos, None]
    q = wl.q8[0, 0, 0].view(torch.float8_e4m3fn).float()
    cos = (k @ q) / (k.norm(dim=1) * q.norm())
    assert float(cos.min()) > 0.99          # the same direction, up to fp8 rounding
    wl2 = make_decode_workload(seed=9, seq_lens=[5000], T=1, n_needles=6)
    assert np.array_equal(wl2.needles[0].numpy(), pos.numpy())
