"""dsa_topk_select_noalloc -- the selection for callers that cannot allocate
device memory (a host framework that owns all device allocations, a
latency-critical loop that must not reach the allocator, a plug-in given only
its input and output buffers).  It must select exactly what dsa_topk_select
selects with a caller workspace, call after call, although every call reuses
the library's one static scratch array.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import local_attention_decode_b200 as dsa  # noqa: E402

DEV = "cuda"


def _with_workspace(scores, q_pos, top_k):
    B, T, Lmax = scores.shape
    idx = torch.full((B, T, top_k), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, T), -7, dtype=torch.int32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_TOPK, B, T, Lmax, top_k)
    dsa.dsa_topk_select(scores, q_pos, Lmax, top_k, idx, cnt, ws)
    return idx, cnt


def _without_workspace(scores, q_pos, top_k):
    """Straight through the C ABI, no workspace argument."""
    B, T, Lmax = scores.shape
    idx = torch.full((B, T, top_k), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, T), -7, dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = dsa._lib.dsa_topk_select_noalloc(ctypes.c_void_p(scores.data_ptr()), Lmax,
                                          ctypes.c_void_p(q_pos.data_ptr()), B, T, Lmax, top_k,
                                          ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()), stream)
    assert rc == dsa.DSA_OK, dsa._lib.dsa_last_error()
    return idx, cnt


def _many_rows_with_ties(g):
    s = torch.randn((74, 1, 10000), generator=g, device=DEV)
    s[3, 0] = torch.randint(0, 3, (10000,), generator=g, device=DEV).float()
    return s.contiguous()


def test_noalloc_topk_matches_workspace_topk_on_consecutive_calls():
    g = torch.Generator(device=DEV).manual_seed(1234)
    cases = [
        # one 1M-position row (split across many CTAs: uses the cross-CTA scratch)
        (torch.rand((1, 1, 1048576), generator=g, device=DEV), None, 2048),
        # four rows of a speculative block with heavy ties, then again with other data
        (torch.randint(0, 7, (1, 4, 70000), generator=g, device=DEV).float(), None, 2048),
        (torch.randn((2, 4, 50000), generator=g, device=DEV), "ragged", 2048),
        # 74 rows of ~10,000 positions: two CTAs per row, and the fixed scratch
        # of 74 rows leaves room for a candidate list of only 976 entries
        # (shortened to fit the 2 MiB array); row 3 has so many tied scores that
        # the list overflows and the selection exchanges every digit instead
        (_many_rows_with_ties(g), None, 2048),
    ]
    for scores, pos_kind, k in cases:
        B, T, L = scores.shape
        if pos_kind == "ragged":
            q_pos = torch.randint(0, L, (B, T), generator=g, device=DEV, dtype=torch.int32)
            q_pos[0, 0] = 5
        else:
            q_pos = torch.full((B, T), L - 1, dtype=torch.int32, device=DEV)
        ref_idx, ref_cnt = _with_workspace(scores, q_pos, k)
        for _ in range(2):   # two calls in a row on the shared scratch
            idx, cnt = _without_workspace(scores, q_pos, k)
            torch.cuda.synchronize()
            assert torch.equal(cnt, ref_cnt)
            assert torch.equal(idx, ref_idx)
