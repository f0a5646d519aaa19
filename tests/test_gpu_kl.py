"""Parity of dsa_indexer_kl (the indexer warm-up target and KL loss) with the
CPU oracle: the target distribution elementwise (1e-3 relative + 1e-7) and
the KL per token (1e-4 relative, 1e-5 absolute); contiguous and paged
caches, GQA4 and GQA8, ragged positions, peaked and flat attention."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import local_attention_decode_b200 as dsa  # noqa: E402
from workloads import bits16, make_decode_workload, logical_rows  # noqa: E402
from parity import kv_for  # noqa: E402

DEV = "cuda"
SM = 1.0 / math.sqrt(192)


@pytest.mark.parametrize("case", [
    dict(seq_lens=[3000, 700], T=2, G=4, page_size=0, qk_std=1.0),
    dict(seq_lens=[2100, 129, 64], T=1, G=8, page_size=64, qk_std=None),
    dict(seq_lens=[5000], T=3, G=4, page_size=16, qk_std=0.5),
])
def test_indexer_kl_matches_oracle(case):
    wl = make_decode_workload(seed=120, device=DEV, n_needles=4, **case)
    Lmax = int(wl.q_pos.max()) + 1
    scores = torch.full((wl.B, wl.T, Lmax), float("nan"), device=DEV)
    iws = dsa.alloc_workspace(dsa.OP_INDEXER, wl.B, wl.T, Lmax, 1)
    kv = kv_for(wl)
    dsa.dsa_indexer_scores(wl.q8, wl.q_scale, wl.w, kv, wl.q_pos, Lmax, scores, iws)
    kl = torch.full((wl.B, wl.T), float("nan"), device=DEV)
    target = torch.full((wl.B, wl.T, Lmax), -1.0, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_KL, wl.B, wl.T, Lmax, 1)
    dsa.dsa_indexer_kl(wl.Q, kv, scores, wl.q_pos, Lmax, SM, kl, target, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK
    for b in range(wl.B):
        rows = logical_rows(wl, b, int(wl.q_pos[b].max()) + 1)
        K = bits16(wl.K[rows])
        for t in range(wl.T):
            p = int(wl.q_pos[b, t])
            ref_kl, ref_P = oracle.indexer_kl(bits16(wl.Q[b, t]), K[:p + 1], scores[b, t].cpu().numpy(), p, SM)
            got_P = target[b, t, :p + 1].cpu().numpy().astype(np.float64)
            assert np.all(np.abs(got_P - ref_P) <= 1e-3 * ref_P + 1e-7), np.abs(got_P - ref_P).max()
            assert np.all(target[b, t, p + 1:].cpu().numpy() == -1.0)   # past the query: untouched
            assert abs(float(kl[b, t]) - ref_kl) <= 1e-4 * max(1.0, abs(ref_kl)) + 1e-5, (float(kl[b, t]), ref_kl)


def test_indexer_kl_is_deterministic_and_target_optional():
    wl = make_decode_workload(seed=121, seq_lens=[4000], T=2, device=DEV, n_needles=2)
    Lmax = 4000
    scores = torch.randn((1, 2, Lmax), device=DEV)
    kv = kv_for(wl)
    ws = dsa.alloc_workspace(dsa.OP_KL, 1, 2, Lmax, 1)
    a = torch.empty((1, 2), device=DEV)
    b = torch.empty((1, 2), device=DEV)
    dsa.dsa_indexer_kl(wl.Q, kv, scores, wl.q_pos, Lmax, SM, a, None, ws)
    dsa.dsa_indexer_kl(wl.Q, kv, scores, wl.q_pos, Lmax, SM, b, None, ws)
    assert torch.equal(a, b) and torch.all(a > 0)
