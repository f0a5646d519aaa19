"""Device-side failure path: a cross-CTA wait that runs out is reported, the
GPU stays usable, a workspace left half-updated is refused until it is
re-initialised, and after re-initialisation the results are correct again.

The failure is made with the library's own injection (dsa_debug_inject): the
first cross-CTA barrier of a launch waits for one arrival more than will come,
bounded by a 2 ms limit.  Nothing faults, traps or hangs: every CTA gives up
after the limit, records the timeout in the workspace and returns.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import local_attention_decode_b200 as dsa  # noqa: E402
from workloads import CONFIGS, make_decode_workload  # noqa: E402
from parity import kv_for, oracle_attention_rows, assert_attn_close  # noqa: E402

DEV = "cuda"
LIMIT_NS = 2_000_000   # 2 ms
SM = 1.0 / np.sqrt(192)


class injected_timeout:
    def __enter__(self):
        dsa.dsa_debug_inject(dsa.INJECT_BARRIER_TIMEOUT, LIMIT_NS)

    def __exit__(self, *exc):
        dsa.dsa_debug_inject(dsa.INJECT_NONE)
        return False


def test_injection_rejects_bad_arguments():
    with pytest.raises(dsa.DSAError):
        dsa.dsa_debug_inject(7, LIMIT_NS)
    with pytest.raises(dsa.DSAError):
        dsa.dsa_debug_inject(dsa.INJECT_BARRIER_TIMEOUT, 10)


def test_selection_barrier_timeout_is_reported_refused_then_recovered():
    n, k = 300000, 2048   # one row over many CTAs: the row barrier is used
    g = torch.Generator(device=DEV).manual_seed(17)
    scores = (torch.rand((1, 1, n), generator=g, device=DEV) * 10).contiguous()
    q_pos = torch.tensor([[n - 1]], dtype=torch.int32, device=DEV)
    idx = torch.full((1, 1, k), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((1, 1), -7, dtype=torch.int32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_TOPK, 1, 1, n, k)

    with injected_timeout():
        dsa.dsa_topk_select(scores, q_pos, n, k, idx, cnt, ws)
        st, flags = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_ERR_DEVICE_TIMEOUT
    assert flags & dsa.STATUS_NEEDS_INIT
    assert int(cnt) == -7   # nothing was emitted

    # the workspace was left half-updated: the next call refuses it
    dsa.dsa_topk_select(scores, q_pos, n, k, idx, cnt, ws)
    st, flags = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_ERR_DEVICE_TIMEOUT and flags & dsa.STATUS_NEEDS_INIT
    assert int(cnt) == -7

    # re-initialised, it selects exactly the oracle's top-k again
    dsa.dsa_workspace_init(ws)
    dsa.dsa_topk_select(scores, q_pos, n, k, idx, cnt, ws)
    st, flags = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_OK and flags == 0
    ref_idx, ref_cnt = oracle.topk(scores[0, 0].cpu().numpy(), k)
    assert int(cnt) == ref_cnt
    assert np.array_equal(idx[0, 0].cpu().numpy(), np.sort(ref_idx))


def test_fused_layer_grid_barrier_timeout_is_reported_refused_then_recovered():
    wl = make_decode_workload(device=DEV, **CONFIGS["tiny_8k"])
    L, k = int(wl.q_pos.max()) + 1, 2048
    O = torch.empty((1, 1, 64, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((1, 1, 64), dtype=torch.float32, device=DEV)
    idx = torch.empty((1, 1, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((1, 1), dtype=torch.int32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_LAYER, 1, 1, L, k)
    kv = kv_for(wl)

    def run():
        dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, L, k, wl.sink, SM, O, lse, idx, cnt, ws)
        return dsa.dsa_check_device_status(ws)

    with injected_timeout():
        st, flags = run()
    assert st == dsa.DSA_ERR_DEVICE_TIMEOUT and flags & dsa.STATUS_NEEDS_INIT
    st, flags = run()   # refused: the grid barrier words are not clean
    assert st == dsa.DSA_ERR_DEVICE_TIMEOUT and flags & dsa.STATUS_NEEDS_INIT

    dsa.dsa_workspace_init(ws)
    for _ in range(2):   # and the call after a good one is good too (self-cleaning scratch)
        st, flags = run()
        assert st == dsa.DSA_OK and flags == 0
        assert int(cnt) == k
        ref_o, ref_l = oracle_attention_rows(wl, 0, 0, idx[0, 0].cpu().numpy(), wl.sink, SM)
        assert_attn_close(O[0, 0], ref_o, lse[0, 0], ref_l)
