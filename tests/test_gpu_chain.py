"""dsa_layer_chain: the layer pattern's repeating unit -- five sliding-window
layer-steps and one DSA layer-step ("What 'no full-attention layers' means":
five SWA layers then one DSA layer per module) -- enqueued as one chain of
programmatic dependent launches gives bit-identical outputs to the same calls
made one by one, and the chained DSA step still matches the oracle."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import local_attention_decode_b200 as dsa  # noqa: E402
from workloads import make_decode_workload, make_swa_window_workload  # noqa: E402
from parity import kv_for, oracle_attention_rows, assert_attn_close  # noqa: E402

DEV = "cuda"
SM = 1.0 / math.sqrt(192)


def _same(a, b):
    if a.dtype == torch.bfloat16:
        a, b = a.view(torch.int16), b.view(torch.int16)
    return torch.equal(a, b)


@pytest.mark.parametrize("case", ["capture_path", "separate_kernels"])
def test_chain_of_five_swa_and_one_dsa_equals_the_calls(case):
    if case == "capture_path":       # B * T <= 4: the one-barrier layer-step kernel
        lens, T = [100000], 1
    else:                            # B * T > 16: indexer, selection, attention, combine kernels
        lens, T = [3000, 9000, 20000, 40000, 2500], 4
    wl = make_decode_workload(seed=95, seq_lens=lens, T=T, device=DEV, n_needles=4, page_size=64)
    B = wl.B
    Lmax = int(wl.q_pos.max()) + 1
    swa = [make_swa_window_workload(200 + i, [int(p) + 1 for p in wl.q_pos[:, -1].tolist()], device=DEV)
           for i in range(5)]
    # the SWA workloads have one query token per sequence
    outs = {k: [] for k in ("one_by_one", "chain")}
    for mode in outs:
        Os = [torch.empty((B, 1, 64, 128), dtype=torch.bfloat16, device=DEV) for _ in swa]
        Ls = [torch.empty((B, 1, 64), dtype=torch.float32, device=DEV) for _ in swa]
        O = torch.empty((B, T, 64, 128), dtype=torch.bfloat16, device=DEV)
        lse = torch.empty((B, T, 64), dtype=torch.float32, device=DEV)
        idx = torch.empty((B, T, 2048), dtype=torch.int32, device=DEV)
        cnt = torch.empty((B, T), dtype=torch.int32, device=DEV)
        ws_swa = dsa.alloc_workspace(dsa.OP_SWA_ATTN, B, 1, 1, 128)
        ws = dsa.alloc_workspace(dsa.OP_LAYER, B, T, Lmax, 2048)
        swa_kv = [kv_for(s, with_index=False) for s in swa]
        kv = kv_for(wl)
        if mode == "one_by_one":
            for s, k, o, l in zip(swa, swa_kv, Os, Ls):
                dsa.swa_attn_decode(s.Q, k, s.q_pos, 128, s.sink, SM, o, l, ws_swa)
            dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, Lmax, 2048, wl.sink, SM, O, lse, idx,
                                 cnt, ws)
        else:
            steps = [dsa.swa_step(s.Q, k, s.q_pos, 128, s.sink, SM, o, l, ws_swa)
                     for s, k, o, l in zip(swa, swa_kv, Os, Ls)]
            steps.append(dsa.dsa_step(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, Lmax, 2048, wl.sink, SM, O, lse,
                                      idx, cnt, ws))
            dsa.dsa_layer_chain(steps)
        torch.cuda.synchronize()
        assert dsa.dsa_check_device_status(ws)[0] == dsa.DSA_OK
        assert dsa.dsa_check_device_status(ws_swa)[0] == dsa.DSA_OK
        outs[mode] = Os + Ls + [O, lse, idx, cnt]
    for a, b in zip(outs["one_by_one"], outs["chain"]):
        assert _same(a, b)
    # and the chained DSA step is the layer-step: its attention against the oracle over its selection
    O, lse, idx, cnt = outs["chain"][-4:]
    for b in range(B):
        for t in range(T):
            c = int(cnt[b, t])
            ref_o, ref_l = oracle_attention_rows(wl, b, t, idx[b, t, :c].cpu().numpy(), wl.sink, SM)
            assert_attn_close(O[b, t], ref_o, lse[b, t], ref_l)


def test_chain_checks_every_step_before_enqueueing():
    wl = make_decode_workload(seed=96, seq_lens=[5000], T=1, device=DEV, n_needles=2)
    O = torch.full((1, 1, 64, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_SWA_ATTN, 1, 1, 1, 128)
    kvs = kv_for(wl, with_index=False)
    good = dsa.swa_step(wl.Q, kvs, wl.q_pos, 128, wl.sink, SM, O, None, ws)
    bad = dict(good, top_k=4096)   # a window beyond what is built
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_layer_chain([good, bad])
    assert e.value.code == dsa.DSA_ERR_UNSUPPORTED_SHAPE and "step 1" in str(e.value)
    torch.cuda.synchronize()
    assert torch.all(O == 7.0)   # nothing ran, not even the good first step
