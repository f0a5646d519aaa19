"""Parity of dsa_index_produce (LayerNorm -> partial RoPE -> per-token e4m3 ->
index-key cache write; the index queries' RoPE and e4m3) with the CPU oracle.

Codes are compared exactly, except where the oracle's value / scale lies
within 1e-5 relative of a midpoint between two e4m3 values: there the fp32
rounding of the kernel's LayerNorm / rotation may land on either neighbour,
and both are accepted.  Scales agree to 1e-5 relative.  Positions up to
1,048,575 check the rotary angles at the native context.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import local_attention_decode_b200 as dsa  # noqa: E402
from workloads import bits16, make_layout  # noqa: E402

DEV = "cuda"
ROT, BASE, EPS = 42, 1e7, 1e-5
GRID = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def assert_codes_match(gpu, ref, v):
    """gpu, ref: uint8 codes; v: the oracle's value / scale (float64)."""
    gpu, ref, v = gpu.reshape(-1), ref.reshape(-1), v.reshape(-1)
    for i in np.flatnonzero(gpu != ref):
        a = abs(v[i])
        j = np.searchsorted(GRID, a)
        assert 0 < j < len(GRID), (i, v[i])
        mid = (GRID[j - 1] + GRID[j]) / 2
        assert abs(a - mid) <= 1e-5 * a, f"code {gpu[i]:#x} != {ref[i]:#x} at value {v[i]!r} (not a rounding tie)"
        sign = 0x80 if v[i] < 0 else 0
        assert gpu[i] in (sign | (j - 1), sign | j)


def _run(B, T, positions, page_size=0, seq_len=4096, with_q=True, seed=0):
    g = torch.Generator(device=DEV).manual_seed(seed)
    lay = make_layout([seq_len] * B, page_size=page_size, seed=seed, device=DEV)
    rows = lay.num_rows
    index_k = torch.full((rows, 128), 0xAB, dtype=torch.uint8, device=DEV)
    index_ks = torch.full((rows,), -1.0, dtype=torch.float32, device=DEV)
    kv = dsa.KV(index_k=index_k, index_k_scale=index_ks, num_kv_heads=4, seq_stride=lay.seq_stride,
                block_table=lay.block_table, page_size=lay.page_size, num_rows=rows)
    k_in = (torch.randn((B, T, 128), generator=g, device=DEV) * 3 + 1).to(torch.bfloat16)
    q_in = torch.randn((B, T, 16, 128), generator=g, device=DEV).to(torch.bfloat16) if with_q else None
    ln_w = (torch.rand(128, generator=g, device=DEV) + 0.5).contiguous()
    ln_b = (torch.randn(128, generator=g, device=DEV) * 0.1).contiguous()
    q_pos = torch.tensor(positions, dtype=torch.int32, device=DEV).view(B, T)
    q8 = torch.zeros((B, T, 16, 128), dtype=torch.uint8, device=DEV)
    qs = torch.zeros((B, T, 16), dtype=torch.float32, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_PRODUCE, B, T, 1, 1)
    dsa.dsa_index_produce(k_in, q_in, ln_w, ln_b, EPS, ROT, BASE, kv, q_pos, q8 if with_q else None,
                          qs if with_q else None, ws)
    st, _ = dsa.dsa_check_device_status(ws)
    return dict(lay=lay, index_k=index_k, index_ks=index_ks, k_in=k_in, q_in=q_in, ln_w=ln_w.cpu().numpy(),
                ln_b=ln_b.cpu().numpy(), q_pos=q_pos, q8=q8, qs=qs, status=st)


def _check(r, with_q=True):
    assert r["status"] == dsa.DSA_OK
    lay, q_pos = r["lay"], r["q_pos"]
    B, T = q_pos.shape
    written = set()
    for b in range(B):
        for t in range(T):
            pos = int(q_pos[b, t])
            row = int(lay.rows(b, torch.tensor([pos], device=DEV))[0])
            written.add(row)
            codes, scale, y = oracle.index_k_produce(bits16(r["k_in"][b, t]), r["ln_w"], r["ln_b"], EPS, ROT, BASE,
                                                     pos)
            gs = float(r["index_ks"][row])
            assert abs(gs - scale) <= 1e-5 * scale
            assert_codes_match(r["index_k"][row].cpu().numpy(), codes, y / scale)
            if with_q:
                qc, qscale, qy = oracle.index_q_produce(bits16(r["q_in"][b, t]), ROT, BASE, pos)
                gq = r["qs"][b, t].cpu().numpy()
                assert np.all(np.abs(gq - qscale) <= 1e-5 * qscale)
                assert_codes_match(r["q8"][b, t].cpu().numpy(), qc, qy / qscale)
    # every other cache row is untouched
    untouched = np.setdiff1d(np.arange(lay.num_rows), np.array(sorted(written)))
    sample = untouched[:: max(1, len(untouched) // 4096)]
    assert np.all(r["index_k"][sample].cpu().numpy() == 0xAB)
    assert np.all(r["index_ks"][sample].cpu().numpy() == -1.0)


def test_produce_contiguous_batch():
    rng = np.random.default_rng(1)
    r = _run(3, 2, rng.integers(0, 4096, 6).tolist(), seed=1)
    _check(r)


def test_produce_paged_batch_and_key_only():
    rng = np.random.default_rng(2)
    r = _run(2, 3, rng.integers(0, 4096, 6).tolist(), page_size=64, seed=2)
    _check(r)
    r = _run(2, 2, [0, 63, 64, 4095], page_size=16, seed=3, with_q=False)   # page boundaries, no query
    _check(r, with_q=False)


def test_produce_at_the_native_context_positions():
    """Rotary angles at positions near 2^20 (the highest frequency turns by
    about a million radians)."""
    r = _run(1, 4, [1048572, 1048573, 1048574, 1048575], seq_len=1048576, seed=4)
    _check(r)


def test_produce_flags_a_position_outside_the_cache():
    lay = make_layout([256], page_size=64, seed=5, device=DEV)
    index_k = torch.full((lay.num_rows, 128), 0xAB, dtype=torch.uint8, device=DEV)
    index_ks = torch.full((lay.num_rows,), -1.0, dtype=torch.float32, device=DEV)
    kv = dsa.KV(index_k=index_k, index_k_scale=index_ks, num_kv_heads=4, block_table=lay.block_table,
                page_size=64, num_rows=lay.num_rows)
    k_in = torch.randn((1, 2, 128), device=DEV).to(torch.bfloat16)
    q_pos = torch.tensor([[10, 5000]], dtype=torch.int32, device=DEV)   # 5000 is past the sequence's pages
    ones, zeros = torch.ones(128, device=DEV), torch.zeros(128, device=DEV)
    ws = dsa.alloc_workspace(dsa.OP_PRODUCE, 1, 2, 1, 1)
    dsa.dsa_index_produce(k_in, None, ones, zeros, EPS, ROT, BASE, kv, q_pos, None, None, ws)
    st, flags = dsa.dsa_check_device_status(ws)
    assert st == dsa.DSA_ERR_DEVICE_BAD_INDEX
    row10 = int(lay.rows(0, torch.tensor([10], device=DEV))[0])
    changed = (index_k != 0xAB).any(dim=1).nonzero().flatten().tolist()
    assert changed == [row10]
