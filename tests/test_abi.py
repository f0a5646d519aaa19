"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments on the host before touching a GPU (runs without one)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT, load_golden

HEADER = os.path.join(ROOT, "include", "dsa.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)) - {"defined"})


@pytest.fixture(scope="module")
def dsa():
    import local_attention_decode_b200 as m
    return m


def test_header_declares_the_expected_entry_points():
    names = _declared_functions()
    for n in ("dsa_indexer_scores", "dsa_topk_select", "sparse_gqa_attn_decode", "swa_attn_decode",
              "dsa_layer_decode", "dsa_prefill", "dsa_workspace_size", "dsa_check_device_status",
              "dsa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(dsa):
    lib = ctypes.CDLL(dsa.LIB_PATH)
    for n in _declared_functions():
        assert hasattr(lib, n), n
    assert set(dsa.EXPORTED) <= set(_declared_functions())


def test_compiled_dims_match_the_pages(dsa):
    g = load_golden("stack_constants.txt")
    dims = dsa.get_dims()
    assert dims[0] == int(g["index_heads"][0])
    assert dims[2] == int(g["num_attention_heads"][0])
    assert dims[3] == int(g["head_dim"][0])
    assert dims[4] == int(g["v_head_dim"][0])
    assert dims[5] >= int(g["index_top_k"][0])
    assert dims[1] == 128


def test_host_side_argument_errors(dsa):
    lib = dsa._lib
    out = ctypes.c_size_t(0)
    assert lib.dsa_workspace_size(99, 1, 1, 100, 10, ctypes.byref(out)) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_workspace_size(dsa.OP_TOPK, 0, 1, 100, 10, ctypes.byref(out)) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert lib.dsa_workspace_size(dsa.OP_TOPK, 1, 17, 100, 10, ctypes.byref(out)) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert lib.dsa_workspace_size(dsa.OP_TOPK, 1, 1, 100, 4096, ctypes.byref(out)) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert b"top_k" in lib.dsa_last_error()
    assert lib.dsa_workspace_size(dsa.OP_SWA_ATTN, 1, 1, 100, 128, ctypes.byref(out)) == dsa.DSA_OK
    assert out.value > 0
    # null pointers are rejected before any CUDA call
    kv = dsa.dsa_kv_t()
    assert lib.dsa_indexer_scores(None, None, None, ctypes.byref(kv), None, 1, 1, 10, None, 10, None, 0,
                                  None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk_select(None, 10, None, 1, 1, 10, 5, None, None, None, 0, None) == dsa.DSA_ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)
    kv.k = fake
    kv.v = fake
    kv.num_kv_heads = 3          # not a divisor of 64
    kv.num_rows = 10
    kv.seq_stride = 10
    rc = lib.sparse_gqa_attn_decode(fake, ctypes.byref(kv), fake, fake, 1, 1, 16, None, ctypes.c_float(0.1), fake,
                                    None, fake, 1 << 20, None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    kv.num_kv_heads = 4
    kv.block_table = fake
    kv.page_size = 48            # pages must tile 128-key blocks
    kv.max_pages = 4
    rc = lib.swa_attn_decode(fake, ctypes.byref(kv), fake, 1, 1, 128, None, ctypes.c_float(0.1), fake, None, fake,
                             1 << 20, None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    kv.page_size = 64
    kv.num_rows = 128
    rc = lib.swa_attn_decode(fake, ctypes.byref(kv), fake, 1, 1, 128, None, ctypes.c_float(0.1), fake, None, fake,
                             16, None)
    assert rc == dsa.DSA_ERR_WORKSPACE_TOO_SMALL


def test_workspace_sizes_grow_with_the_problem(dsa):
    a = dsa.workspace_size(dsa.OP_LAYER, 1, 1, 8192, 2048)
    b = dsa.workspace_size(dsa.OP_LAYER, 1, 4, 65536, 2048)
    assert b > a > 8192 * 4


def test_prefill_workspace_covers_every_block(dsa):
    """dsa_prefill runs 16-token blocks and a shorter last one on one
    workspace layout: at least what each block needs, at most what both would
    need side by side."""
    for nq, last in ((40, 8), (16, 16), (5, 5)):
        need = dsa.workspace_size(dsa.OP_PREFILL, 1, nq, 8192, 2048)
        sizes = [dsa.workspace_size(dsa.OP_LAYER, 1, t, 8192, 2048) for t in {min(16, nq), last}]
        assert max(sizes) <= need <= sum(sizes)
    size = ctypes.c_size_t(0)
    assert dsa._lib.dsa_workspace_size(dsa.OP_PREFILL, 2, 40, 8192, 2048, ctypes.byref(size)) == \
        dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert dsa._lib.dsa_workspace_size(dsa.OP_PREFILL, 1, 0, 8192, 2048, ctypes.byref(size)) == \
        dsa.DSA_ERR_UNSUPPORTED_SHAPE


def test_batched_contiguous_stride_rejected_on_the_host(dsa):
    """B > 1 sequences in one contiguous index cache need seq_stride % 16 == 0
    (the per-row scale copies start at b * seq_stride); the check happens on
    the host, before any device memory is touched, so placeholder (never
    dereferenced) 16-byte-aligned addresses are enough here."""
    lib = dsa._lib
    fake = ctypes.c_void_p(1 << 20)
    kv = dsa.dsa_kv_t()
    kv.k = kv.v = kv.index_k = kv.index_k_scale = fake
    kv.num_kv_heads = 4
    kv.seq_stride = 1001
    kv.num_rows = 4096
    rc = lib.dsa_layer_decode(fake, fake, fake, fake, ctypes.byref(kv), fake, 2, 1, 1000, 2048, None,
                              ctypes.c_float(0.07), fake, None, None, None, fake, 1 << 20, None, None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert b"seq_stride" in lib.dsa_last_error()
    rc = lib.dsa_indexer_scores(fake, fake, fake, ctypes.byref(kv), fake, 2, 1, 1000, fake, 1000, fake, 1 << 20,
                                None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE


def test_debug_inject_arguments_checked_on_the_host(dsa):
    lib = dsa._lib
    assert lib.dsa_debug_inject(5, 2_000_000) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_debug_inject(dsa.INJECT_BARRIER_TIMEOUT, 0) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_debug_inject(dsa.INJECT_NONE, 0) == dsa.DSA_OK


def test_trace_and_path_count_arguments_checked_on_the_host(dsa):
    lib = dsa._lib
    assert lib.dsa_trace_phases(None, -1) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_trace_phases(None, 8) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_trace_phases(None, 0) == dsa.DSA_OK            # switched off
    fake = ctypes.c_void_p(1 << 20)                                # never dereferenced: only stored
    assert lib.dsa_trace_phases(fake, 148 * dsa.TRACE_MARKS) == dsa.DSA_OK
    assert lib.dsa_trace_phases(None, 0) == dsa.DSA_OK
    out = ctypes.c_uint32(0)
    assert lib.dsa_layer_path_counts(None, None, ctypes.byref(out), ctypes.byref(out)) == dsa.DSA_ERR_INVALID_ARG
    m = re.search(r"#define DSA_TRACE_MARKS (\d+)", open(HEADER).read())
    assert m and int(m.group(1)) == dsa.TRACE_MARKS
