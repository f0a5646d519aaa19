"""Python binding of libdsa: DSA / SWA decode layer-step kernels for B200.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libdsa.so`` (built from ``csrc/`` for sm_100a, C ABI in
``include/dsa.h``).  PyTorch provides device memory and streams.  There is no
fallback path: if the library is missing, importing this package fails.

Function names match the C entry points.  Tensors must be CUDA tensors of the
documented dtype and shape, contiguous, on the current device; the calls are
enqueued on the current torch stream (or ``stream=``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libdsa.so is not built: run `python -c 'import __graft_entry__ as g; g.build()'` "
        "or `python local_attention_decode_b200/_build.py` first")

_lib = ctypes.CDLL(LIB_PATH)

# status codes and constants (include/dsa.h)
DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED_SHAPE = 2
DSA_ERR_WORKSPACE_TOO_SMALL = 3
DSA_ERR_CUDA = 4
DSA_ERR_DEVICE_TIMEOUT = 5
DSA_ERR_DEVICE_BAD_INDEX = 6
OP_INDEXER, OP_TOPK, OP_SPARSE_ATTN, OP_SWA_ATTN, OP_LAYER, OP_PREFILL, OP_PRODUCE, OP_KL = range(8)
STATUS_NEEDS_INIT = 0x80000000
INJECT_NONE, INJECT_BARRIER_TIMEOUT = 0, 1
TRACE_MARKS = 16   # phase marks per CTA of the one-barrier layer-step (dsa_trace_phases)

EXPORTED = ("dsa_last_error", "dsa_get_dims", "dsa_workspace_size", "dsa_workspace_init",
            "dsa_check_device_status", "dsa_indexer_scores", "dsa_topk_select",
            "sparse_gqa_attn_decode", "swa_attn_decode", "dsa_layer_decode", "dsa_topk_select_noalloc",
            "dsa_prefill", "dsa_debug_inject", "dsa_index_produce", "dsa_layer_chain", "dsa_indexer_kl",
            "dsa_shard_positions", "dsa_shard_candidates", "dsa_shard_merge", "dsa_shard_combine",
            "dsa_layer_path_counts", "dsa_trace_phases")


class DSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libdsa error {code}: {msg}")
        self.code = code


class dsa_kv_t(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("index_k", ctypes.c_void_p),
        ("index_k_scale", ctypes.c_void_p),
        ("num_kv_heads", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("seq_stride", ctypes.c_int64),
        ("num_rows", ctypes.c_int64),
        ("block_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


P = ctypes.c_void_p
I32, I64, SZ, F32 = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_lib.dsa_last_error.restype = ctypes.c_char_p
_lib.dsa_last_error.argtypes = []
_lib.dsa_get_dims.argtypes = [P, I32]
_lib.dsa_workspace_size.argtypes = [I32, I32, I32, I64, I32, ctypes.POINTER(ctypes.c_size_t)]
_lib.dsa_workspace_init.argtypes = [P, SZ, P]
_lib.dsa_check_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_uint32)]
_lib.dsa_layer_path_counts.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32)]
_lib.dsa_trace_phases.argtypes = [P, I64]
_lib.dsa_indexer_scores.argtypes = [P, P, P, ctypes.POINTER(dsa_kv_t), P, I32, I32, I64, P, I64, P, SZ, P]
_lib.dsa_topk_select.argtypes = [P, I64, P, I32, I32, I64, I32, P, P, P, SZ, P]
_lib.sparse_gqa_attn_decode.argtypes = [P, ctypes.POINTER(dsa_kv_t), P, P, I32, I32, I32, P, F32, P, P, P, SZ, P]
_lib.swa_attn_decode.argtypes = [P, ctypes.POINTER(dsa_kv_t), P, I32, I32, I32, P, F32, P, P, P, SZ, P]
_lib.dsa_topk_select_noalloc.argtypes = [P, I64, P, I32, I32, I64, I32, P, P, P]
_lib.dsa_layer_decode.argtypes = [P, P, P, P, ctypes.POINTER(dsa_kv_t), P, I32, I32, I64, I32, P, F32, P, P, P, P,
                                  P, SZ, P, P]
_lib.dsa_debug_inject.argtypes = [I32, I64]
_lib.dsa_index_produce.argtypes = [P, P, P, P, F32, I32, ctypes.c_double, ctypes.POINTER(dsa_kv_t), P, I32, I32, P,
                                   P, P, SZ, P]
_lib.dsa_layer_chain.argtypes = [P, I32, P]
_lib.dsa_shard_positions.argtypes = [P, I32, I32, I64, I64, P, P, SZ, P]
_lib.dsa_shard_candidates.argtypes = [P, I64, P, I32, I32, I32, I64, P, P, P]
_lib.dsa_shard_merge.argtypes = [P, P, I32, I32, I32, I32, I64, I64, P, P, P, P, P]
_lib.dsa_shard_combine.argtypes = [P, P, I32, I32, I32, P, P, P, P]
_lib.dsa_indexer_kl.argtypes = [P, ctypes.POINTER(dsa_kv_t), P, I64, P, I32, I32, I64, F32, P, P, I64, P, SZ, P]
_lib.dsa_prefill.argtypes = [P, P, P, P, ctypes.POINTER(dsa_kv_t), P, I32, I64, I32, P, F32, P, P, P, P, P, SZ, P]
for _name in EXPORTED[1:]:
    getattr(_lib, _name).restype = ctypes.c_int


def _check(rc: int):
    if rc != DSA_OK:
        raise DSAError(rc, _lib.dsa_last_error().decode(errors="replace"))


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def get_dims():
    dims = (ctypes.c_int32 * 7)()
    _check(_lib.dsa_get_dims(ctypes.cast(dims, P), 7))
    return list(dims)


def workspace_size(op: int, B: int, T: int, Lmax: int, top_k: int) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.dsa_workspace_size(op, B, T, Lmax, top_k, ctypes.byref(out)))
    return out.value


def alloc_workspace(op: int, B: int, T: int, Lmax: int, top_k: int, device=None) -> torch.Tensor:
    """A zeroed workspace (uint8, 256-byte aligned by the caching allocator)."""
    n = workspace_size(op, B, T, Lmax, top_k)
    ws = torch.zeros(n, dtype=torch.uint8, device=device or "cuda")
    assert ws.data_ptr() % 256 == 0
    return ws


def dsa_workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.dsa_workspace_init(_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def dsa_debug_inject(kind: int, wait_limit_ns: int = 0):
    """Failure injection for tests (include/dsa.h): INJECT_BARRIER_TIMEOUT makes
    the first cross-CTA barrier of the next launches run out after
    wait_limit_ns; INJECT_NONE turns it off."""
    _check(_lib.dsa_debug_inject(int(kind), int(wait_limit_ns)))


def dsa_layer_path_counts(ws: torch.Tensor, stream=None):
    """(fast, general): layer-steps the one-barrier kernel ran on each of its
    paths since the workspace was zeroed; synchronises the stream."""
    f = ctypes.c_uint32(0)
    g = ctypes.c_uint32(0)
    _check(_lib.dsa_layer_path_counts(_ptr(ws, torch.uint8, "ws"), _stream(stream), ctypes.byref(f), ctypes.byref(g)))
    return f.value, g.value


def dsa_trace_phases(buf):
    """Set (a uint64 tensor on the device, viewed as int64 too) or clear
    (None) the phase-trace buffer of the one-barrier layer-step kernel."""
    if buf is None:
        _check(_lib.dsa_trace_phases(None, 0))
    else:
        if buf.dtype not in (torch.int64, torch.uint64) or not buf.is_contiguous():
            raise ValueError("trace buffer must be a contiguous 64-bit tensor")
        _check(_lib.dsa_trace_phases(ctypes.c_void_p(buf.data_ptr()), buf.numel()))


def dsa_check_device_status(ws: torch.Tensor, stream=None):
    """(status, flags) of the device status word; synchronises the stream."""
    st = ctypes.c_int(0)
    fl = ctypes.c_uint32(0)
    _check(_lib.dsa_check_device_status(_ptr(ws, torch.uint8, "ws"), _stream(stream), ctypes.byref(st),
                                        ctypes.byref(fl)))
    return st.value, fl.value


STEP_SWA, STEP_DSA = 1, 2


class dsa_layer_step_t(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32), ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("Lmax", ctypes.c_int64),
        ("q8", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("w", ctypes.c_void_p),
        ("Q", ctypes.c_void_p), ("kv", ctypes.c_void_p), ("q_pos", ctypes.c_void_p),
        ("sink", ctypes.c_void_p), ("sm_scale", ctypes.c_float), ("reserved", ctypes.c_int32),
        ("O", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("idx_out", ctypes.c_void_p),
        ("count_out", ctypes.c_void_p), ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t),
    ]


class KV:
    """KV-cache description (dsa_kv_t) over caller-owned tensors.

    k [rows, G, 192] bf16, v [rows, G, 128] bf16, index_k [rows, 128] uint8 (e4m3
    codes), index_k_scale [rows] f32; contiguous layout with ``seq_stride`` rows
    per sequence, or paged with ``block_table`` [B, max_pages] int32 and
    ``page_size``.
    """

    def __init__(self, *, k=None, v=None, index_k=None, index_k_scale=None, num_kv_heads=None,
                 seq_stride=0, block_table=None, page_size=0, num_rows=None):
        self._keep = (k, v, index_k, index_k_scale, block_table)
        rows = None
        for t in (index_k, k, v, index_k_scale):
            if t is not None:
                rows = t.shape[0]
                break
        if num_rows is None:
            num_rows = rows
        if num_kv_heads is None:
            num_kv_heads = k.shape[1] if k is not None else 0
        s = dsa_kv_t()
        s.k = _ptr(k, torch.bfloat16, "k") if k is not None else None
        s.v = _ptr(v, torch.bfloat16, "v") if v is not None else None
        s.index_k = _ptr(index_k, torch.uint8, "index_k") if index_k is not None else None
        s.index_k_scale = _ptr(index_k_scale, torch.float32, "index_k_scale") if index_k_scale is not None else None
        s.num_kv_heads = int(num_kv_heads)
        s.page_size = int(page_size)
        s.seq_stride = int(seq_stride)
        s.num_rows = int(num_rows)
        s.block_table = _ptr(block_table, torch.int32, "block_table") if block_table is not None else None
        s.max_pages = int(block_table.shape[1]) if block_table is not None else 0
        s.reserved = 0
        self.struct = s

    @property
    def ref(self):
        return ctypes.byref(self.struct)


def _bt(t: torch.Tensor, trailing: Sequence[int], name: str):
    if tuple(t.shape[2:]) != tuple(trailing):
        raise ValueError(f"{name}: expected [B, T, {', '.join(map(str, trailing))}], got {tuple(t.shape)}")
    return t.shape[0], t.shape[1]


def dsa_indexer_scores(q8, q_scale, w, kv: KV, q_pos, Lmax: int, scores, ws, stream=None):
    B, T = _bt(q8, (16, 128), "q8")
    _check(_lib.dsa_indexer_scores(_ptr(q8, torch.uint8, "q8"), _ptr(q_scale, torch.float32, "q_scale"),
                                   _ptr(w, torch.float32, "w"), kv.ref, _ptr(q_pos, torch.int32, "q_pos"), B, T,
                                   int(Lmax), _ptr(scores, torch.float32, "scores"), scores.shape[-1],
                                   _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def dsa_index_produce(k_in, q_in, ln_w, ln_b, ln_eps: float, rope_dim: int, rope_base: float, kv: KV, q_pos,
                      q8_out=None, q_scale_out=None, ws=None, stream=None):
    """k_in [B, T, 128] bf16 (and q_in [B, T, 16, 128] bf16 or None) -> index-key
    cache rows at q_pos, and q8_out [B, T, 16, 128] uint8 / q_scale_out [B, T, 16]."""
    if k_in.dim() != 3 or k_in.shape[2] != 128:
        raise ValueError("k_in must be [B, T, 128]")
    B, T = k_in.shape[:2]
    _check(_lib.dsa_index_produce(_ptr(k_in, torch.bfloat16, "k_in"), _ptr(q_in, torch.bfloat16, "q_in"),
                                  _ptr(ln_w, torch.float32, "ln_w"), _ptr(ln_b, torch.float32, "ln_b"),
                                  float(ln_eps), int(rope_dim), float(rope_base), kv.ref,
                                  _ptr(q_pos, torch.int32, "q_pos"), B, T, _ptr(q8_out, torch.uint8, "q8_out"),
                                  _ptr(q_scale_out, torch.float32, "q_scale_out"), _ptr(ws, torch.uint8, "ws"),
                                  ws.numel(), _stream(stream)))


def dsa_indexer_kl(Q, kv: "KV", scores, q_pos, Lmax: int, sm_scale: float, kl_out, target=None, ws=None,
                   stream=None):
    """KL(head-mean dense attention || softmax(indexer scores)) per query token,
    kl_out [B, T]; target [B, T, >= Lmax] receives the dense distribution."""
    B, T = _bt(Q, (64, 192), "Q")
    _check(_lib.dsa_indexer_kl(_ptr(Q, torch.bfloat16, "Q"), kv.ref, _ptr(scores, torch.float32, "scores"),
                               scores.shape[-1], _ptr(q_pos, torch.int32, "q_pos"), B, T, int(Lmax), float(sm_scale),
                               _ptr(kl_out, torch.float32, "kl_out"), _ptr(target, torch.float32, "target"),
                               target.shape[-1] if target is not None else 0, _ptr(ws, torch.uint8, "ws"), ws.numel(),
                               _stream(stream)))


def dsa_topk_select(scores, q_pos, Lmax: int, top_k: int, idx, count, ws, stream=None):
    B, T = q_pos.shape
    _check(_lib.dsa_topk_select(_ptr(scores, torch.float32, "scores"), scores.shape[-1],
                                _ptr(q_pos, torch.int32, "q_pos"), B, T, int(Lmax), int(top_k),
                                _ptr(idx, torch.int32, "idx"), _ptr(count, torch.int32, "count"),
                                _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def dsa_topk_select_noalloc(scores, q_pos, Lmax: int, top_k: int, idx, count, stream=None):
    """dsa_topk_select without a workspace: the library's own 2 MiB device
    scratch is used (see include/dsa.h for who needs this and its limits)."""
    B, T = q_pos.shape
    _check(_lib.dsa_topk_select_noalloc(_ptr(scores, torch.float32, "scores"), scores.shape[-1],
                                        _ptr(q_pos, torch.int32, "q_pos"), B, T, int(Lmax), int(top_k),
                                        _ptr(idx, torch.int32, "idx"), _ptr(count, torch.int32, "count"),
                                        _stream(stream)))


def sparse_gqa_attn_decode(Q, kv: KV, idx, count, top_k: int, sink, sm_scale: float, O, lse=None, ws=None,
                           stream=None):
    B, T = _bt(Q, (64, 192), "Q")
    _check(_lib.sparse_gqa_attn_decode(_ptr(Q, torch.bfloat16, "Q"), kv.ref, _ptr(idx, torch.int32, "idx"),
                                       _ptr(count, torch.int32, "count"), B, T, int(top_k),
                                       _ptr(sink, torch.float32, "sink"), float(sm_scale),
                                       _ptr(O, torch.bfloat16, "O"), _ptr(lse, torch.float32, "lse"),
                                       _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def swa_attn_decode(Q, kv: KV, q_pos, window: int, sink, sm_scale: float, O, lse=None, ws=None, stream=None):
    B, T = _bt(Q, (64, 192), "Q")
    _check(_lib.swa_attn_decode(_ptr(Q, torch.bfloat16, "Q"), kv.ref, _ptr(q_pos, torch.int32, "q_pos"), B, T,
                                int(window), _ptr(sink, torch.float32, "sink"), float(sm_scale),
                                _ptr(O, torch.bfloat16, "O"), _ptr(lse, torch.float32, "lse"),
                                _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def dsa_layer_decode(q8, q_scale, w, Q, kv: KV, q_pos, Lmax: int, top_k: int, sink, sm_scale: float, O, lse=None,
                     idx_out=None, count_out=None, ws=None, stream=None, stage_events=None):
    B, T = _bt(q8, (16, 128), "q8")
    ev = None
    if stage_events is not None:
        arr = (ctypes.c_void_p * 5)(*[ctypes.c_void_p(e.cuda_event) if e is not None else None
                                      for e in stage_events])
        ev = ctypes.cast(arr, P)
    _check(_lib.dsa_layer_decode(_ptr(q8, torch.uint8, "q8"), _ptr(q_scale, torch.float32, "q_scale"),
                                 _ptr(w, torch.float32, "w"), _ptr(Q, torch.bfloat16, "Q"), kv.ref,
                                 _ptr(q_pos, torch.int32, "q_pos"), B, T, int(Lmax), int(top_k),
                                 _ptr(sink, torch.float32, "sink"), float(sm_scale), _ptr(O, torch.bfloat16, "O"),
                                 _ptr(lse, torch.float32, "lse"), _ptr(idx_out, torch.int32, "idx_out"),
                                 _ptr(count_out, torch.int32, "count_out"), _ptr(ws, torch.uint8, "ws"),
                                 ws.numel(), _stream(stream), ev))


def dsa_prefill(q8, q_scale, w, Q, kv: KV, q_pos, Lmax: int, top_k: int, sink, sm_scale: float, O, lse=None,
                idx_out=None, count_out=None, ws=None, stream=None):
    """NQ query tokens of one sequence: q8 [NQ, 16, 128], Q [NQ, 64, 192], q_pos [NQ], O [NQ, 64, 128]."""
    if q8.dim() != 3 or tuple(q8.shape[1:]) != (16, 128):
        raise ValueError("q8 must be [NQ, 16, 128]")
    NQ = int(q8.shape[0])
    _check(_lib.dsa_prefill(_ptr(q8, torch.uint8, "q8"), _ptr(q_scale, torch.float32, "q_scale"),
                            _ptr(w, torch.float32, "w"), _ptr(Q, torch.bfloat16, "Q"), kv.ref,
                            _ptr(q_pos, torch.int32, "q_pos"), NQ, int(Lmax), int(top_k),
                            _ptr(sink, torch.float32, "sink"), float(sm_scale), _ptr(O, torch.bfloat16, "O"),
                            _ptr(lse, torch.float32, "lse"), _ptr(idx_out, torch.int32, "idx_out"),
                            _ptr(count_out, torch.int32, "count_out"), _ptr(ws, torch.uint8, "ws"),
                            ws.numel(), _stream(stream)))


def swa_step(Q, kv: "KV", q_pos, window: int, sink, sm_scale: float, O, lse=None, ws=None) -> dict:
    """A sliding-window layer-step of a chain (arguments as swa_attn_decode)."""
    B, T = _bt(Q, (64, 192), "Q")
    return dict(kind=STEP_SWA, B=B, T=T, top_k=int(window), Lmax=0, q8=None, q_scale=None, w=None,
                Q=_ptr(Q, torch.bfloat16, "Q"), kv=kv, q_pos=_ptr(q_pos, torch.int32, "q_pos"),
                sink=_ptr(sink, torch.float32, "sink"), sm_scale=float(sm_scale), O=_ptr(O, torch.bfloat16, "O"),
                lse=_ptr(lse, torch.float32, "lse"), idx_out=None, count_out=None, ws=_ptr(ws, torch.uint8, "ws"),
                ws_bytes=ws.numel())


def dsa_step(q8, q_scale, w, Q, kv: "KV", q_pos, Lmax: int, top_k: int, sink, sm_scale: float, O, lse=None,
             idx_out=None, count_out=None, ws=None) -> dict:
    """A DSA layer-step of a chain (arguments as dsa_layer_decode)."""
    B, T = _bt(q8, (16, 128), "q8")
    return dict(kind=STEP_DSA, B=B, T=T, top_k=int(top_k), Lmax=int(Lmax), q8=_ptr(q8, torch.uint8, "q8"),
                q_scale=_ptr(q_scale, torch.float32, "q_scale"), w=_ptr(w, torch.float32, "w"),
                Q=_ptr(Q, torch.bfloat16, "Q"), kv=kv, q_pos=_ptr(q_pos, torch.int32, "q_pos"),
                sink=_ptr(sink, torch.float32, "sink"), sm_scale=float(sm_scale), O=_ptr(O, torch.bfloat16, "O"),
                lse=_ptr(lse, torch.float32, "lse"), idx_out=_ptr(idx_out, torch.int32, "idx_out"),
                count_out=_ptr(count_out, torch.int32, "count_out"), ws=_ptr(ws, torch.uint8, "ws"),
                ws_bytes=ws.numel())


def dsa_layer_chain(steps, stream=None):
    """Enqueue the steps (swa_step / dsa_step dicts) as one chained sequence."""
    arr = (dsa_layer_step_t * len(steps))()
    keep = []
    for i, st in enumerate(steps):
        for k, v in st.items():
            if k == "kv":
                keep.append(v)
                arr[i].kv = ctypes.cast(ctypes.pointer(v.struct), ctypes.c_void_p)
            else:
                setattr(arr[i], k, v.value if isinstance(v, ctypes.c_void_p) else v)
    _check(_lib.dsa_layer_chain(ctypes.cast(arr, P), len(steps), _stream(stream)))


# ------------------------------------------------- context-sharded decode
def dsa_shard_positions(q_pos, shard_offset: int, shard_len: int, q_pos_local, ws, stream=None):
    B, T = q_pos.shape
    _check(_lib.dsa_shard_positions(_ptr(q_pos, torch.int32, "q_pos"), B, T, int(shard_offset), int(shard_len),
                                    _ptr(q_pos_local, torch.int32, "q_pos_local"), _ptr(ws, torch.uint8, "ws"),
                                    ws.numel(), _stream(stream)))


def dsa_shard_candidates(scores, idx, top_k: int, shard_offset: int, cand_score, cand_pos, stream=None):
    B, T = idx.shape[:2]
    _check(_lib.dsa_shard_candidates(_ptr(scores, torch.float32, "scores"), scores.shape[-1],
                                     _ptr(idx, torch.int32, "idx"), B, T, int(top_k), int(shard_offset),
                                     _ptr(cand_score, torch.float32, "cand_score"),
                                     _ptr(cand_pos, torch.int32, "cand_pos"), _stream(stream)))


def dsa_shard_merge(cand_score_all, cand_pos_all, top_k: int, shard_offset: int, shard_len: int, idx_out, count_out,
                    local_idx=None, local_count=None, stream=None):
    N, B, T = cand_pos_all.shape[:3]
    _check(_lib.dsa_shard_merge(_ptr(cand_score_all, torch.float32, "cand_score_all"),
                                _ptr(cand_pos_all, torch.int32, "cand_pos_all"), N, B, T, int(top_k),
                                int(shard_offset), int(shard_len), _ptr(idx_out, torch.int32, "idx_out"),
                                _ptr(count_out, torch.int32, "count_out"), _ptr(local_idx, torch.int32, "local_idx"),
                                _ptr(local_count, torch.int32, "local_count"), _stream(stream)))


def dsa_shard_combine(O_all, lse_all, sink, O, lse=None, stream=None):
    N, B, T = lse_all.shape[:3]
    _check(_lib.dsa_shard_combine(_ptr(O_all, torch.bfloat16, "O_all"), _ptr(lse_all, torch.float32, "lse_all"), N, B,
                                  T, _ptr(sink, torch.float32, "sink"), _ptr(O, torch.bfloat16, "O"),
                                  _ptr(lse, torch.float32, "lse"), _stream(stream)))
