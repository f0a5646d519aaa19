"""ctypes marshalling for oracle.c (test infrastructure only; see __init__)."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (plain -O2; OpenMP for the
    loops over positions and heads, one thread unless set_threads says more)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        P = ctypes.c_void_p
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_fp8_dot.restype = ctypes.c_double
        lib.oracle_fp8_dot.argtypes = [P, P, ctypes.c_int]
        lib.oracle_indexer_scores.restype = None
        lib.oracle_indexer_scores.argtypes = [P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int64, P]
        lib.oracle_topk.restype = ctypes.c_int
        lib.oracle_topk.argtypes = [P, ctypes.c_int64, ctypes.c_int, P]
        lib.oracle_topk_select.restype = ctypes.c_int
        lib.oracle_topk_select.argtypes = [P, ctypes.c_int64, ctypes.c_int, P]
        lib.oracle_gqa_attention.restype = None
        lib.oracle_gqa_attention.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P,
                                             ctypes.c_double, P, P]
        lib.oracle_swa_indices.restype = ctypes.c_int
        lib.oracle_swa_indices.argtypes = [ctypes.c_int64, ctypes.c_int, P]
        lib.oracle_layernorm.restype = None
        lib.oracle_layernorm.argtypes = [P, ctypes.c_int, P, P, ctypes.c_double, P]
        lib.oracle_rope_partial.restype = None
        lib.oracle_rope_partial.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_double]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_index_k_produce.restype = ctypes.c_float
        lib.oracle_index_k_produce.argtypes = [P, P, P, ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                               ctypes.c_int64, P, P]
        lib.oracle_index_q_produce.restype = ctypes.c_float
        lib.oracle_index_q_produce.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                               ctypes.c_int64, P, P]
        lib.oracle_indexer_kl.restype = ctypes.c_double
        lib.oracle_indexer_kl.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, ctypes.c_int64,
                                          ctypes.c_double, P]
        lib.oracle_set_threads.restype = None
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_set_threads(1)   # one thread unless asked (results do not depend on it)
        _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> int:
    """Host threads for the position / head loops; returns the count in use."""
    lib = _load()
    lib.oracle_set_threads(int(n))
    return lib.oracle_max_threads()


def e4m3_to_float64(codes) -> np.ndarray:
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib.oracle_e4m3_to_double(i) for i in range(256)], dtype=np.float64)
    return table[codes]


def bf16_to_float64(bits) -> np.ndarray:
    lib = _load()
    bits = np.asarray(bits, dtype=np.uint16)
    flat = bits.reshape(-1)
    out = np.array([lib.oracle_bf16_to_double(int(b)) for b in flat], dtype=np.float64)
    return out.reshape(bits.shape)


def fp8_dot(a, b) -> float:
    lib = _load()
    a, pa = _c(a, np.uint8)
    b, pb = _c(b, np.uint8)
    assert a.shape == b.shape and a.ndim == 1
    return lib.oracle_fp8_dot(pa, pb, a.shape[0])


def indexer_scores(q8, q_scale, w, k8, k_scale, q_pos) -> np.ndarray:
    """Scores [T, L] for one sequence; q8 [T,H,D], k8 [L,D], q_pos [T]."""
    lib = _load()
    q8, pq = _c(q8, np.uint8)
    T, H, D = q8.shape
    q_scale, pqs = _c(np.broadcast_to(q_scale, (T, H)), np.float32)
    w, pw = _c(np.broadcast_to(w, (T, H)), np.float32)
    k8, pk = _c(k8, np.uint8)
    L = k8.shape[0]
    assert k8.shape[1] == D
    k_scale, pks = _c(k_scale, np.float32)
    q_pos, pp = _c(q_pos, np.int32)
    out = np.empty((T, L), dtype=np.float32)
    lib.oracle_indexer_scores(pq, pqs, pw, pk, pks, pp, T, H, D, L,
                              out.ctypes.data_as(ctypes.c_void_p))
    return out


def topk(scores, k: int):
    """(idx[k] int32 with -1 padding, count) over the visible scores."""
    lib = _load()
    s, ps = _c(scores, np.float32)
    idx = np.empty(k, dtype=np.int32)
    cnt = lib.oracle_topk(ps, s.shape[0], k, idx.ctypes.data_as(ctypes.c_void_p))
    return idx, cnt


def topk_select(scores, k: int):
    lib = _load()
    s, ps = _c(scores, np.float32)
    idx = np.empty(k, dtype=np.int32)
    cnt = lib.oracle_topk_select(ps, s.shape[0], k, idx.ctypes.data_as(ctypes.c_void_p))
    return idx, cnt


def gqa_attention(Q, K, V, idx, sink, sm_scale: float):
    """One query token. Q [H,Dk] bf16 bits (uint16); K [L,G,Dk]; V [L,G,Dv];
    idx [n] positions; sink [H] float or None.  Returns (out [H,Dv], lse [H])."""
    lib = _load()
    Q, pQ = _c(Q, np.uint16)
    K = np.asarray(K)
    V = np.asarray(V)
    assert K.dtype == np.uint16 and V.dtype == np.uint16
    if not K.flags.c_contiguous:
        K = np.ascontiguousarray(K)
    if not V.flags.c_contiguous:
        V = np.ascontiguousarray(V)
    H, Dk = Q.shape
    L, G, Dk2 = K.shape
    assert Dk2 == Dk and V.shape[:2] == (L, G)
    Dv = V.shape[2]
    idx, pidx = _c(idx, np.int32)
    assert idx.size == 0 or (idx.min() >= 0 and idx.max() < L)
    if sink is None:
        psink = None
    else:
        sink, psink = _c(sink, np.float32)
    out = np.empty((H, Dv), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    lib.oracle_gqa_attention(pQ, K.ctypes.data_as(ctypes.c_void_p),
                             V.ctypes.data_as(ctypes.c_void_p), L, H, G, Dk, Dv, pidx,
                             idx.shape[0], psink, float(sm_scale),
                             out.ctypes.data_as(ctypes.c_void_p),
                             lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def swa_indices(p: int, window: int) -> np.ndarray:
    lib = _load()
    idx = np.empty(max(window, 1), dtype=np.int32)
    n = lib.oracle_swa_indices(int(p), int(window), idx.ctypes.data_as(ctypes.c_void_p))
    return idx[:n].copy()


def dsa_layer_decode(q8, q_scale, w, k8, k_scale, Q, K, V, q_pos, top_k, sink, sm_scale):
    """One sequence, T query tokens: indexer -> top-k -> sparse attention.

    q8 [T,16,128]; q_scale, w [T,16]; k8 [L,128]; k_scale [L]; Q [T,H,Dk];
    K [L,G,Dk]; V [L,G,Dv]; q_pos [T].  Returns dict with scores [T,L],
    idx [T,top_k], count [T], out [T,H,Dv] (float64), lse [T,H].
    """
    q_pos = np.asarray(q_pos, dtype=np.int32)
    T = q_pos.shape[0]
    scores = indexer_scores(q8, q_scale, w, k8, k_scale, q_pos)
    idx = np.full((T, top_k), -1, dtype=np.int32)
    count = np.zeros(T, dtype=np.int32)
    H, Dv = Q.shape[1], V.shape[2]
    out = np.zeros((T, H, Dv), dtype=np.float64)
    lse = np.zeros((T, H), dtype=np.float64)
    for t in range(T):
        n = int(q_pos[t]) + 1
        idx[t], count[t] = topk(scores[t, :n], top_k)
        out[t], lse[t] = gqa_attention(Q[t], K, V, idx[t, :count[t]], sink, sm_scale)
    return dict(scores=scores, idx=idx, count=count, out=out, lse=lse)


def swa_layer_decode(Q, K, V, q_pos, window, sink, sm_scale):
    """One sequence, T query tokens of sliding-window attention."""
    q_pos = np.asarray(q_pos, dtype=np.int32)
    T = q_pos.shape[0]
    H, Dv = Q.shape[1], V.shape[2]
    out = np.zeros((T, H, Dv), dtype=np.float64)
    lse = np.zeros((T, H), dtype=np.float64)
    for t in range(T):
        idx = swa_indices(int(q_pos[t]), window)
        out[t], lse[t] = gqa_attention(Q[t], K, V, idx, sink, sm_scale)
    return dict(out=out, lse=lse)


# ------------------------------------------------ index-K / index-Q producer
def layernorm(x, w, b, eps: float) -> np.ndarray:
    lib = _load()
    x, px = _c(x, np.float64)
    w, pw = _c(w, np.float32)
    b, pb = _c(b, np.float32)
    y = np.empty_like(x)
    lib.oracle_layernorm(px, x.shape[0], pw, pb, float(eps), y.ctypes.data_as(ctypes.c_void_p))
    return y


def rope_partial(x, rot: int, pos: int, base: float) -> np.ndarray:
    lib = _load()
    y = np.ascontiguousarray(x, dtype=np.float64).copy()
    lib.oracle_rope_partial(y.ctypes.data_as(ctypes.c_void_p), y.shape[0], int(rot), int(pos), float(base))
    return y


def e4m3_encode(v) -> np.ndarray:
    lib = _load()
    v = np.asarray(v, dtype=np.float32)
    return np.array([lib.oracle_e4m3_encode(float(x)) for x in v.reshape(-1)], dtype=np.uint8).reshape(v.shape)


def index_k_produce(k_bits, ln_w, ln_b, eps: float, rot: int, base: float, pos: int):
    """One token's index key: bf16 bits k [D] -> (codes [D] uint8, scale, y [D] before quantisation)."""
    lib = _load()
    k, pk = _c(k_bits, np.uint16)
    w, pw = _c(ln_w, np.float32)
    b, pb = _c(ln_b, np.float32)
    D = k.shape[0]
    codes = np.empty(D, np.uint8)
    y = np.empty(D, np.float64)
    s = lib.oracle_index_k_produce(pk, pw, pb, float(eps), D, int(rot), float(base), int(pos),
                                   codes.ctypes.data_as(ctypes.c_void_p), y.ctypes.data_as(ctypes.c_void_p))
    return codes, float(np.float32(s)), y


def index_q_produce(q_bits, rot: int, base: float, pos: int):
    """One token's index query: bf16 bits q [H, D] -> (codes [H, D], scale, y [H, D])."""
    lib = _load()
    q, pq = _c(q_bits, np.uint16)
    H, D = q.shape
    codes = np.empty((H, D), np.uint8)
    y = np.empty((H, D), np.float64)
    s = lib.oracle_index_q_produce(pq, H, D, int(rot), float(base), int(pos),
                                   codes.ctypes.data_as(ctypes.c_void_p), y.ctypes.data_as(ctypes.c_void_p))
    return codes, float(np.float32(s)), y


# ------------------------------------------------ indexer warm-up KL target
def indexer_kl(Q_bits, K_bits, I, p: int, sm_scale: float):
    """One query token at position p: Q [H, Dk] bf16 bits, K [L, G, Dk] bf16
    bits (rows 0..p visible), I [>= p + 1] indexer scores.  Returns (KL, P [p + 1])."""
    lib = _load()
    Q, pQ = _c(Q_bits, np.uint16)
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    H, Dk = Q.shape
    G = K.shape[1]
    I, pI = _c(np.asarray(I)[: p + 1], np.float32)
    P = np.empty(p + 1, np.float64)
    kl = lib.oracle_indexer_kl(pQ, K.ctypes.data_as(ctypes.c_void_p), H, G, Dk, pI, int(p), float(sm_scale),
                               P.ctypes.data_as(ctypes.c_void_p))
    return float(kl), P
