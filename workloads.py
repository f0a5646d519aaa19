"""Seeded synthetic inputs for the DSA / SWA decode layer-step.

This module only draws random numbers and lays them out; it holds none of the
layer-step's arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle
consume the tensors it returns.  Shapes and distributions follow the decode
workloads described for the hybrid SWA + DSA model (index heads 16 x 128 with
one shared key head in fp8_e4m3, 64 query heads with qk dim 192 and v dim 128,
GQA4 on DSA layers and GQA8 on SWA layers, top-2,048 selection, window 128,
native context 1,048,576):

* indexer query q [B,T,16,128] and key k [rows,128] ~ N(0,1), each quantised to
  e4m3 with a per-token fp32 scale amax/448 (scale 1 for an all-zero token),
  round-to-nearest-even, saturating at +-448; the query scale is stored per
  (token, head) by broadcasting the per-token value;
* head weights w ~ U(0,1)/16;
* backbone Q [B,T,64,192], K [rows,G,192], V [rows,G,128] ~ N(0,1)/sqrt(192)
  (``qk_std`` overrides the Q/K standard deviation for peaked-attention cases),
  stored as bf16;
* per-head sink logits ~ N(0,1);
* planted "needles": indexer keys set, before quantisation, to the direction
  of the sequence's first query token's head-0 index query, scaled to norm
  sqrt(128); placed uniformly or Zipf(1)-distributed by distance from the end;
* decode queries occupy the last T positions of each sequence: 0-based
  p_t = L - T + t.

Random numbers come from a torch.Generator seeded with ``seed`` on the device
the tensors are made on, so a workload is identified by (recipe, seed, device).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

E4M3_MAX = 448.0
INDEX_HEADS = 16
INDEX_DIM = 128
Q_HEADS = 64
QK_DIM = 192
V_DIM = 128


def quantize_e4m3_rows(x: torch.Tensor):
    """Per-row e4m3 quantisation of x [..., D] -> (codes uint8 [..., D], scale f32 [...])."""
    amax = x.abs().amax(dim=-1).float()
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x.float() / scale.unsqueeze(-1)).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


@dataclass
class KVLayout:
    """Where the rows of each sequence live.

    contiguous: row(b, pos) = b * seq_stride + pos
    paged:      row(b, pos) = block_table[b, pos // page_size] * page_size + pos % page_size
    """
    seq_lens: list
    seq_stride: int = 0
    page_size: int = 0
    block_table: Optional[torch.Tensor] = None   # int32 [B, max_pages]
    num_rows: int = 0

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    def rows(self, b: int, pos: torch.Tensor) -> torch.Tensor:
        if not self.paged:
            return b * self.seq_stride + pos
        bt = self.block_table[b].to(pos.device).long()
        return bt[pos // self.page_size] * self.page_size + pos % self.page_size


def make_layout(seq_lens, page_size: int = 0, seed: int = 0, device="cpu") -> KVLayout:
    seq_lens = [int(x) for x in seq_lens]
    B = len(seq_lens)
    if page_size <= 0:
        stride = max(seq_lens) if B == 1 else -(-max(seq_lens) // 128) * 128
        return KVLayout(seq_lens=seq_lens, seq_stride=stride, num_rows=B * stride)
    pages = [math.ceil(L / page_size) for L in seq_lens]
    total = sum(pages)
    g = torch.Generator(device="cpu").manual_seed(seed + 7919)
    perm = torch.randperm(total, generator=g).to(torch.int32)
    max_pages = max(pages)
    bt = torch.zeros((B, max_pages), dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    return KVLayout(seq_lens=seq_lens, page_size=page_size, block_table=bt.to(device),
                    num_rows=total * page_size)


@dataclass
class DecodeWorkload:
    layout: KVLayout
    q_pos: torch.Tensor          # int32 [B, T]
    q8: torch.Tensor             # uint8 [B, T, 16, 128]
    q_scale: torch.Tensor        # f32   [B, T, 16]
    w: torch.Tensor              # f32   [B, T, 16]
    k8: torch.Tensor             # uint8 [rows, 128]
    k_scale: torch.Tensor        # f32   [rows]
    Q: torch.Tensor              # bf16  [B, T, 64, 192]
    K: torch.Tensor              # bf16  [rows, G, 192]
    V: torch.Tensor              # bf16  [rows, G, 128]
    sink: torch.Tensor           # f32   [64]
    needles: list = field(default_factory=list)   # per sequence: int64 positions
    G: int = 4

    @property
    def B(self):
        return self.q_pos.shape[0]

    @property
    def T(self):
        return self.q_pos.shape[1]


def _needle_positions(g: torch.Generator, L: int, n: int, mode: str) -> torch.Tensor:
    n = min(n, L)
    if n <= 0:
        return torch.zeros(0, dtype=torch.int64)
    if mode == "uniform":
        return torch.randperm(L, generator=g)[:n].sort().values
    if mode == "zipf":
        # distance from the end r in [1, L] with P(r) ~ 1/r; duplicates resampled
        # continuous inverse CDF of P(r) ~ 1/r on [1, L]: r = L^u
        chosen = set()
        while len(chosen) < n:
            u = torch.rand(4 * n, generator=g, dtype=torch.float64)
            r = torch.exp(u * math.log(L)).floor().clamp(1, L).long()
            for v in r.tolist():
                if len(chosen) < n:
                    chosen.add(L - v)
        return torch.tensor(sorted(chosen), dtype=torch.int64)
    raise ValueError(mode)


def make_decode_workload(seed: int, seq_lens, T: int = 1, G: int = 4, n_needles: int = 0,
                         needle_mode: str = "uniform", page_size: int = 0,
                         device="cpu", qk_std: Optional[float] = None) -> DecodeWorkload:
    """A batch of B = len(seq_lens) decode sequences with T query tokens each."""
    device = torch.device(device)
    layout = make_layout(seq_lens, page_size=page_size, seed=seed, device=device)
    B = len(layout.seq_lens)
    g = torch.Generator(device=device).manual_seed(seed)
    gc = torch.Generator(device="cpu").manual_seed(seed + 1)
    rows = layout.num_rows

    q = torch.randn((B, T, INDEX_HEADS, INDEX_DIM), generator=g, device=device)
    q_codes, q_tok_scale = quantize_e4m3_rows(q.reshape(B, T, INDEX_HEADS * INDEX_DIM))
    q8 = q_codes.reshape(B, T, INDEX_HEADS, INDEX_DIM).contiguous()
    q_scale = q_tok_scale.unsqueeze(-1).expand(B, T, INDEX_HEADS).contiguous()
    w = (torch.rand((B, T, INDEX_HEADS), generator=g, device=device) / 16.0).contiguous()

    k = torch.randn((rows, INDEX_DIM), generator=g, device=device)
    needles = []
    for b, L in enumerate(layout.seq_lens):
        pos = _needle_positions(gc, L, n_needles, needle_mode)
        needles.append(pos)
        if pos.numel():
            d = q[b, 0, 0]
            d = d / d.norm() * math.sqrt(INDEX_DIM)
            k[layout.rows(b, pos.to(device))] = d
    k8, k_scale = quantize_e4m3_rows(k)
    del k

    std = qk_std if qk_std is not None else 1.0 / math.sqrt(QK_DIM)
    vstd = 1.0 / math.sqrt(QK_DIM)
    Q = (torch.randn((B, T, Q_HEADS, QK_DIM), generator=g, device=device) * std).to(torch.bfloat16)
    K = torch.empty((rows, G, QK_DIM), dtype=torch.bfloat16, device=device)
    V = torch.empty((rows, G, V_DIM), dtype=torch.bfloat16, device=device)
    step = 1 << 18
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        K[r0:r1] = (torch.randn((r1 - r0, G, QK_DIM), generator=g, device=device) * std).to(torch.bfloat16)
        V[r0:r1] = (torch.randn((r1 - r0, G, V_DIM), generator=g, device=device) * vstd).to(torch.bfloat16)
    sink = torch.randn((Q_HEADS,), generator=g, device=device).float()

    q_pos = torch.tensor([[L - T + t for t in range(T)] for L in layout.seq_lens],
                         dtype=torch.int32, device=device)
    return DecodeWorkload(layout=layout, q_pos=q_pos, q8=q8, q_scale=q_scale, w=w, k8=k8,
                          k_scale=k_scale, Q=Q, K=K, V=V, sink=sink, needles=needles, G=G)


def log_uniform_lengths(seed: int, B: int, lo: int, hi: int) -> list:
    g = torch.Generator(device="cpu").manual_seed(seed + 104729)
    u = torch.rand(B, generator=g, dtype=torch.float64)
    return [int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo))))) for x in u]


# ---------------------------------------------------------------- recipes
# The five workloads: tiny decode, speculative-verify block at 65,536, native
# 1,048,576 context, a ragged paged batch, and a chunked prefill.
CONFIGS = {
    "tiny_8k": dict(seed=0, seq_lens=[8192], T=1, n_needles=16, needle_mode="uniform"),
    "verify_64k_t4": dict(seed=1, seq_lens=[65536], T=4, n_needles=64, needle_mode="uniform"),
    "ctx_1m": dict(seed=2, seq_lens=[1048576], T=1, n_needles=256, needle_mode="zipf"),
}


def ragged_batch_lengths(seed: int = 3, B: int = 64):
    return log_uniform_lengths(seed, B, 4096, 262144)


# The ragged serving batch: 64 sequences, contexts log-uniform in
# [4,096, 262,144], paged caches with 64-position pages.  One "mix" is the
# five SWA layer-steps and one DSA layer-step the layer pattern repeats.
CONFIGS["ragged_b64"] = dict(seed=3, seq_lens=ragged_batch_lengths(3, 64), T=1, page_size=64, n_needles=4,
                             needle_mode="uniform")


# The chunked prefill: the last 8,192 positions (1,040,384..1,048,575) of a
# 1,048,576-token context, each query token attending causally.
CONFIGS["prefill_8k_1m"] = dict(seed=4, seq_lens=[1048576], T=8192, n_needles=256, needle_mode="zipf")


def make_swa_window_workload(seed: int, seq_lens, window: int = 128, page_size: int = 64, G: int = 8,
                             device="cpu") -> DecodeWorkload:
    """An SWA layer's decode inputs for sequences of the given lengths, T = 1.

    Only the pages that hold the last `window` positions of each sequence are
    allocated (the rest of the block table is -1): an SWA layer never reads
    further back.  Q ~ N(0,1)/sqrt(192) and K, V ~ N(0,1)/sqrt(192) bf16, sink
    ~ N(0,1), as for the DSA layers; no index keys."""
    device = torch.device(device)
    seq_lens = [int(x) for x in seq_lens]
    B = len(seq_lens)
    g = torch.Generator(device=device).manual_seed(seed)
    gc = torch.Generator(device="cpu").manual_seed(seed + 7919)
    max_pages = max(math.ceil(L / page_size) for L in seq_lens)
    bt = torch.full((B, max_pages), -1, dtype=torch.int32)
    first = [max(0, L - window) // page_size for L in seq_lens]
    last = [(L - 1) // page_size for L in seq_lens]
    total = sum(l - f + 1 for f, l in zip(first, last))
    perm = torch.randperm(total, generator=gc).to(torch.int32)
    off = 0
    for b in range(B):
        n = last[b] - first[b] + 1
        bt[b, first[b]:last[b] + 1] = perm[off:off + n]
        off += n
    layout = KVLayout(seq_lens=seq_lens, page_size=page_size, block_table=bt.to(device), num_rows=total * page_size)
    rows = layout.num_rows
    std = 1.0 / math.sqrt(QK_DIM)
    Q = (torch.randn((B, 1, Q_HEADS, QK_DIM), generator=g, device=device) * std).to(torch.bfloat16)
    K = (torch.randn((rows, G, QK_DIM), generator=g, device=device) * std).to(torch.bfloat16)
    V = (torch.randn((rows, G, V_DIM), generator=g, device=device) * std).to(torch.bfloat16)
    sink = torch.randn((Q_HEADS,), generator=g, device=device).float()
    q_pos = torch.tensor([[L - 1] for L in seq_lens], dtype=torch.int32, device=device)
    empty8 = torch.empty((0,), dtype=torch.uint8, device=device)
    emptyf = torch.empty((0,), dtype=torch.float32, device=device)
    return DecodeWorkload(layout=layout, q_pos=q_pos, q8=empty8, q_scale=emptyf, w=emptyf, k8=empty8,
                          k_scale=emptyf, Q=Q, K=K, V=V, sink=sink, needles=[], G=G)


# ---------------------------------------------------------------- views
def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def logical_rows(wl: DecodeWorkload, b: int, L: Optional[int] = None) -> torch.Tensor:
    """Row indices of positions 0..L-1 of sequence b (int64, on the layout's device)."""
    L = wl.layout.seq_lens[b] if L is None else L
    dev = wl.k8.device
    return wl.layout.rows(b, torch.arange(L, device=dev))
