"""Benchmark: one DSA decode layer-step at the native 1,048,576-token context.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path (lightning indexer over every cached
key -> top-2048 selection -> sparse GQA4 attention with sink -> split combine)
for batch 1, one query token, context 1,048,576, on synthetic seeded inputs.
Each rank runs its own replica of the workload (the steps are independent
problems: weak scaling, no data-path collective); ``value`` is the tokens all
ranks decoded divided by the slowest rank's device time.

L2 is flushed between timed steps, outside the timed events: a 256 MB write
evicts everything, then a 256 MB read retires the dirty lines, so each step
starts cold and clean.
Per-stage CUDA events recorded by the library itself give the indexer's
duration for the roofline.  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA layer-step µs & tok/s at 1M ctx; indexer HBM GB/s vs B200 peak"
WORKLOAD = "ctx_1m"
L_CTX = 1048576
TOP_K = 2048
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "local_attention_decode_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_ctx_1m.txt")
FUSED_MAX_ROWS = 16   # dsa_layer_decode runs as one fused kernel for B * T <= 16


WORKLOAD_DESC = {
    "ctx_1m": "ctx_1m: DSA decode layer-step, batch 1, 1 query token at position 1,048,575, context 1,048,576, "
              "top-2048, 64 Q heads / 4 KV heads (GQA4), qk 192, v 128, sink, 256 Zipf needles",
    "verify_64k_t4": "verify_64k_t4: DSA decode layer-step, batch 1, 4 query tokens (speculative verify block) at "
                     "positions 65,532..65,535, context 65,536, top-2048, GQA4, sink, 64 needles",
    "tiny_8k": "tiny_8k: DSA decode layer-step, batch 1, 1 query token, context 8,192, top-2048, GQA4, sink, "
               "16 needles",
    "prefill_8k_1m": "prefill_8k_1m: DSA layer over 8,192 query tokens at positions 1,040,384..1,048,575 of a "
                     "1,048,576-token context, causal, top-2048 each, GQA4, sink, 256 Zipf needles",
    "ragged_b64_mix": "ragged_b64_mix: 64 sequences, 1 query token each, contexts log-uniform in [4,096, 262,144] "
                      "(seed 3), paged caches (64-position pages); one mix = 5 SWA layer-steps (window 128, GQA8, "
                      "window-only caches) + 1 DSA layer-step (top-2048, GQA4, sink)",
}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def indexer_bytes(L: int, T: int) -> int:
    """Algorithmic bytes of one indexer launch for one sequence: every visible
    key read once (128 B of e4m3 codes + 4 B scale), one fp32 score written per
    (query token, key), and the query block (T x (2 KiB codes + 128 B of
    scales and weights))."""
    return L * (128 + 4) + T * L * 4 + T * (16 * 128 + 16 * 8)


def gathered_bytes(T: int, top_k: int, G: int = 4) -> int:
    """Backbone K/V bytes gathered by the sparse attention: top_k rows of G heads x (192 + 128) bf16."""
    return T * top_k * G * (192 + 128) * 2


def _strip_comments(src: str) -> str:
    """C/C++ source without its comments and trailing blanks (string literals
    in these sources contain no comment markers)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_sources_sha() -> str:
    """Hash of the code (comments excluded) of the CUDA sources the timed
    kernels are built from."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            h.update(_strip_comments(open(os.path.join(CSRC, name)).read()).encode())
    return h.hexdigest()


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken on the current kernel sources; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        if d.get("sources_sha256") == kernel_sources_sha() and kernel in d.get("kernels", {}):
            return int(d["kernels"][kernel]["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, bit in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def start(self):
        if self.nv is not None:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.nv is not None:
            self._stop.set()
            if self._t:
                self._t.join()
            self._sample()
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


class L2Flush:
    """Leaves L2 cold and clean between timed steps: write a 256 MB buffer (evicts
    everything), then read another 256 MB buffer so the write-backs of the dirty
    lines happen here, not inside the next timed step."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.w.zero_()
        self.out.copy_(self.r.sum())


# ------------------------------------------------------- multi-rank helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), ws, int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def throughput(tokens_per_rank_step: int, steps: int, world: int, slowest_s: float) -> float:
    """Whole-job tokens per second: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank_step * steps * world / slowest_s


def read_stream_gbps(torch, dev, stream) -> float:
    """Read-only HBM stream rate on this GPU now: a reduction over 1 GiB of
    fp32 (larger than L2), best of 6, timed with CUDA events."""
    x = torch.ones(1 << 28, dtype=torch.float32, device=dev)
    out = torch.empty((), dtype=torch.float32, device=dev)
    best = None
    for _ in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        out.copy_(x.sum())
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    del x
    return (1 << 30) / (best / 1e3) / 1e9


def decode_config(workload: str, world: int, layers: int = 1) -> dict:
    """The `config` object of a decode workload's line (both arms)."""
    from workloads import CONFIGS
    cfg = CONFIGS[workload]
    return {
        "workload": WORKLOAD_DESC[workload],
        "batch": len(cfg["seq_lens"]), "query_tokens": cfg["T"], "context": max(cfg["seq_lens"]), "top_k": TOP_K,
        "seed": cfg["seed"], "needles": cfg["n_needles"], "parallelism": f"replicas x{world}",
        "layers_in_rotation": layers,
        "l2": (f"inputs larger than L2: {layers} layers' caches in rotation, steps back to back, no flush"
               if layers > 1 else
               "flushed between steps outside the timed events (256 MB write, then 256 MB read so no dirty lines remain)"),
    }


# ------------------------------------------------------ the ragged batch mix
MIX_METRIC = "ragged 64-sequence decode layer-mix (5 SWA + 1 DSA layer-steps) tok/s"


def run_mix(args, rank, world, local_rank):
    """One step = the layer pattern's repeating mix over the ragged serving
    batch: five SWA layer-steps (each on its own window-only paged cache) and
    one DSA layer-step (dsa_layer_decode, 64 rows: separate kernels), all 64
    sequences one token each.  L2 flushed before each mix."""
    import torch
    import local_attention_decode_b200 as dsa
    from workloads import CONFIGS, make_decode_workload, make_swa_window_workload

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = CONFIGS["ragged_b64"]
    wl = make_decode_workload(device=dev, **cfg)
    lens = wl.layout.seq_lens
    B = wl.B
    Lmax = max(lens)
    sm_scale = 1.0 / math.sqrt(192)
    kv = dsa.KV(k=wl.K, v=wl.V, index_k=wl.k8, index_k_scale=wl.k_scale, num_kv_heads=wl.G,
                block_table=wl.layout.block_table, page_size=wl.layout.page_size, num_rows=wl.layout.num_rows)
    swa = [make_swa_window_workload(100 + i, lens, device=dev) for i in range(5)]
    swa_kv = [dsa.KV(k=s.K, v=s.V, num_kv_heads=s.G, block_table=s.layout.block_table,
                     page_size=s.layout.page_size, num_rows=s.layout.num_rows) for s in swa]
    O = torch.empty((B, 1, 64, 128), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((B, 1, TOP_K), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, 1), dtype=torch.int32, device=dev)
    ws = dsa.alloc_workspace(dsa.OP_LAYER, B, 1, Lmax, TOP_K, device=dev)
    ws_swa = dsa.alloc_workspace(dsa.OP_SWA_ATTN, B, 1, 1, 128, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step(stage=None):
        for s, k in zip(swa, swa_kv):
            dsa.swa_attn_decode(s.Q, k, s.q_pos, 128, s.sink, sm_scale, O, None, ws_swa)
        dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, Lmax, TOP_K, wl.sink, sm_scale, O,
                             None, idx, cnt, ws, stage_events=stage)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    stages = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    for st_ in stages:
        for e_ in st_:
            e_.record(stream)   # materialise the handles the C API records into
    # The mix is 14 launches from Python; enqueued one call at a time the GPU
    # waits for the host between them.  Timed with the host ahead: a bounded
    # GPU sleep (outside the events) holds the stream while the whole mix is
    # enqueued, so the events see device time.  The per-call (eager) time is
    # reported beside it.
    sleep_cycles = 4_000_000   # about 2 ms
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    barrier(dev)
    torch.cuda.synchronize(dev)
    sampler.start()
    for i in range(K):
        flush()
        torch.cuda._sleep(sleep_cycles)
        ev[i][0].record(stream)
        step(stages[i])
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    clocks = sampler.stop()
    eager = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush()
        eager[i][0].record(stream)
        step()
        eager[i][1].record(stream)
    torch.cuda.synchronize(dev)
    eager_us = statistics.median([a.elapsed_time(b) for a, b in eager]) * 1e3
    # the same mix as one dsa_layer_chain (programmatic dependent launches)
    chain_steps = [dsa.swa_step(s.Q, k, s.q_pos, 128, s.sink, sm_scale, O, None, ws_swa) for s, k in zip(swa, swa_kv)]
    chain_steps.append(dsa.dsa_step(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, Lmax, TOP_K, wl.sink, sm_scale, O,
                                    None, idx, cnt, ws))
    chained = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush()
        torch.cuda._sleep(sleep_cycles)
        chained[i][0].record(stream)
        dsa.dsa_layer_chain(chain_steps)
        chained[i][1].record(stream)
    torch.cuda.synchronize(dev)
    chained_us = statistics.median([a.elapsed_time(b) for a, b in chained]) * 1e3
    med = lambda xs: statistics.median(xs) * 1e3
    stage_us = {"swa_x5": med([ev[i][0].elapsed_time(stages[i][0]) for i in range(K)]),
                "dsa_indexer": med([stages[i][0].elapsed_time(stages[i][1]) for i in range(K)]),
                "dsa_topk": med([stages[i][1].elapsed_time(stages[i][2]) for i in range(K)]),
                "dsa_attention": med([stages[i][2].elapsed_time(stages[i][3]) for i in range(K)]),
                "dsa_combine": med([stages[i][3].elapsed_time(stages[i][4]) for i in range(K)])}
    for w_ in (ws, ws_swa):
        st, _ = dsa.dsa_check_device_status(w_)
        if st != dsa.DSA_OK:
            raise RuntimeError(f"device status {st} after the timed steps")
    ms = [a.elapsed_time(b) for a, b in ev]
    total_s = max_over_ranks(sum(ms) / 1e3, dev)
    peak, peak_kind = measured_peaks()
    dsa_bytes = sum(indexer_bytes(L, 1) for L in lens) + sum(gathered_bytes(1, min(TOP_K, L)) for L in lens)
    swa_bytes = 5 * sum(min(128, L) * 8 * (192 + 128) * 2 for L in lens)
    mix_bytes = dsa_bytes + swa_bytes
    return {
        "metric": MIX_METRIC, "value": throughput(B, K, world, total_s), "unit": "tok/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": total_s * 1e3 / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3xe4m3->f32 indexer; bf16 attention, f32 softmax",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC["ragged_b64_mix"], "batch": B, "query_tokens": 1,
                   "contexts": {"min": min(lens), "max": max(lens), "total": sum(lens)}, "top_k": TOP_K,
                   "seed": cfg["seed"], "parallelism": f"replicas x{world}",
                   "l2": "flushed before each mix outside the timed events"},
        "us_per_mix": total_s * 1e6 / K,
        "timing": "device time: the mix is fully enqueued before its first event (host ahead)",
        "us_per_mix_eager_median": eager_us,
        "us_per_mix_chained": chained_us,
        "stage_us_median": stage_us,
        "roofline": {"kernel": "whole mix (5 swa_attn_decode + dsa_layer_decode launches)", "bound": "hbm",
                     "achieved": mix_bytes / (total_s / K) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": mix_bytes / (total_s / K) / 1e9 / peak, "peak_kind": peak_kind, "traffic": None,
                     "algorithmic_bytes_per_launch": mix_bytes},
        "e2e": None,
        "gpu_launches": (5 + 4) * K,   # one kernel per SWA step, four for the 64-row DSA step
        "clocks": clocks,
    }


# ---------------------------------------------------- the layer stack step
STACK_METRIC = "attention-only decode stack step (39 SWA + 9 DSA layer-steps) at 1M context, tok/s"
DSA_LAYERS = (0, 5, 11, 17, 23, 29, 35, 41, 47)   # the layer pattern: 48 layers, DSA at these


def run_stack(args, rank, world, local_rank):
    """One step = the attention of every layer of the stack for one new token
    at 1,048,576 context: 48 layer-steps in the layer pattern's order, each DSA
    layer with its own 1M-context cache (index keys, K, V), each SWA layer its
    own window-only cache; enqueued as one dsa_layer_chain (the timed value)
    and as 48 separate calls (reported beside it).  L2 flushed before each
    stack step, not between layers."""
    import torch
    import local_attention_decode_b200 as dsa
    from workloads import CONFIGS, make_decode_workload, make_swa_window_workload

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = dict(CONFIGS["ctx_1m"])
    L = cfg["seq_lens"][0]
    sm_scale = 1.0 / math.sqrt(192)
    steps, keep = [], []
    O = torch.empty((1, 1, 64, 128), dtype=torch.bfloat16, device=dev)
    ws_swa = dsa.alloc_workspace(dsa.OP_SWA_ATTN, 1, 1, 1, 128, device=dev)
    ws_dsa = dsa.alloc_workspace(dsa.OP_LAYER, 1, 1, L, TOP_K, device=dev)
    calls = []
    for layer in range(48):
        if layer in DSA_LAYERS:
            wl = make_decode_workload(device=dev, **dict(cfg, seed=1000 + layer))
            kv = dsa.KV(k=wl.K, v=wl.V, index_k=wl.k8, index_k_scale=wl.k_scale, num_kv_heads=wl.G,
                        seq_stride=wl.layout.seq_stride, num_rows=wl.layout.num_rows)
            steps.append(dsa.dsa_step(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, L, TOP_K, wl.sink, sm_scale, O,
                                      None, None, None, ws_dsa))
            calls.append(lambda wl=wl, kv=kv: dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, L,
                                                                   TOP_K, wl.sink, sm_scale, O, ws=ws_dsa))
        else:
            wl = make_swa_window_workload(2000 + layer, [L], device=dev)
            kv = dsa.KV(k=wl.K, v=wl.V, num_kv_heads=wl.G, block_table=wl.layout.block_table,
                        page_size=wl.layout.page_size, num_rows=wl.layout.num_rows)
            steps.append(dsa.swa_step(wl.Q, kv, wl.q_pos, 128, wl.sink, sm_scale, O, None, ws_swa))
            calls.append(lambda wl=wl, kv=kv: dsa.swa_attn_decode(wl.Q, kv, wl.q_pos, 128, wl.sink, sm_scale, O,
                                                                  None, ws_swa))
        keep.append((wl, kv))
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def chained():
        dsa.dsa_layer_chain(steps)

    def eager():
        for c in calls:
            c()

    def timed(fn, K):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            flush()
            torch.cuda._sleep(4_000_000)   # the host enqueues the whole stack ahead of the GPU
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        return [a.elapsed_time(b) for a, b in ev]

    for _ in range(args.warmup):
        flush()
        chained()
        eager()
    torch.cuda.synchronize(dev)
    K = args.steps
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    barrier(dev)
    sampler.start()
    ms = timed(chained, K)
    barrier(dev)
    clocks = sampler.stop()
    ms_eager = timed(eager, K)
    for w_ in (ws_swa, ws_dsa):
        st, _ = dsa.dsa_check_device_status(w_)
        if st != dsa.DSA_OK:
            raise RuntimeError(f"device status {st} after the stack steps")
    total_s = max_over_ranks(sum(ms) / 1e3, dev)
    peak, peak_kind = measured_peaks()
    dsa_bytes = len(DSA_LAYERS) * (indexer_bytes(L, 1) + gathered_bytes(1, TOP_K))
    swa_bytes = (48 - len(DSA_LAYERS)) * 128 * 8 * (192 + 128) * 2
    step_s = total_s / K
    return {
        "metric": STACK_METRIC, "value": throughput(1, K, world, total_s), "unit": "tok/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3xe4m3->f32 indexer; bf16 attention, f32 softmax",
        "data": "synthetic",
        "config": {"workload": "48 layer-steps of one decode token at 1,048,576 context: DSA (top-2048, GQA4, sink) "
                               "at layers 0, 5, 11, 17, 23, 29, 35, 41, 47, SWA (window 128, GQA8, sink) at the "
                               "other 39; each layer its own cache", "parallelism": f"replicas x{world}",
                   "l2": "flushed before each stack step outside the timed events"},
        "us_per_stack_chained": step_s * 1e6,
        "us_per_stack_eager_median": statistics.median(ms_eager) * 1e3,
        "roofline": {"kernel": "whole stack (9 DSA + 39 SWA layer-steps)", "bound": "hbm",
                     "achieved": (dsa_bytes + swa_bytes) / step_s / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": (dsa_bytes + swa_bytes) / step_s / 1e9 / peak, "peak_kind": peak_kind, "traffic": None,
                     "algorithmic_bytes_per_launch": dsa_bytes + swa_bytes},
        "e2e": None,
        "gpu_launches": None,
        "clocks": clocks,
    }


# ------------------------------------------------------------- the prefill
PREFILL_METRIC = "chunked-prefill DSA layer (8,192 query tokens at 1M context) tok/s"


def run_prefill(args, rank, world, local_rank):
    """One step = dsa_prefill over 8,192 query tokens at positions
    1,040,384..1,048,575 of a 1,048,576-token cache (each causal): the sample
    thresholds, the fp8 contraction with the candidate filter on the tensor
    cores, the per-token selection and the attention.  L2 flushed before each
    step."""
    import torch
    import local_attention_decode_b200 as dsa
    from workloads import CONFIGS, make_decode_workload

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = CONFIGS["prefill_8k_1m"]
    wl = make_decode_workload(device=dev, **cfg)
    NQ = wl.T
    L = wl.layout.seq_lens[0]
    sm_scale = 1.0 / math.sqrt(192)
    kv = dsa.KV(k=wl.K, v=wl.V, index_k=wl.k8, index_k_scale=wl.k_scale, num_kv_heads=wl.G,
                seq_stride=wl.layout.seq_stride, num_rows=wl.layout.num_rows)
    O = torch.empty((NQ, 64, 128), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((NQ, TOP_K), dtype=torch.int32, device=dev)
    ws = dsa.alloc_workspace(dsa.OP_PREFILL, 1, NQ, L, TOP_K, device=dev)
    q8, qs, w, Q, qp = wl.q8[0], wl.q_scale[0], wl.w[0], wl.Q[0], wl.q_pos[0]
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        dsa.dsa_prefill(q8, qs, w, Q, kv, qp, L, TOP_K, wl.sink, sm_scale, O, None, idx, None, ws)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    barrier(dev)
    torch.cuda.synchronize(dev)
    sampler.start()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    clocks = sampler.stop()
    st, _ = dsa.dsa_check_device_status(ws)
    if st != dsa.DSA_OK:
        raise RuntimeError(f"device status {st} after the timed steps")
    total_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / 1e3, dev)
    step_s = total_s / K
    pos = wl.q_pos[0].cpu().double()
    flops = float(((pos + 1) * 16 * 128 * 2).sum())          # the indexer contraction, causal
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
        fp8_peak, fp8_kind = 2.0 * bf16, "measured bf16 x 2 (nominal fp8 : bf16 ratio)"
    except Exception:
        fp8_peak, fp8_kind = 2.0 * 1590.0, "fallback bf16 x 2"
    key_bytes = indexer_bytes(L, 0)                           # the keys streamed once by the contraction
    peak, peak_kind = measured_peaks()
    return {
        "metric": PREFILL_METRIC, "value": throughput(NQ, K, world, total_s), "unit": "tok/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3xe4m3->f32 indexer; bf16 attention, f32 softmax",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC["prefill_8k_1m"], "query_tokens": NQ, "context": L, "top_k": TOP_K,
                   "seed": cfg["seed"], "parallelism": f"replicas x{world}",
                   "l2": "flushed before each step outside the timed events"},
        "roofline": {"kernel": "the whole dsa_prefill call (sample thresholds, prefill_capture_kernel contraction, "
                               "per-token selection, attention); FLOPs of the indexer contraction only",
                     "bound": "tensor",
                     "achieved": flops / step_s / 1e12, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": flops / step_s / 1e12 / fp8_peak, "peak_kind": fp8_kind, "traffic": None,
                     "algorithmic_flops_per_step": flops},
        "hbm_view": {"key_bytes_per_step": key_bytes, "achieved_GBps": key_bytes / step_s / 1e9, "peak": peak,
                     "frac": key_bytes / step_s / 1e9 / peak, "peak_kind": peak_kind},
        "e2e": None,
        "gpu_launches": (6 + -(-NQ // 1024) * 2) * K,   # sample, indexer, selection, metadata, capture, select; attention + combine per 1,024 tokens
        "clocks": clocks,
    }


# ------------------------------------------------------------------ ours
def run_ours(args, rank, world, local_rank):
    """The layer-step at the workload's configuration.  Timed: K steps issued
    back to back, as a decode issues a model's DSA layers, each step on the
    next of R layers' own caches (index keys, K, V and queries drawn with
    their own seeds), so no step finds its keys in L2 -- the R caches hold
    R x 2.7 GB at 1M context against a 126 MB L2.  The R steps are one CUDA
    graph replayed K / R times: no host launch gaps.  Reported beside it: the
    same step isolated (L2 flushed, events around the one call), and the
    one-barrier kernel's phase trace."""
    import torch
    import local_attention_decode_b200 as dsa
    from workloads import CONFIGS, make_decode_workload

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = CONFIGS[args.workload]
    R = max(1, args.layers)
    layers = []
    for r in range(R):
        c = dict(cfg)
        c["seed"] = cfg["seed"] + 1000 * r
        w_r = make_decode_workload(device=dev, **c)
        kv_r = dsa.KV(k=w_r.K, v=w_r.V, index_k=w_r.k8, index_k_scale=w_r.k_scale, num_kv_heads=w_r.G,
                      seq_stride=w_r.layout.seq_stride, num_rows=w_r.layout.num_rows)
        layers.append((w_r, kv_r))
    wl, kv = layers[0]
    B, T = wl.B, wl.T
    L = wl.layout.seq_lens[0]
    sm_scale = 1.0 / math.sqrt(192)
    O = torch.empty((B, T, 64, 128), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((B, T, TOP_K), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, T), dtype=torch.int32, device=dev)
    ws = dsa.alloc_workspace(dsa.OP_LAYER, B, T, L, TOP_K, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)   # materialise the handle
        return evs

    def step(i=0, events=None):
        w_i, kv_i = layers[i % R]
        dsa.dsa_layer_decode(w_i.q8, w_i.q_scale, w_i.w, w_i.Q, kv_i, w_i.q_pos, L, TOP_K, w_i.sink, sm_scale, O,
                             None, idx, cnt, ws, stage_events=events)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    st, _ = dsa.dsa_check_device_status(ws)
    if st != dsa.DSA_OK:
        raise RuntimeError(f"device status {st} after warm-up")

    # ---- the R layer-steps captured once into a CUDA graph
    graph_note = f"{R} layers' steps in one CUDA graph, replayed"
    graph = None
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(R):
                step(i)
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(R):
                step(i)
        torch.cuda.synchronize(dev)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize(dev)
    except Exception as e:   # a launch that cannot be captured: eager launches
        graph = None
        graph_note = f"eager launches (graph capture failed: {type(e).__name__}: {e})"
        torch.cuda.synchronize(dev)

    K = max(R, args.steps // R * R)
    fused = B * T <= FUSED_MAX_ROWS
    paths0 = dsa.dsa_layer_path_counts(ws)
    t0, t1 = new_events(2)
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    barrier(dev)
    torch.cuda.synchronize(dev)
    sampler.start()
    t0.record(stream)
    if graph is not None:
        for _ in range(K // R):
            graph.replay()
    else:
        for i in range(K):
            step(i)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    clocks = sampler.stop()
    total_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, dev)
    paths1 = dsa.dsa_layer_path_counts(ws)
    st, _ = dsa.dsa_check_device_status(ws)
    if st != dsa.DSA_OK:
        raise RuntimeError(f"device status {st} after the timed steps")

    # ---- the same step isolated: L2 flushed, events around the one call
    K_iso = min(K, 100)
    stage = [new_events(5) for _ in range(K_iso)]
    if fused:
        stage = [[ev[0], None, None, None, ev[4]] for ev in stage]
    torch.cuda.synchronize(dev)
    for i in range(K_iso):
        flush()
        step(0, stage[i])
    torch.cuda.synchronize(dev)
    iso_ms = [stage[i][0].elapsed_time(stage[i][4]) for i in range(K_iso)]
    if not fused:
        idx_ms = [stage[i][0].elapsed_time(stage[i][1]) for i in range(K_iso)]
        topk_ms = [stage[i][1].elapsed_time(stage[i][2]) for i in range(K_iso)]
        attn_ms = [stage[i][2].elapsed_time(stage[i][3]) for i in range(K_iso)]
        comb_ms = [stage[i][3].elapsed_time(stage[i][4]) for i in range(K_iso)]

    # ---- the one-barrier kernel's phases (trace marks; steps back to back, untimed)
    phases = trace_phases(dsa, torch, dev, lambda i: step(i), R)

    # ---- the indexer on its own (dsa_indexer_scores) over the R layers' caches, back to back
    idx_ws = dsa.alloc_workspace(dsa.OP_INDEXER, B, T, L, 1, device=dev)
    scores = torch.empty((B, T, L), dtype=torch.float32, device=dev)
    ikvs = [dsa.KV(index_k=w_r.k8, index_k_scale=w_r.k_scale, num_kv_heads=w_r.G, seq_stride=w_r.layout.seq_stride,
                   num_rows=w_r.layout.num_rows) for w_r, _ in layers]

    def ind(i):
        w_i = layers[i % R][0]
        dsa.dsa_indexer_scores(w_i.q8, w_i.q_scale, w_i.w, ikvs[i % R], w_i.q_pos, L, scores, idx_ws)

    for i in range(R):
        ind(i)
    K2 = max(R, min(K, 400) // R * R)
    igraph = None
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(R):
                ind(i)
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        igraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(igraph):
            for i in range(R):
                ind(i)
        torch.cuda.synchronize(dev)
        igraph.replay()
    except Exception:
        igraph = None
    torch.cuda.synchronize(dev)
    a_, b_ = new_events(2)
    a_.record(stream)
    if igraph is not None:
        for _ in range(K2 // R):
            igraph.replay()
    else:
        for i in range(K2):
            ind(i)
    b_.record(stream)
    torch.cuda.synchronize(dev)
    ind_avg_s = a_.elapsed_time(b_) / 1e3 / K2
    # and isolated (L2 flushed; a bounded GPU sleep outside the events holds the
    # stream while the host prepares the call, so the events see only the kernel)
    K3 = min(K2, 100)
    iev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K3)]
    for i in range(K3):
        flush()
        torch.cuda._sleep(200_000)
        iev[i][0].record(stream)
        ind(0)
        iev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    ind_iso_ms = [a.elapsed_time(b) for a, b in iev]
    del scores

    # ---- a read-only stream reference measured in this run (torch sum over 1 GiB):
    # the indexer and the layer-step mostly read, so this is the closer ceiling
    read_gbs = read_stream_gbps(torch, dev, stream)

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, dsa, torch, layers, dev, stream, sm_scale, ws, flush)

    tokens = B * T
    value = throughput(tokens, K, world, total_s)
    peak, peak_kind = measured_peaks()
    ib = indexer_bytes(L, T)
    layer_bytes = ib + gathered_bytes(T, TOP_K)
    one_barrier = paths1[0] + paths1[1] > paths0[0] + paths0[1]
    if fused:   # one kernel does the whole step: its roofline is the whole step's bytes
        kern = "dsa_layer_capture_kernel" if one_barrier else "dsa_layer_fused_kernel"
        kern_bytes, kern_avg_s = layer_bytes, total_s / K
    else:
        kern, kern_bytes, kern_avg_s = "indexer_kernel", ib, ind_avg_s
    achieved = kern_bytes / kern_avg_s / 1e9
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tok/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_s * 1e3 / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3xe4m3->f32 indexer; bf16 attention, f32 softmax",
        "data": "synthetic",
        "config": decode_config(args.workload, world, R),
        "us_per_layer_step": total_s * 1e6 / K,
        "timing": f"{K} steps back to back over {R} layers' caches ({graph_note}); one event pair around them",
        "path": ("one cooperative kernel" if fused else "four kernels"),
        "timed_steps_by_path": {"one_barrier_fast": paths1[0] - paths0[0],
                                "one_barrier_general": paths1[1] - paths0[1],
                                "other": K - (paths1[0] - paths0[0]) - (paths1[1] - paths0[1])},
        "isolated_step_us": {"median": statistics.median(iso_ms) * 1e3, "mean": statistics.fmean(iso_ms) * 1e3,
                             "how": "L2 flushed before each step; events around the one call (launch included)"},
        "stage_us_median": ({"layer_step_isolated": statistics.median(iso_ms) * 1e3} if fused else {
            "indexer": statistics.median(idx_ms) * 1e3, "topk": statistics.median(topk_ms) * 1e3,
            "attention": statistics.median(attn_ms) * 1e3, "combine": statistics.median(comb_ms) * 1e3,
        }),
        "phase_us": phases,
        "indexer_standalone": {
            "us_mean": ind_avg_s * 1e6, "bytes": ib,
            "GBps": ib / ind_avg_s / 1e9, "frac_of_measured_peak": ib / ind_avg_s / 1e9 / peak,
            "frac_of_8TBps_nominal": ib / ind_avg_s / 1e9 / NOMINAL_HBM_GBS,
            "how": f"{K2} launches back to back over the {R} layers' index caches, one event pair",
            "isolated_us_median": statistics.median(ind_iso_ms) * 1e3,
        },
        "layer_step_byte_roofline_us": {
            "bytes": layer_bytes,
            "at_measured_peak": layer_bytes / (peak * 1e9) * 1e6,
            "at_8TBps_nominal": layer_bytes / (NOMINAL_HBM_GBS * 1e9) * 1e6,
            "at_read_stream": layer_bytes / (read_gbs * 1e9) * 1e6,
        },
        "read_stream_reference": {"GBps": read_gbs, "how": "torch sum over 1 GiB fp32, best of 6, CUDA events",
                                  "layer_step_frac": kern_bytes / kern_avg_s / 1e9 / read_gbs if fused else None,
                                  "indexer_frac": ib / ind_avg_s / 1e9 / read_gbs},
        "roofline": {
            "kernel": kern, "bound": "hbm", "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
            "frac_of_8TBps_nominal": achieved / NOMINAL_HBM_GBS,
            "traffic": recorded_traffic(kern), "algorithmic_bytes_per_launch": kern_bytes,
            "avg_launch_us": kern_avg_s * 1e6,
        },
        "e2e": e2e,
        "gpu_launches": (1 if fused else 4) * K,
        "clocks": clocks,
        "_workload": wl,
    }
    return line


def trace_phases(dsa, torch, dev, step, R, n=8):
    """Median over n steps of each phase mark of the one-barrier layer-step
    kernel, in us after the first CTA's entry, as the latest CTA reached it
    (dsa_trace_phases); {} when that kernel did not run."""
    import numpy as np
    tr = torch.zeros(148 * 2 * dsa.TRACE_MARKS, dtype=torch.int64, device=dev)
    names = {10: "first_key_tile_requested", 12: "first_tile_scored", 7: "sample_handed_in", 1: "thresholds_seen",
             2: "key_stream_done", 15: "candidates_captured", 3: "past_grid_barrier", 8: "candidates_in_smem",
             9: "kth_key_found",
             4: "selection_done", 5: "attention_units_done", 6: "exit"}
    rows, mids, spans = [], [], {}
    chain = [2, 15, 3, 8, 9, 4, 5, 6]
    dsa.dsa_trace_phases(tr)
    try:
        for i in range(n):
            tr.zero_()
            step(i)
            torch.cuda.synchronize(dev)
            m = tr.view(-1, dsa.TRACE_MARKS).cpu().numpy().astype(np.float64)
            m = m[m[:, 0] > 0]
            if len(m) == 0:
                return {}
            t0 = m[:, 0].min()
            rows.append({k: (m[:, k][m[:, k] > 0].max() - t0) / 1e3 for k in names if (m[:, k] > 0).any()})
            mids.append({k: (np.median(m[:, k][m[:, k] > 0]) - t0) / 1e3 for k in names if (m[:, k] > 0).any()})
            # each CTA's own time between consecutive marks of the post-stream chain
            for a_, b_ in zip(chain[:-1], chain[1:]):
                ok = (m[:, a_] > 0) & (m[:, b_] > 0)
                if ok.any():
                    d = (m[ok, b_] - m[ok, a_]) / 1e3
                    spans.setdefault((a_, b_), []).append((np.median(d), d.max()))
    finally:
        dsa.dsa_trace_phases(None)
    out = {names[k]: float(np.median([r[k] for r in rows if k in r])) for k in names if any(k in r for r in rows)}
    out["how"] = "latest CTA at each mark, us after the first CTA entered; median of 8 steps"
    out["median_cta"] = {names[k]: round(float(np.median([r[k] for r in mids if k in r])), 3)
                         for k in names if any(k in r for r in mids)}
    out["per_cta_span_us"] = {f"{names[a_]}->{names[b_]}": {"median": round(float(np.median([x[0] for x in v])), 3),
                                                           "max": round(float(np.median([x[1] for x in v])), 3)}
                              for (a_, b_), v in spans.items()}
    return out


def run_e2e(args, dsa, torch, layers, dev, stream, sm_scale, ws, flush):
    """Same metric through the public API with host buffers.  Per step, the new
    token's raw inputs -- its index query (16 heads) and index key before
    normalisation, RoPE and fp8 (bf16), the head weights, the backbone query,
    its position, and its backbone K / V rows -- go host -> device in one copy
    from pinned memory; dsa_index_produce normalises, rotates and quantises the
    index key into the cache row and the index queries into their e4m3 codes;
    the K / V rows are written into the cache; the layer-step runs; the output
    and the selection come back to the host in one copy.  The steps run back to
    back over the layers' caches in rotation, as the headline's do (inputs
    larger than L2), with every step's two copies inside the timed region; the
    same step isolated (L2 flushed, events around it) is reported beside."""
    wl = layers[0][0]
    R = len(layers)
    B, T = wl.B, wl.T
    L = wl.layout.seq_lens[0]
    G = wl.G
    row = L - 1
    g = torch.Generator(device="cpu").manual_seed(77)
    # packed per-step input: each part 256-byte aligned inside one buffer
    parts = [("q_in", torch.bfloat16, (B, T, 16, 128)), ("k_in", torch.bfloat16, (B, T, 128)),
             ("w", torch.float32, (B, T, 16)), ("Q", torch.bfloat16, (B, T, 64, 192)),
             ("pos", torch.int32, (B, T)), ("K", torch.bfloat16, (G, 192)), ("V", torch.bfloat16, (G, 128))]
    offs, off = {}, 0
    for name, dt, shape in parts:
        nbytes = math.prod(shape) * torch.tensor([], dtype=dt).element_size()
        offs[name] = (off, dt, shape, nbytes)
        off = (off + nbytes + 255) // 256 * 256
    h_in = torch.empty(off, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(off, dtype=torch.uint8, device=dev)

    def view(buf, name):
        o, dt, shape, nbytes = offs[name]
        return buf[o:o + nbytes].view(dt).view(shape)

    view(h_in, "q_in").copy_(torch.randn((B, T, 16, 128), generator=g).to(torch.bfloat16))
    view(h_in, "k_in").copy_(torch.randn((B, T, 128), generator=g).to(torch.bfloat16))
    view(h_in, "w").copy_(wl.w.cpu())
    view(h_in, "Q").copy_(wl.Q.cpu())
    view(h_in, "pos").copy_(wl.q_pos.cpu())
    view(h_in, "K").copy_(wl.K[row].cpu())
    view(h_in, "V").copy_(wl.V[row].cpu())
    d_qin, d_kin, d_w, d_Q, d_pos, d_K, d_V = (view(d_in, n) for n, _, _ in parts)
    ln_w = torch.ones(128, device=dev)
    ln_b = torch.zeros(128, device=dev)
    q8 = torch.empty((B, T, 16, 128), dtype=torch.uint8, device=dev)
    qs = torch.empty((B, T, 16), dtype=torch.float32, device=dev)
    ws_p = dsa.alloc_workspace(dsa.OP_PRODUCE, B, T, 1, 1, device=dev)
    # outputs: O and the selection in one device buffer, read back in one copy
    o_bytes = B * T * 64 * 128 * 2
    i_bytes = B * T * TOP_K * 4
    d_out = torch.empty(o_bytes + i_bytes, dtype=torch.uint8, device=dev)
    h_out = torch.empty(o_bytes + i_bytes, dtype=torch.uint8).pin_memory()
    O = d_out[:o_bytes].view(torch.bfloat16).view(B, T, 64, 128)
    idx = d_out[o_bytes:].view(torch.int32).view(B, T, TOP_K)
    cnt = torch.empty((B, T), dtype=torch.int32, device=dev)
    h2d = off
    d2h = o_bytes + i_bytes

    def step(i=0):
        w_i, kv_i = layers[i % R]
        d_in.copy_(h_in, non_blocking=True)
        dsa.dsa_index_produce(d_kin, d_qin, ln_w, ln_b, 1e-5, 42, 1e7, kv_i, d_pos, q8, qs, ws_p)
        torch._foreach_copy_([w_i.K[row], w_i.V[row]], [d_K, d_V], non_blocking=True)   # (one launch)
        dsa.dsa_layer_decode(q8, qs, d_w, d_Q, kv_i, d_pos, L, TOP_K, w_i.sink, sm_scale, O, None, idx, cnt, ws)
        h_out.copy_(d_out, non_blocking=True)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    K = max(R, args.steps // R * R)

    # the same step isolated: L2 flushed, events around the one step (eager)
    K_iso = min(K, 50)
    iso = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_iso)]
    for i in range(K_iso):
        flush()
        iso[i][0].record(stream)
        step(0)
        iso[i][1].record(stream)
    torch.cuda.synchronize(dev)
    iso_ms = statistics.median([a.elapsed_time(b) for a, b in iso])

    # the R steps captured once into a CUDA graph (copies, producer, cache
    # writes, layer-step, copy back), replayed K / R times back to back
    graph_note = f"{R} layers' steps captured once in a CUDA graph, replayed back to back"
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(R):
                step(i)   # one more warm-up on the capture stream
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(graph):
            for i in range(R):
                step(i)
        torch.cuda.synchronize(dev)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize(dev)
    except Exception as e:   # a launch that cannot be captured: eager steps
        graph = None
        graph_note = f"eager steps back to back (graph capture failed: {type(e).__name__}: {e})"
        torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    if graph is not None:
        for _ in range(K // R):
            graph.replay()
    else:
        for i in range(K):
            step(i)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    for w_ in (ws, ws_p):
        st, _ = dsa.dsa_check_device_status(w_)
        if st != dsa.DSA_OK:
            raise RuntimeError(f"device status {st} after the end-to-end steps")
    total_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, dev)
    import torch.distributed as dist
    world = dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1
    return {"value": throughput(B * T, K, world, total_s), "unit": "tok/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": total_s * 1e3 / K, "steps": K,
            "per_step": "1 pinned H2D copy of the token's raw inputs; dsa_index_produce (index key into the cache, "
                        "index query codes); the K/V rows copied into the cache (one launch); dsa_layer_decode; "
                        "1 D2H copy of O and the selection -- " + graph_note,
            "l2": f"inputs larger than L2: {R} layers' caches in rotation, no flush",
            "ms_per_step_isolated_median": iso_ms,
            "isolated": "L2 flushed before each step, events around the one eager step"}


# ------------------------------------------------------- CPU oracle timing
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def oracle_step(host, n_keys: int):
    """One layer-step of the CPU oracle on the first n_keys keys of a host copy
    of the workload (`host`: q8, q_scale, w, k8, k_scale, Q, sink, K/V row
    getter): indexer over the n_keys keys, top-2048, attention over the
    selected rows.  Returns (seconds of indexer + selection, seconds of
    attention)."""
    import numpy as np
    import oracle
    t0 = time.perf_counter()
    s = oracle.indexer_scores(host["q8"], host["q_scale"], host["w"], host["k8"][:n_keys], host["k_scale"][:n_keys],
                              np.array([n_keys - 1], np.int32))
    sel, c = oracle.topk(s[0], TOP_K)
    t1 = time.perf_counter()
    sel = sel[:c]
    Kr, Vr = host["kv_rows"](sel)
    oracle.gqa_attention(host["Q"], Kr, Vr, np.arange(len(sel), dtype=np.int32), host["sink"],
                         1.0 / math.sqrt(192))
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def host_copy(wl):
    """Host arrays of a one-sequence, one-token decode workload for the oracle
    (the K/V rows are copied only where the selection points)."""
    from workloads import bits16
    K, V = wl.K, wl.V
    return {"q8": wl.q8[0].cpu().numpy(), "q_scale": wl.q_scale[0].cpu().numpy(), "w": wl.w[0].cpu().numpy(),
            "k8": wl.k8.cpu().numpy(), "k_scale": wl.k_scale.cpu().numpy(), "Q": bits16(wl.Q[0, 0]),
            "sink": wl.sink.cpu().numpy(),
            "kv_rows": lambda sel: (bits16(K[sel]), bits16(V[sel]))}


def cpu_baseline_line(wl, full_budget_s: float = 40.0):
    """The oracle on the host cores, on this run's own ctx_1m inputs: the whole
    1,048,576-key step on all cores (timed, not extrapolated) when a first
    sample says it fits the budget, and a single-core sample of 65,536 keys
    scaled to the full context beside it."""
    import oracle
    host = host_copy(wl)
    L = host["k8"].shape[0]
    cores = oracle.set_threads(host_cores())
    n0 = min(L, 65536)
    a, b = oracle_step(host, n0)
    est = a * L / n0 + b
    if est <= full_budget_s:
        a, b = oracle_step(host, L)
        all_s, all_kind = a + b, f"the whole {L}-key step, timed"
    else:
        all_s, all_kind = est, f"the first {n0} keys, indexer and selection time scaled by {L}/{n0}"
    oracle.set_threads(1)
    a1, b1 = oracle_step(host, n0)
    one_s = a1 * L / n0 + b1
    return {"value": 1.0 / all_s, "unit": "tok/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cores": host_cores(),
            "sample": f"one ctx_1m layer-step (indexer over the keys, top-2048, attention over the selection) of "
                      f"this run's inputs on {cores} host threads: {all_kind}; C oracle in double",
            "single_core": {"value": 1.0 / one_s, "unit": "tok/s", "cores": 1,
                            "sample": f"first {n0} keys on one thread, indexer and selection scaled by {L}/{n0}"}}


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step one ctx_1m layer-step on all
    host cores -- the whole 1,048,576 keys when (steps + warm-up) of those fit
    about 150 s, otherwise the first n keys with the indexer and selection
    time scaled by 1,048,576 / n (and labelled as extrapolated)."""
    if rank != 0:
        return None
    import oracle
    from workloads import CONFIGS, make_decode_workload
    wl = make_decode_workload(**CONFIGS[WORKLOAD])
    host = host_copy(wl)
    L = host["k8"].shape[0]
    cores = oracle.set_threads(host_cores())
    steps = args.steps + args.warmup
    budget_s = 150.0
    n0 = min(L, 65536)
    a, b = oracle_step(host, n0)
    per_key = a / n0
    n = int(min(L, max(TOP_K, (budget_s / steps - b) / max(per_key, 1e-12))))
    n = max(TOP_K, n - n % 128)
    times = []
    for i in range(steps):
        a, b = oracle_step(host, n)
        if i >= args.warmup:
            times.append(a * L / n + b)
    total = sum(times)
    value = len(times) / total
    how = (f"each step the whole {L}-key ctx_1m layer-step on {cores} host threads, timed" if n == L else
           f"each step the first {n} keys of the ctx_1m inputs on {cores} host threads, indexer and selection "
           f"time extrapolated by {L}/{n} (the full step does not fit the run's time budget)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total * 1e3 / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(WORKLOAD, world, args.layers),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": how,
                         "cpu_model": cpu_model(), "extrapolated": n != L},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--layers", type=int, default=4,
                    help="layers' caches the timed decode steps rotate over (inputs larger than L2)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--profile", type=int, default=0, metavar="N",
                    help="no timing: N iterations of (L2 flush, dsa_indexer_scores, L2 flush, dsa_layer_decode) on "
                         "the workload, for a profiler to attach to; prints the device status")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the ragged-mix and prefill lines that the default run adds as extra keys")
    ap.add_argument("--workload", choices=["tiny_8k", "verify_64k_t4", "ctx_1m", "ragged_b64_mix", "prefill_8k_1m",
                                           "stack_1m"],
                    default=WORKLOAD,
                    help="decode workload recipe (workloads.CONFIGS); the headline metric is on ctx_1m")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local_rank = dist_env()

    if args.profile > 0:
        profile_run(args)
        return
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run = {"ragged_b64_mix": run_mix, "prefill_8k_1m": run_prefill, "stack_1m": run_stack}.get(args.workload,
                                                                                                    run_ours)
        line = run(args, rank, world, local_rank)
        wl = line.pop("_workload", None)
        if args.workload == WORKLOAD and not args.no_secondary:
            # the other benchmarked workloads, a few steps each, as extra keys
            line["secondary"] = secondary_lines(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and args.workload == WORKLOAD and wl is not None:
                line["cpu_baseline"] = cpu_baseline_line(wl)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


def profile_run(args):
    """Untimed iterations of the indexer and the layer-step for ncu (one GPU):
    each call after an L2 flush, so counters see a cold L2."""
    import torch
    import local_attention_decode_b200 as dsa
    from workloads import CONFIGS, make_decode_workload
    dev = torch.device("cuda", 0)
    wl = make_decode_workload(device=dev, **CONFIGS[args.workload])
    B, T = wl.B, wl.T
    L = wl.layout.seq_lens[0]
    kv = dsa.KV(k=wl.K, v=wl.V, index_k=wl.k8, index_k_scale=wl.k_scale, num_kv_heads=wl.G,
                seq_stride=wl.layout.seq_stride, num_rows=wl.layout.num_rows)
    ikv = dsa.KV(index_k=wl.k8, index_k_scale=wl.k_scale, num_kv_heads=wl.G, seq_stride=wl.layout.seq_stride,
                 num_rows=wl.layout.num_rows)
    O = torch.empty((B, T, 64, 128), dtype=torch.bfloat16, device=dev)
    scores = torch.empty((B, T, L), dtype=torch.float32, device=dev)
    ws = dsa.alloc_workspace(dsa.OP_LAYER, B, T, L, TOP_K, device=dev)
    iws = dsa.alloc_workspace(dsa.OP_INDEXER, B, T, L, 1, device=dev)
    flush = L2Flush(dev)
    for _ in range(args.profile):
        flush()
        dsa.dsa_indexer_scores(wl.q8, wl.q_scale, wl.w, ikv, wl.q_pos, L, scores, iws)
        flush()
        dsa.dsa_layer_decode(wl.q8, wl.q_scale, wl.w, wl.Q, kv, wl.q_pos, L, TOP_K, wl.sink, 1.0 / math.sqrt(192), O,
                             ws=ws)
    torch.cuda.synchronize(dev)
    print(json.dumps({"profile_iterations": args.profile, "workload": args.workload,
                      "status": [dsa.dsa_check_device_status(w)[0] for w in (ws, iws)],
                      "layer_step_paths": dsa.dsa_layer_path_counts(ws)}), flush=True)


def secondary_lines(args, rank, world, local_rank):
    """The ragged 64-sequence layer mix and the chunked prefill, a few timed
    steps each (every rank runs them; the same collective steps on all ranks)."""
    import torch
    out = {}
    for name, fn, steps in (("ragged_b64_mix", run_mix, 20), ("stack_1m", run_stack, 10),
                            ("prefill_8k_1m", run_prefill, 3)):
        sub = argparse.Namespace(**vars(args))
        sub.steps, sub.warmup, sub.workload = steps, 3, name
        try:
            line = fn(sub, rank, world, local_rank)
            out[name] = {k: line[k] for k in ("metric", "value", "unit", "ms_per_step", "steps", "warmup", "roofline",
                                             "clocks", "gpu_launches", "config") if k in line}
            for k in ("us_per_mix", "stage_us_median", "hbm_view", "us_per_stack_chained", "us_per_stack_eager_median",
                      "us_per_mix_eager_median", "us_per_mix_chained"):
                if k in line:
                    out[name][k] = line[k]
        except Exception as e:   # reported, not fatal for the headline line
            out[name] = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    main()
