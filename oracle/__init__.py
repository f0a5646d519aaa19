"""CPU oracle for the DSA / SWA decode layer-step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does.  The arithmetic lives in ``oracle.c``; this
module is argument marshalling plus the composition of the steps in the order
the explainer page gives them ("Naive-N0.5-Flash: no full-attention layers, and
a runtime built by AI", section "Inside a DSA layer: the lightning indexer"):
indexer scores -> top-k positions -> attention over the selected keys.
"""
from .oracle import (  # noqa: F401
    build_oracle,
    set_threads,
    e4m3_to_float64,
    bf16_to_float64,
    fp8_dot,
    indexer_scores,
    topk,
    topk_select,
    gqa_attention,
    swa_indices,
    dsa_layer_decode,
    swa_layer_decode,
    layernorm,
    rope_partial,
    e4m3_encode,
    index_k_produce,
    index_q_produce,
    indexer_kl,
)
