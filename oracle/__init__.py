"""CPU oracle for the PLE n-gram embedding layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. The product path (the CUDA library and its Python
binding) never imports it. See ``ple_oracle`` for the definition and readings.
"""
from .ple_oracle import (  # noqa: F401
    E2M1_VALUES, E4M3_VALUES, HEAD_MIX, HEADS_PER_ORDER, P0, P1, P2, ArrayTable, HeadsArrayTable,
    Nvfp4ArrayTable, bf16_bits_to_f64, dequantise, ngram_ids_heads, row_ids,
    dequantise_nvfp4, e2m1_decode, e4m3_decode, embed, table_rows, unpack_fp4,
    end_state, fold, gate, ngram_contexts, ngram_ids, ngram_keys, ple_decode_step,
    ple_forward, project, sequence_map, short_conv, to_bf16_bits, to_f32,
)
