"""CPU oracle for the CSA2 decode path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package; the product path never does.
"""
from .csa2_oracle import *  # noqa: F401,F403
from .csa2_oracle import (FULL, REINDEX, REUSE, LayerResult, attention_combine, attention_set, decode_layer_plan,
                          e2m1_decode, e4m3_decode, e4m3_encode_rne, fp4_dequant, fp4_quantize,
                          full_index, index_scores, kv_rows_local_window, prefill_query, reindex,
                          score_bound, sparse_attention, top_k_positions)
