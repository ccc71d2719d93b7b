"""fp64 CPU oracle for the Star / Pulsar two-phase attention path.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the Pulsar Attention and Star Attention pages define.  It
shares no code with the CUDA path and imports nothing from it.  Only the test
suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference arm of
``bench.py`` may import or run it; the product path never does.

Parity status of each function is stated in its module's header.
"""
from .pulsar_oracle import (  # noqa: F401
    document_frequency,
    idf_table,
    chunk_scores,
    chunk_min_df,
    select_summaries,
    host_positions,
    host_row_offsets,
    rope,
    causal_attention,
    phase1_encode,
    retained_kv,
    shard_bounds,
    phase2_partials,
    lse_merge,
    phase2_attend,
    phase1_flops,
    chunk_mean_idf,
    chunk_df_product,
    select_evenly_spaced,
    select_summaries_mean_idf,
    chunk_entropy,
    chunk_tf_power_product,
    select_summaries_entropy,
    chunk_bm25,
    select_summaries_bm25,
    phase2_attend_with_self,
    phase2_attend_art,
)
