"""fp64 CPU oracle of the DSA decode step. Test infrastructure only: the product
path never imports it (tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs are its only users)."""
from .dsa_oracle import (  # noqa: F401
    decode_e4m3, decode_bf16, dequant_index_queries, dequant_index_keys, dequant_latent_rows,
    visible_lengths, physical_slots, pagemap, indexer_scores, topk_logical,
    mla_sparse_attention, mla_partials, combine_partials, mla_sparse_attention_split,
    decode_layer, encode_e4m3, quantize_e4m3, encode_bf16, rope_interleaved, new_token_positions,
    physical_slots_rows, rope_quantize_append, shard_candidates, shard_global_select,
    sharded_decode_layer,
)
