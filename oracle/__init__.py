"""fp64 CPU oracle (test infrastructure only; never imported by the product path)."""
from .attention import (  # noqa: F401
    NEG_INF, SkipRecord, allowed_mask, bf16_bits_to_f64, combine_partials, gather_paged,
    group_attention, kv_head_of, literal_group_attention, paged_decode, paged_prefill, round_f64_to_bf16,
    smallseq_attention, smallseq_backward, softmax_over_kept, split_partials, tile_decisions, tile_ratio,
    unit_skipped, varlen_attention, varlen_backward,
)
