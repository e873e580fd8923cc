"""CPU oracle (test infrastructure only; never imported by the product path)."""
from .dkv_oracle import (  # noqa: F401
    FLAG_CAPACITY, FLAG_RANGE, CapacityError, OracleCache, OracleRaggedCache, bf16_to_f32, bf16_to_f64,
    bool_to_mask_words, dense_attention_f64, mask_words_to_bool, pack_codes,
    quantize_groups, quantize_stream_oneshot, sanitize, to_fp16, unpack_codes,
)
