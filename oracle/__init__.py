"""CPU float64 oracle (test infrastructure only; see ``mqa_oracle``)."""
from .mqa_oracle import (  # noqa: F401
    dot_product_attention,
    oracle_decode,
    oracle_decode_step,
    oracle_kv_append,
    oracle_prefill,
    oracle_decode_beam,
)
