"""CPU fp64 oracle (test infrastructure only; see mla_oracle's header)."""
from .mla_oracle import (  # noqa: F401
    cache_elements_per_token,
    cache_rows,
    cache_rows_from_hidden,
    decode_absorbed,
    decode_expanded,
    output_projection,
    rms_norm,
    rope,
)
