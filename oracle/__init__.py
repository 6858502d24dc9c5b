"""fp64 CPU oracle for the TPA hot path — test infrastructure only (see tpa_oracle)."""
from .tpa_oracle import (  # noqa: F401
    FACTOR_NAMES, Dims, factor_widths, cache_elements_per_token, rope_inv_freq,
    rope_rotate, split_factors, project, materialize, causal_attention, tpa_forward,
    attend_from_factors, decode_query, decode_attention, tpa_forward_rows, output_projection,
    broadcast_basis, shared_basis_tables,
)
