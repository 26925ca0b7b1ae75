"""Float64 CPU oracle of the iS-KV hot path (test infrastructure only; see iskv_oracle)."""
from .iskv_oracle import (OracleCache, OracleUnit, attention, chunk_scores, fold,  # noqa: F401
                          fold_from_coords, n_compressed, protected_positions, residual_basis,
                          rope, round_bf16, svd_r, value_protected)
