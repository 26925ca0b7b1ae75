"""Float64 CPU oracle of the iS-KV hot path (test infrastructure only; see iskv_oracle)."""
from .iskv_oracle import (OracleCache, OracleUnit, attention, fold, fold_from_coords,  # noqa: F401
                          n_compressed, residual_basis, rope, round_bf16, svd_r)
