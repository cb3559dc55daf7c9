"""fp64 CPU oracle of the SALR linear layer (test infrastructure only; see salr_oracle)."""
from .salr_oracle import *  # noqa: F401,F403
from .salr_oracle import (abs_bound, check_tolerance, concat_adapters, decode_format,
                          encode_format, keep_count, linear, magnitude_mask, mse_factor,
                          prune, residual, truncated_svd_adapter, OracleError)
