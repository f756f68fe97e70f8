"""fp64 CPU oracle (test infrastructure only; see dark_oracle's header)."""
from .dark_oracle import (attention, attention_rows, decode_step, exponent_range,  # noqa: F401
                          feature_exponents, feature_map, kernel_matrix)
