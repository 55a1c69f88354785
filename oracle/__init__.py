"""fp64 CPU oracle (test infrastructure only; never imported by the product path)."""
from .streamkl_oracle import (  # noqa: F401
    allowed,
    oracle_bwd,
    oracle_bwd_teacher,
    oracle_dk_rows,
    oracle_fwd,
    oracle_row_work,
    oracle_rows,
    row_pair_count,
)
