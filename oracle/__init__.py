"""fp64 CPU oracle (test infrastructure only; never imported by the product path)."""
from .streamkl_oracle import (  # noqa: F401
    allowed,
    oracle_bwd,
    oracle_bwd_gqa,
    oracle_bwd_teacher,
    oracle_bwd_teacher_gqa,
    oracle_bwd_teacher_varlen,
    oracle_bwd_varlen,
    oracle_dk_rows,
    oracle_fwd,
    oracle_fwd_gqa,
    oracle_fwd_varlen,
    oracle_row_work,
    oracle_rows,
    row_pair_count,
)
