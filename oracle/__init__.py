"""fp64 CPU oracle for exact softmax attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does.
"""
from .oracle import (  # noqa: F401
    CAUSAL, SPARSE, build, fwd_rows, fwd, online_softmax_fwd, bwd_full,
    bwd_dq_rows, bwd_dkdv_cols, library_path,
    e4m3_values, e4m3_round, rotate_f32, fp8_quantize, fwd_fp8, fp8_o_bounds, fwd_varlen, bwd_varlen,
)
