"""fp64 CPU oracle for differential attention (test infrastructure only).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never touches it, and the two share no code.
"""
from .oracle import (  # noqa: F401
    build,
    lambda_init,
    lambda_from_params,
    v1_rows,
    v2_rows,
    v2_oproj_rows,
    v2_decode_rows,
    v1_decode_rows,
    n_threads,
    v1_query_weights,
    snr,
    v1_bwd,
    v2_bwd,
    lambda_params_bwd,
)
