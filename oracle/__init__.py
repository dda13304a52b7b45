"""fp64 CPU oracle for the CSA/HCA attention path (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA path.
"""
from .csa_oracle import (  # noqa: F401
    RMS_EPS,
    as_f64,
    attend,
    compress,
    hca_mqa,
    index_scores,
    index_topk,
    n_entries,
    n_visible,
    rms_norm,
    round_to,
    sparse_mqa,
    topk,
    window_rows,
)
