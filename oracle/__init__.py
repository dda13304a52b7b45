"""fp64 CPU oracle for the CSA/HCA attention path (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA path.
"""
from .csa_oracle import (  # noqa: F401
    RMS_EPS,
    as_f64,
    attend,
    compress,
    compress_rope,
    e4m3_decode,
    e4m3_encode,
    hadamard_matrix,
    hadamard_rotate,
    hca_mqa,
    index_compress,
    index_scores,
    index_scores_fp8,
    index_topk,
    index_topk_fp8,
    n_entries,
    n_visible,
    quantize_rows_e4m3,
    rms_norm,
    rope_last_dims,
    round_to,
    sparse_mqa,
    topk,
    window_rows,
)
