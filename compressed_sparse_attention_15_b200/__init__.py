"""B200-native hybrid compressed-sparse attention (CSA / HCA) hot path.

The path -- gated-pooling KV compressor, ReLU-weighted indexer with top-k,
and 64:1 MQA over the selected entries + a 128-token sliding window + a
per-head sink -- runs in hand-written sm_100a CUDA kernels behind the C ABI of
libcsa.so (include/csa.h). ``ops`` holds the torch-facing wrappers; the
library is loaded on first use and its absence is an error.
"""
from . import ops, step, synth, workloads  # noqa: F401
from .ops import (  # noqa: F401
    Workspace,
    compress,
    hca_mqa,
    index_scores,
    index_topk,
    sparse_mqa,
    topk,
    num_entries,
    visible_entries,
    workspace_status,
)


def build(force: bool = False) -> str:
    """Compile libcsa.so in-tree (nvcc, sm_100a)."""
    from .build import build as _build

    return _build(force=force)
from .step import DecodeStep  # noqa: F401,E402
