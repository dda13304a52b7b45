"""csa_index_topk_noalloc: the indexer + top-k for callers that cannot
allocate device memory.

Such callers -- a plugin that a host framework hands only input and output
pointers while it owns every device allocation, or a decode loop that must
not stall on cudaMalloc in the middle of a step -- cannot supply the
workspace csa_index_topk needs. The no-allocation entry point uses a scratch
buffer built into the library instead. It has to return exactly what
csa_index_topk returns with a caller-provided workspace, call after call,
even though every call reuses the same buffer. This file runs last so that a
failure here cannot hide any other test's result.
"""
import ctypes

import pytest
import torch

from compressed_sparse_attention_15_b200 import _lib, ops, synth

CSA_ERR_SCRATCH_LIMIT = 6


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(seed, Q, B, N, Hi, Di, dtype, dev):
    qi = synth.normal(seed, 4, (Q, Hi, Di), dtype=dtype, device=dev)
    wi = synth.uniform(seed, 5, (Q, Hi), device=dev)
    ki = synth.normal(seed, 6, (B, N, Di), dtype=dtype, device=dev)
    n = torch.tensor([N - (q % 3) * 7 for q in range(Q)], dtype=torch.int32, device=dev)
    return qi, wi, ki, n


@pytest.mark.gpu
@pytest.mark.parametrize("Q,B,N,Hi,Di,k,dtype", [
    (32, 32, 16383, 64, 128, 512, torch.bfloat16),   # the 64 K-context decode batch (tensor-core scorer)
    (12, 3, 3001, 4, 16, 16, torch.float32),         # small fp32 case (generic scorer)
    # no cluster fits (75 queries on 148 SMs) and the lists exceed the one-block
    # key cache: the two-stage selection, whose segment winners live in the
    # shared buffer beyond the scores
    (75, 75, 52000, 4, 16, 16, torch.float32),
])
def test_noalloc_matches_the_workspace_entry_point_twice(cuda_device, Q, B, N, Hi, Di, k, dtype):
    L = _lib.lib()
    code = _lib.CSA_DTYPE_BF16 if dtype == torch.bfloat16 else _lib.CSA_DTYPE_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    # Two calls in a row with different inputs: the second must not see
    # anything the first left in the shared scratch buffer.
    for seed in (1, 2):
        qi, wi, ki, n = _inputs(seed, Q, B, N, Hi, Di, dtype, cuda_device)
        want = ops.index_topk(qi, wi, ki, n, k, q_per_seq=Q // B)
        got = torch.full((Q, k), -7, dtype=torch.int32, device=cuda_device)
        rc = L.csa_index_topk_noalloc(_p(qi), _p(wi), _p(ki), _p(n), k, _p(got), Q, B, Hi, Di, N, Q // B, code,
                                      stream)
        assert rc == 0, _lib.strerror(rc)
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"seed {seed}: no-allocation result differs from csa_index_topk"


@pytest.mark.gpu
def test_noalloc_rejects_requests_beyond_its_scratch(cuda_device):
    L = _lib.lib()
    Q, N, k = 4096, 33791, 512  # 553 MB of scores: far beyond the built-in scratch
    assert L.csa_index_topk_workspace_bytes(Q, N, k) > (16 << 20)
    x = torch.zeros(16, dtype=torch.int32, device=cuda_device)
    before = L.csa_launch_count()
    rc = L.csa_index_topk_noalloc(_p(x), _p(x), _p(x), _p(x), k, _p(x), Q, 1, 64, 128, N, Q, _lib.CSA_DTYPE_BF16,
                                  ctypes.c_void_p(0))
    assert rc == CSA_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.strerror(rc)
    assert L.csa_launch_count() == before  # nothing was launched


@pytest.mark.gpu
def test_noalloc_rejects_bad_arguments_before_any_work(cuda_device):
    L = _lib.lib()
    x = torch.zeros(16, dtype=torch.int32, device=cuda_device)
    before = L.csa_launch_count()
    # Hi above the limit, then a misaligned output: rejected on the host like csa_index_topk
    rc = L.csa_index_topk_noalloc(_p(x), _p(x), _p(x), _p(x), 8, _p(x), 4, 1, 129, 16, 64, 4, _lib.CSA_DTYPE_F32,
                                  ctypes.c_void_p(0))
    assert rc == 1
    rc = L.csa_index_topk_noalloc(_p(x), _p(x), _p(x), _p(x), 8, ctypes.c_void_p(x.data_ptr() + 2), 4, 1, 4, 16, 64,
                                  4, _lib.CSA_DTYPE_F32, ctypes.c_void_p(0))
    assert rc == 1
    assert L.csa_launch_count() == before
