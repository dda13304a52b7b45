"""The Python binding marshals arguments only: every entry point refuses host
(CPU) tensors with an error instead of computing anything itself, so there is
no CPU fallback behind the C ABI. Runs without a GPU."""
import pytest
import torch

from compressed_sparse_attention_15_b200 import ops

f32, bf16, i32, u8 = torch.float32, torch.bfloat16, torch.int32, torch.uint8


def z(*shape, dtype=bf16):
    return torch.zeros(shape, dtype=dtype)


CALLS = {
    "compress": lambda: ops.compress(z(1, 16, 8), z(1, 16, 8), z(8, 8, dtype=f32), z(8, dtype=f32), 8, 4),
    "index_compress": lambda: ops.index_compress(z(1, 16, 64), z(1, 16, 64), z(8, 64, dtype=f32),
                                                 z(64, dtype=f32), 8, 4),
    "hadamard_rows": lambda: ops.hadamard_rows(z(4, 64)),
    "index_scores": lambda: ops.index_scores(z(2, 4, 16), z(2, 4, dtype=f32), z(1, 32, 16), z(2, dtype=i32)),
    "index_topk": lambda: ops.index_topk(z(2, 4, 16), z(2, 4, dtype=f32), z(1, 32, 16), z(2, dtype=i32), 8),
    "topk": lambda: ops.topk(z(2, 32, dtype=f32), z(2, dtype=i32), 8),
    "index_topk_fp8": lambda: ops.index_topk_fp8(z(2, 4, 16, dtype=u8), z(2, 4, dtype=f32), z(2, 4, dtype=f32),
                                                 z(1, 32, 16, dtype=u8), z(1, 32, dtype=f32), z(2, dtype=i32), 8),
    "sparse_mqa": lambda: ops.sparse_mqa(z(2, 4, 16), z(1, 32, 16), z(2, 8, dtype=i32), z(1, 16, 16),
                                         z(2, dtype=i32), z(4, dtype=f32), 0.25, 16),
    "topk_sparse_mqa": lambda: ops.topk_sparse_mqa(z(2, 32, dtype=f32), z(2, dtype=i32), 8, z(2, 4, 16),
                                                   z(1, 32, 16), z(1, 16, 16), z(2, dtype=i32), z(4, dtype=f32),
                                                   0.25, 16),
    "hca_mqa": lambda: ops.hca_mqa(z(2, 4, 16), z(1, 32, 16), z(2, dtype=i32), z(1, 16, 16), z(2, dtype=i32),
                                   z(4, dtype=f32), 0.25, 16),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused(name):
    with pytest.raises(ValueError, match="CUDA tensor"):
        CALLS[name]()
