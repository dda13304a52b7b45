"""A1 compressor: CUDA vs the fp64 oracle on seeded inputs."""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import ops, synth, workloads as WL
from helpers import assert_close, f64

pytestmark = pytest.mark.gpu


def _inputs(seed, B, T, D, win, dtype, dev, gate_scale=1.0):
    kv = synth.normal(seed, 8, (B, T, D), dtype=dtype)
    gate = synth.normal(seed, 9, (B, T, D), std=gate_scale, dtype=dtype)
    ape = synth.normal(seed, 10, (win, D), std=0.1)
    w = 0.5 + synth.uniform(seed, 11, (D,))
    return kv, gate, ape, w, [t.to(dev) for t in (kv, gate, ape, w)]


def _oracle(kv, gate, ape, w, win, stride):
    return np.stack([O.compress(kv[b], gate[b], ape, w, win, stride) for b in range(kv.shape[0])])


@pytest.mark.parametrize("B,T,D,win,stride,dtype", [
    (1, 256, 16, 8, 4, torch.float32),       # the tiny configuration
    (3, 1003, 512, 8, 4, torch.bfloat16),    # CSA, ragged tail, vectorised path
    (2, 1000, 512, 128, 128, torch.bfloat16),  # HCA geometry, partial last window dropped
    (2, 77, 100, 8, 4, torch.bfloat16),      # D not a multiple of 8: generic kernel
    (2, 300, 64, 5, 3, torch.float32),       # other window geometry
    (1, 8, 512, 8, 4, torch.bfloat16),       # exactly one window
    (4, 130, 256, 128, 128, torch.bfloat16),  # one HCA window per sequence, D = 256
    (3, 200, 512, 48, 16, torch.bfloat16),   # cluster of 3 blocks per entry, 16 positions each
    (2, 150, 512, 40, 8, torch.bfloat16),    # cluster of 2, 20 positions each (ragged over 8 groups)
    (2, 300, 512, 64, 32, torch.bfloat16),   # cluster of 4
])
def test_compress_matches_oracle(cuda_device, B, T, D, win, stride, dtype):
    kv, gate, ape, w, dev = _inputs(1, B, T, D, win, dtype, cuda_device, gate_scale=2.0)
    out = ops.compress(*dev, win, stride)
    torch.cuda.synchronize()
    ref = _oracle(kv, gate, ape, w, win, stride)
    assert out.shape == ref.shape
    assert_close(out, ref, dtype, f"compress B{B} T{T} D{D} win{win}")


def test_compress_writes_into_a_strided_cache(cuda_device):
    # The decode-time append: the newest window of each sequence's raw
    # buffer goes straight into row n-1 of each sequence's cache.
    B, Tb, D, N = 5, 128, 512, 40
    kv_buf = synth.normal(2, 3, (B, Tb, D), dtype=torch.bfloat16)
    gate = synth.normal(2, 9, (B, 8, D), dtype=torch.bfloat16)
    ape = synth.normal(2, 10, (8, D), std=0.1)
    w = torch.ones(D)
    cache = torch.zeros((B, N, D), dtype=torch.bfloat16, device=cuda_device)
    kvd = kv_buf.to(cuda_device)
    ops.compress(kvd[:, 120:128], gate.to(cuda_device), ape.to(cuda_device), w.to(cuda_device), 8, 4,
                 out=cache[:, N - 1:N])
    torch.cuda.synchronize()
    ref = _oracle(kv_buf[:, 120:128], gate, ape, w, 8, 4)
    assert_close(cache[:, N - 1:N], ref, torch.bfloat16, "append")
    assert torch.count_nonzero(cache[:, : N - 1]) == 0  # nothing else written


def test_compress_constant_kv_survives_pooling(cuda_device):
    # Constant kv along the window: the pooled vector is that constant, so
    # the output is RMSNorm(c) for any gate; exercises large gate spreads.
    B, T, D = 2, 64, 512
    c = synth.normal(3, 8, (D,))
    kv = c.expand(B, T, D).contiguous().to(torch.bfloat16)
    gate = synth.normal(3, 9, (B, T, D), std=30.0, dtype=torch.bfloat16)
    ape = synth.normal(3, 10, (8, D), std=5.0)
    w = torch.ones(D)
    out = ops.compress(kv.to(cuda_device), gate.to(cuda_device), ape.to(cuda_device), w.to(cuda_device), 8, 4)
    cb = f64(kv[0, 0])
    want = cb / np.sqrt(np.mean(cb * cb) + 1e-6)
    assert_close(out, np.broadcast_to(want, out.shape), torch.bfloat16, "constant kv")


def test_compress_full_1m_tokens_sampled(cuda_device):
    # Full size: 1,048,576 raw tokens -> 262,143 entries, in the launch
    # configuration the benchmark uses; 2,048 seeded entries + both ends
    # are checked against the oracle.
    w = WL.WORKLOADS["csa_decode_1m"]
    kv = WL.make(w, "kv_raw", cuda_device)
    gate = WL.make(w, "gate_raw", cuda_device)
    ape = WL.make(w, "ape", cuda_device)
    nw = WL.norm_w(w, cuda_device)
    out = ops.compress(kv, gate, ape, nw, 8, 4)
    torch.cuda.synchronize()
    assert out.shape == (1, 262143, 512)
    u = synth.uniform_at(7, 1, torch.arange(2048, dtype=torch.int64))
    ents = torch.unique(torch.cat([(u * 262143).long(), torch.tensor([0, 1, 262141, 262142])]))
    ape_h = WL.make(w, "ape")
    got = out[0, ents.to(cuda_device)].cpu()
    ref = []
    for j in ents.tolist():
        toks = torch.arange(4 * j, 4 * j + 8)
        ref.append(O.compress(WL.rows(w, "kv_raw", toks), WL.rows(w, "gate_raw", toks), ape_h, np.ones(512), 8, 4)[0])
    assert_close(got, np.stack(ref), torch.bfloat16, "compress 1M sampled")


@pytest.mark.parametrize("B,T,D,win,stride,dtype", [
    (3, 1003, 512, 8, 4, torch.bfloat16),     # many entries: the streaming kernel
    (32, 8, 512, 8, 4, torch.bfloat16),       # the decode append: one entry per sequence (window kernel)
    (2, 1000, 512, 128, 128, torch.bfloat16),  # HCA windows: a cluster of blocks per entry
    (2, 300, 64, 8, 4, torch.float32),        # the generic kernel (pairs split across lanes)
    (2, 100, 128, 8, 4, torch.bfloat16),      # generic kernel, bf16
])
def test_compress_rope_matches_oracle(cuda_device, B, T, D, win, stride, dtype):
    # row f3 (reading R20): the pool + RMSNorm + RoPE on the last 64 dims at
    # each entry's last-token position, with large absolute positions
    kv, gate, ape, w, dev = _inputs(5, B, T, D, win, dtype, cuda_device)
    pos0 = torch.tensor([[0, 65408 + 120, 1048448, 7][b % 4] + 3 * b for b in range(B)], dtype=torch.int64)
    rd = min(64, D)
    out = ops.compress(*dev, win, stride, rope=(rd, 160000.0, pos0.to(cuda_device)))
    torch.cuda.synchronize()
    ref = np.stack([O.compress_rope(kv[b], gate[b], ape, w, win, stride, int(pos0[b]), 160000.0, rd)
                    for b in range(B)])
    assert_close(out, ref, dtype, f"compress+rope B{B} T{T} D{D} win{win}")
    # the dims before the rope dims are exactly csa_compress's
    plain = ops.compress(*dev, win, stride)
    assert torch.equal(out[..., :D - rd], plain[..., :D - rd])
