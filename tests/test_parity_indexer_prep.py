"""Row f2 (reading R19): the indexer's own compressor (pool + RMSNorm +
Hadamard rotation), the query rotation and their FP8 encodings, against the
fp64 oracle; and the whole FP8 indexer chain from raw indexer KV to top-k."""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import ops, synth
from helpers import assert_close, f64

pytestmark = pytest.mark.gpu


def _raw(seed, B, T, D, win, dtype):
    kv = synth.normal(seed, 21, (B, T, D), dtype=dtype)
    gate = synth.normal(seed, 22, (B, T, D), dtype=dtype)
    ape = synth.normal(seed, 23, (win, D), std=0.1)
    norm_w = 0.5 + synth.uniform(seed, 24, (D,))
    return kv, gate, ape, norm_w


def _check_codes(codes, scales, x_exact, what):
    """GPU E4M3 rows vs the exact rows: scales within fp32 rounding of
    amax / 448, every value within half an E4M3 step (plus fp32 slack) of the
    exact value, and almost all codes equal to the oracle's own encoding."""
    codes = codes.cpu().numpy().reshape(-1, x_exact.shape[-1])
    scales = f64(scales).reshape(-1)
    x = x_exact.reshape(-1, x_exact.shape[-1])
    want_codes, want_scales = O.quantize_rows_e4m3(x)
    assert np.allclose(scales, want_scales, rtol=1e-5, atol=0), f"{what}: scales"
    deq = O.e4m3_decode(codes) * scales[:, None]
    step = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scales[:, None])  # half the E4M3 spacing
    assert np.all(np.abs(deq - x) <= step * (1 + 1e-3) + 1e-6 * np.abs(x)), f"{what}: values"
    same = np.mean(codes == want_codes)
    assert same >= 0.995, f"{what}: only {same:.4f} of the codes match the oracle's encoding"
    # a differing code is the neighbour of the oracle's (a rounding-boundary case)
    diff = codes != want_codes
    if diff.any():
        a, b = O.e4m3_decode(codes[diff]), O.e4m3_decode(want_codes[diff])
        nb = np.abs(a - b) <= np.maximum(np.abs(b) * 2.0 ** -3, 2.0 ** -9) * 1.0001
        assert nb.all(), f"{what}: codes more than one step apart"


@pytest.mark.parametrize("B,T,D,dtype", [
    (3, 1003, 128, torch.bfloat16),   # the indexer head dim, ragged tail
    (2, 300, 64, torch.float32),
    (1, 8, 256, torch.bfloat16),      # exactly one window
    (2, 200, 512, torch.bfloat16),
])
def test_index_compress_matches_oracle(cuda_device, B, T, D, dtype):
    kv, gate, ape, nw = _raw(1, B, T, D, 8, dtype)
    d = lambda t: t.to(cuda_device)
    out = ops.index_compress(d(kv), d(gate), d(ape), d(nw), 8, 4)
    ref = np.stack([O.index_compress(kv[b], gate[b], ape, nw, 8, 4) for b in range(B)])
    assert_close(out, ref, dtype, "index_compress")
    codes, scales = ops.index_compress(d(kv), d(gate), d(ape), d(nw), 8, 4, fp8=True)
    _check_codes(codes, scales, ref, "index_compress fp8")


@pytest.mark.parametrize("R,D,dtype", [(64 * 7, 128, torch.bfloat16), (33, 64, torch.float32), (5, 512, torch.bfloat16)])
def test_hadamard_rows_match_oracle(cuda_device, R, D, dtype):
    x = synth.normal(2, 25, (R, D), dtype=dtype)
    x[3] = 0  # a zero row: scale 1, all codes zero
    out = ops.hadamard_rows(x.to(cuda_device))
    ref = O.hadamard_rotate(x)
    assert_close(out, ref, dtype, "hadamard_rows")
    codes, scales = ops.hadamard_rows(x.to(cuda_device), fp8=True)
    _check_codes(codes, scales, ref, "hadamard_rows fp8")
    assert float(scales[3]) == 1.0 and int((codes[3].cpu() & 0x7F).sum()) == 0


def test_fp8_indexer_chain_from_raw_kv(cuda_device):
    # raw indexer KV -> compressor + rotation + FP8 (f2) -> FP8 scores + top-k
    # (f1), each side on its own; queries rotated and encoded the same way.
    B, T, D, Hi, k = 2, 8192, 128, 64, 256
    kv, gate, ape, nw = _raw(3, B, T, D, 8, torch.bfloat16)
    qi = synth.normal(3, 26, (B, Hi, D), dtype=torch.bfloat16)
    wi = synth.uniform(3, 27, (B, Hi))
    d = lambda t: t.to(cuda_device)
    ki8, sk = ops.index_compress(d(kv), d(gate), d(ape), d(nw), 8, 4, fp8=True)
    qi8, sq = ops.hadamard_rows(d(qi), fp8=True)
    N = ki8.shape[1]
    n = torch.full((B,), N, dtype=torch.int32, device=cuda_device)
    idx = ops.index_topk_fp8(qi8, sq, d(wi), ki8, sk, n, k).cpu().numpy()
    for b in range(B):
        ki_o, sk_o = O.quantize_rows_e4m3(O.index_compress(kv[b], gate[b], ape, nw, 8, 4))
        qi_o, sq_o = O.quantize_rows_e4m3(O.hadamard_rotate(qi[b]))
        s = O.index_scores_fp8(qi_o, sq_o, wi[b], ki_o, sk_o, N)
        ref = set(O.topk(s, k).tolist())
        got = set(idx[b].tolist())
        # the two sides' codes may differ by one step on rounding-boundary
        # values; swaps are only allowed near the k-th score
        kth = np.sort(s)[::-1][k - 1]
        for j in got ^ ref:
            assert abs(s[j] - kth) <= 0.02 * abs(kth), f"seq {b}: entry {j} far from the selection boundary"
        assert len(got & ref) >= k - 8
