"""A4 sparse MQA and A5 HCA MQA: CUDA vs the fp64 oracle.

The index lists fed to both sides are seeded inputs (not a GPU selection),
so a legitimate tie swap in top-k can never fail an attention check."""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import ops, synth, workloads as WL
from helpers import assert_close, seeded_idx

pytestmark = pytest.mark.gpu


def _mqa_inputs(seed, Q, B, N, T_raw, H, D, dtype):
    q = synth.normal(seed, 1, (Q, H, D), dtype=dtype)
    kv_cmp = synth.normal(seed, 2, (B, N, D), dtype=dtype)
    kv_win = synth.normal(seed, 3, (B, T_raw, D), dtype=dtype)
    sink = synth.normal(seed, 7, (H,))
    return q, kv_cmp, kv_win, sink


def _dev(cuda_device, *ts):
    return [t.to(cuda_device) for t in ts]


@pytest.mark.parametrize("Q,B,N,T_raw,H,D,k,W,dtype", [
    (256, 1, 63, 256, 4, 16, 16, 16, torch.float32),     # tiny: causal positions 0..255
    (6, 3, 2000, 200, 64, 512, 512, 128, torch.bfloat16),  # Flash shape, multi-sequence
    (5, 5, 3000, 128, 64, 512, 1024, 128, torch.bfloat16),
    (4, 2, 100, 64, 64, 512, 40, 128, torch.bfloat16),   # window clipped by T_raw/sequence start
    (3, 1, 50, 30, 8, 64, 7, 5, torch.bfloat16),         # small odd shapes (generic kernel)
    (4, 4, 300, 40, 64, 512, 200, 16, torch.float32),
    (4, 2, 2000, 200, 128, 512, 1024, 128, torch.bfloat16),  # V4-Pro: 128 heads (two 64-head groups), top-1024
    # 16+ queries: one CTA per (query, 64 heads) walking all of the query's tiles
    (16, 4, 2000, 200, 64, 512, 512, 128, torch.bfloat16),
    (18, 6, 100, 64, 64, 512, 40, 128, torch.bfloat16),   # one selected tile, windows clipped
    (16, 2, 2000, 200, 128, 512, 1024, 128, torch.bfloat16),  # 128 heads, 18 tiles per query
])
def test_sparse_mqa_matches_oracle(cuda_device, Q, B, N, T_raw, H, D, k, W, dtype):
    q, kv_cmp, kv_win, sink = _mqa_inputs(1, Q, B, N, T_raw, H, D, dtype)
    qps = Q // B
    # ragged selections: full, partially padded, empty
    n_sel = [[k, k // 2, 0, 1][i % 4] for i in range(Q)]
    idx = seeded_idx(5, Q, N, k, n_sel)
    win_end = torch.tensor([(T_raw - 1 - 3 * i) % T_raw for i in range(Q)], dtype=torch.int32)
    if Q == 256:
        win_end = torch.arange(256, dtype=torch.int32)
    scale = 1.0 / np.sqrt(D)
    out = ops.sparse_mqa(*_dev(cuda_device, q, kv_cmp, idx, kv_win, win_end, sink), scale, W, q_per_seq=qps)
    torch.cuda.synchronize()
    ref = np.stack([O.sparse_mqa(q[i], kv_cmp[i // qps], idx[i].numpy(), kv_win[i // qps], int(win_end[i]), W,
                                 sink, scale) for i in range(Q)])
    assert_close(out, ref, dtype, f"sparse_mqa Q{Q} H{H} D{D} k{k}")


@pytest.mark.parametrize("Q,B,N,T_raw,H,D,W,dtype", [
    (8, 8, 1000, 128, 64, 512, 128, torch.bfloat16),
    (6, 2, 333, 150, 64, 512, 128, torch.bfloat16),
    (16, 1, 40, 64, 4, 16, 16, torch.float32),
    (5, 5, 700, 128, 128, 512, 128, torch.bfloat16),    # V4-Pro: 128 heads
])
def test_hca_mqa_matches_oracle(cuda_device, Q, B, N, T_raw, H, D, W, dtype):
    q, kv_cmp, kv_win, sink = _mqa_inputs(2, Q, B, N, T_raw, H, D, dtype)
    qps = Q // B
    n_cmp = torch.tensor([[N, 0, 1, N // 3][i % 4] for i in range(Q)], dtype=torch.int32)
    win_end = torch.tensor([(T_raw - 1 - 5 * i) % T_raw for i in range(Q)], dtype=torch.int32)
    scale = 1.0 / np.sqrt(D)
    out = ops.hca_mqa(*_dev(cuda_device, q, kv_cmp, n_cmp, kv_win, win_end, sink), scale, W, q_per_seq=qps)
    torch.cuda.synchronize()
    ref = np.stack([O.hca_mqa(q[i], kv_cmp[i // qps], int(n_cmp[i]), kv_win[i // qps], int(win_end[i]), W, sink,
                              scale) for i in range(Q)])
    assert_close(out, ref, dtype, f"hca_mqa Q{Q} N{N}")


def test_sparse_with_all_entries_equals_hca(cuda_device):
    # top-k covering every visible entry == dense HCA attention (GPU vs GPU
    # and both vs the oracle).
    Q, B, N, T_raw, H, D = 4, 2, 700, 128, 64, 512
    q, kv_cmp, kv_win, sink = _mqa_inputs(3, Q, B, N, T_raw, H, D, torch.bfloat16)
    idx = torch.arange(N, dtype=torch.int32).repeat(Q, 1)
    n_cmp = torch.full((Q,), N, dtype=torch.int32)
    we = torch.full((Q,), T_raw - 1, dtype=torch.int32)
    a = ops.sparse_mqa(*_dev(cuda_device, q, kv_cmp, idx, kv_win, we, sink), 0.04, 128)
    b = ops.hca_mqa(*_dev(cuda_device, q, kv_cmp, n_cmp, kv_win, we, sink), 0.04, 128)
    ref = np.stack([O.hca_mqa(q[i], kv_cmp[i // 2], N, kv_win[i // 2], T_raw - 1, 128, sink, 0.04) for i in range(Q)])
    assert_close(a, ref, torch.bfloat16, "sparse(all)")
    assert_close(b, ref, torch.bfloat16, "hca")


@pytest.mark.parametrize("mode,Q", [("sparse", 3), ("hca", 3), ("sparse", 16)])
def test_mqa_growing_logits_force_running_max_updates(cuda_device, mode, Q):
    # Row norms grow along the row list and the softmax scale is large, so
    # later 128-row tiles raise the per-head running maximum far past the
    # first tile's: exercises the deferred rescaling of the accumulator.
    B, N, T_raw, H, D, k, W = Q, 900, 128, 64, 512, 768, 128
    q, kv_cmp, kv_win, sink = _mqa_inputs(6, Q, B, N, T_raw, H, D, torch.float32)
    grow = torch.linspace(0.2, 2.0, N).reshape(1, N, 1)
    kv_cmp = (kv_cmp * grow).to(torch.bfloat16)
    q, kv_win = q.to(torch.bfloat16), kv_win.to(torch.bfloat16)
    scale = 0.15
    we = torch.full((Q,), T_raw - 1, dtype=torch.int32)
    if mode == "sparse":
        idx = torch.arange(k, dtype=torch.int32).repeat(Q, 1)  # ascending: norms grow tile by tile
        out = ops.sparse_mqa(*_dev(cuda_device, q, kv_cmp, idx, kv_win, we, sink), scale, W)
        ref = [O.sparse_mqa(q[i], kv_cmp[i], idx[i].numpy(), kv_win[i], T_raw - 1, W, sink, scale) for i in range(Q)]
    else:
        n = torch.tensor([N, N // 2, 300][:Q], dtype=torch.int32)
        out = ops.hca_mqa(*_dev(cuda_device, q, kv_cmp, n, kv_win, we, sink), scale, W)
        ref = [O.hca_mqa(q[i], kv_cmp[i], int(n[i]), kv_win[i], T_raw - 1, W, sink, scale) for i in range(Q)]
    torch.cuda.synchronize()
    assert_close(out, np.stack(ref), torch.bfloat16, f"growing logits {mode}")


def test_sink_at_minus_inf_without_entries_is_window_attention(cuda_device):
    Q, D, H, W = 40, 16, 4, 16
    q, _, kv_win, _ = _mqa_inputs(4, Q, 1, 1, Q, H, D, torch.float32)
    sink = torch.full((H,), -float("inf"))
    idx = torch.full((Q, 8), -1, dtype=torch.int32)
    we = torch.arange(Q, dtype=torch.int32)
    out = ops.sparse_mqa(*_dev(cuda_device, q, torch.zeros(1, 1, D), idx, kv_win, we, sink), 0.25, W, q_per_seq=Q)
    ref = np.stack([O.sparse_mqa(q[i], np.zeros((1, D)), idx[i].numpy(), kv_win[0], i, W, sink, 0.25)
                    for i in range(Q)])
    assert_close(out, ref, torch.float32, "window only")


@pytest.mark.parametrize("name", ["csa_decode_64k", "csa_decode_1m", "csa_prefill_chunk_4k"])
def test_sparse_mqa_full_size(cuda_device, name):
    w = WL.WORKLOADS[name]
    q, kv_cmp, kv_win, sink = (WL.make(w, t, cuda_device) for t in ("q", "kv_cmp", "kv_win", "sink"))
    n = ops.visible_entries(w.positions(), w.win, w.stride)
    idx = seeded_idx(9, w.Q, w.N, w.k, n_vis=n)
    we = w.win_end()
    out = ops.sparse_mqa(q, kv_cmp, idx.to(cuda_device), kv_win, we.to(cuda_device), sink, w.scale, w.W,
                         q_per_seq=w.q_per_seq)
    torch.cuda.synchronize()
    del kv_cmp
    qs = np.unique(np.linspace(0, w.Q - 1, min(w.Q, 32)).round().astype(int))
    sink_h = WL.make(w, "sink")
    got, ref = [], []
    for i in qs:
        b = int(i) // w.q_per_seq
        sel = idx[i][idx[i] >= 0].long()
        rows_c = WL.rows(w, "kv_cmp", b * w.N + sel)
        e = int(we[i])
        lo = max(0, e - w.W + 1)
        rows_w = WL.rows(w, "kv_win", b * w.T_raw + torch.arange(lo, e + 1))
        qi = WL.rows(w, "q", int(i) * w.H + torch.arange(w.H))
        rows = torch.cat([rows_c, rows_w])
        ref.append(O.attend(qi, rows, sink_h, w.scale)[0])
        got.append(out[i].cpu())
    assert_close(torch.stack(got), np.stack(ref), w.dtype, f"{name} sparse_mqa")


def test_hca_mqa_full_size(cuda_device):
    w = WL.WORKLOADS["hca_decode_1m"]
    q, kv_cmp, kv_win, sink = (WL.make(w, t, cuda_device) for t in ("q", "kv_cmp", "kv_win", "sink"))
    n = ops.visible_entries(w.positions(), w.win, w.stride)
    assert int(n[0]) == w.N
    we = w.win_end()
    out = ops.hca_mqa(q, kv_cmp, n.to(cuda_device), kv_win, we.to(cuda_device), sink, w.scale, w.W)
    torch.cuda.synchronize()
    sink_h = WL.make(w, "sink")
    got, ref = [], []
    for i in range(w.Q):
        rows_c = WL.rows(w, "kv_cmp", torch.arange(i * w.N, (i + 1) * w.N))
        rows_w = WL.rows(w, "kv_win", torch.arange(i * w.T_raw, (i + 1) * w.T_raw))
        qi = WL.rows(w, "q", i * w.H + torch.arange(w.H))
        ref.append(O.attend(qi, torch.cat([rows_c, rows_w]), sink_h, w.scale)[0])
        got.append(out[i].cpu())
    assert_close(torch.stack(got), np.stack(ref), w.dtype, "hca full")
