"""The whole path chained (compress -> index/top-k -> sparse MQA), each side
running its own chain from the same seeded raw inputs; plus the device
status word for out-of-range device-side values."""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import ops, workloads as WL
from compressed_sparse_attention_15_b200.step import DecodeStep
from helpers import assert_close, check_topk_set

pytestmark = pytest.mark.gpu


def test_tiny_fp32_chain(cuda_device):
    w = WL.WORKLOADS["tiny_csa_prefill_fp32"]
    host = {t: WL.make(w, t) for t in ("q", "kv_win", "qi", "wi", "ki", "sink", "gate", "ape")}
    dev = {t: v.to(cuda_device) for t, v in host.items()}
    nw = WL.norm_w(w, cuda_device)
    kv_cmp = ops.compress(dev["kv_win"], dev["gate"], dev["ape"], nw, w.win, w.stride)
    p = w.positions()
    n = ops.visible_entries(p, w.win, w.stride)
    idx = ops.index_topk(dev["qi"], dev["wi"], dev["ki"], n.to(cuda_device), w.k)
    out = ops.sparse_mqa(dev["q"], kv_cmp, idx, dev["kv_win"], w.win_end().to(cuda_device), dev["sink"], w.scale, w.W)
    torch.cuda.synchronize()
    # oracle chain
    cmp_ref = O.compress(host["kv_win"][0], host["gate"][0], host["ape"], np.ones(w.D), w.win, w.stride)
    assert_close(kv_cmp[0], cmp_ref, torch.float32, "tiny compress")
    cmp_ref = O.round_to(cmp_ref, "fp32")  # the cache is stored in the input dtype
    idx_h = idx.cpu().numpy()
    compared = 0
    for q in range(w.Q):
        ref_idx, ref_s = O.index_topk(host["qi"][q], host["wi"][q], host["ki"][0], int(p[q]), w.k, w.win, w.stride)
        swaps = check_topk_set(idx_h[q], ref_idx, ref_s, w.k, int(n[q]))
        if swaps:
            continue  # a legitimate boundary tie: the outputs are not comparable
        ref = O.sparse_mqa(host["q"][q], cmp_ref, ref_idx, host["kv_win"][0], int(p[q]), w.W, host["sink"], w.scale)
        assert_close(out[q], ref, torch.float32, f"tiny chain q={q}")
        compared += 1
    assert compared >= w.Q - 4


def test_csa_decode_step_chain(cuda_device):
    # One decode step of the 64 K workload as the benchmark runs it: append
    # the newest window to the cache, select, attend. Checked on 8 queries.
    w = WL.WORKLOADS["csa_decode_64k"]
    d = {t: WL.make(w, t, cuda_device) for t in ("q", "kv_cmp", "kv_win", "qi", "wi", "ki", "sink", "gate", "ape")}
    nw = WL.norm_w(w, cuda_device)
    ops.compress(d["kv_win"][:, w.c_src0:w.c_src0 + w.T_c], d["gate"], d["ape"], nw, w.win, w.stride,
                 out=d["kv_cmp"][:, w.c_dst0:w.c_dst0 + 1])
    n = ops.visible_entries(w.positions().to(cuda_device), w.win, w.stride)
    idx = ops.index_topk(d["qi"], d["wi"], d["ki"], n, w.k)
    out = ops.sparse_mqa(d["q"], d["kv_cmp"], idx, d["kv_win"], w.win_end().to(cuda_device), d["sink"], w.scale, w.W)
    torch.cuda.synchronize()
    idx_h = idx.cpu().numpy()
    ape, sink = WL.make(w, "ape"), WL.make(w, "sink")
    for q in range(0, w.Q, 4):
        b = q
        ki = WL.rows(w, "ki", torch.arange(b * w.N, (b + 1) * w.N))
        ref_idx, ref_s = O.index_topk(WL.rows(w, "qi", q * w.Hi + torch.arange(w.Hi)), WL.make(w, "wi")[q], ki,
                                      w.pos0, w.k, w.win, w.stride)
        if check_topk_set(idx_h[q], ref_idx, ref_s, w.k, w.N):
            continue
        sel = ref_idx[ref_idx >= 0]
        rows_c = O.round_to(WL.rows(w, "kv_cmp", b * w.N + torch.as_tensor(sel)), "bf16")
        # the appended entry, from the raw window tokens
        raw = WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.c_src0, w.c_src0 + w.T_c))
        gate = WL.rows(w, "gate", b * w.T_c + torch.arange(w.T_c))
        new = O.round_to(O.compress(raw, gate, ape, np.ones(w.D), w.win, w.stride), "bf16")[0]
        rows_c[sel == w.c_dst0] = new
        rows_w = O.as_f64(WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.T_raw)))
        qh = WL.rows(w, "q", q * w.H + torch.arange(w.H))
        ref = O.attend(qh, np.concatenate([rows_c, rows_w]), sink, w.scale)[0]
        assert_close(out[q], ref, torch.bfloat16, f"decode chain q={q}")


def test_fp8_indexer_decode_step_chain(cuda_device):
    # The 64 K decode step with the FP8 indexer, run as one graph replay of
    # DecodeStep (append, FP8 select, attend); checked against the oracle chain
    # on four queries.
    w = WL.WORKLOADS["csa_decode_64k_fp8"]
    names = ("q", "kv_cmp", "kv_win", "sink", "gate", "ape", "qi8", "sq", "wi", "ki8", "sk")
    d = {t: WL.make(w, t, cuda_device) for t in names}
    ds = DecodeStep(q=d["q"], kv_cmp=d["kv_cmp"], kv_win=d["kv_win"], sink=d["sink"], scale=w.scale, win_len=w.W,
                    win_end=w.win_end().to(cuda_device),
                    n_cmp=ops.visible_entries(w.positions().to(cuda_device), w.win, w.stride), ape=d["ape"],
                    norm_w=WL.norm_w(w, cuda_device), gate=d["gate"], append_src0=w.c_src0, append_dst0=w.c_dst0,
                    win=w.win, stride=w.stride, qi8=d["qi8"], sq=d["sq"], wi=d["wi"], ki8=d["ki8"], sk=d["sk"],
                    k=w.k)
    out = ds.run()
    torch.cuda.synchronize()
    assert ds.status() == 0
    idx_h = ds.idx.cpu().numpy()
    ape, sink = WL.make(w, "ape"), WL.make(w, "sink")
    qi8, sq, wi = (WL.make(w, t) for t in ("qi8", "sq", "wi"))
    compared = 0
    for q in (0, 9, 18, 27):
        b = q
        rows = torch.arange(b * w.N, (b + 1) * w.N)
        ref_s = O.index_scores_fp8(qi8[q].numpy(), sq[q], wi[q], WL.rows(w, "ki8", rows).numpy(),
                                   WL.rows(w, "sk", rows), w.N)
        ref_idx = O.topk(ref_s, w.k)
        if check_topk_set(idx_h[q], ref_idx, ref_s, w.k, w.N):
            continue
        sel = ref_idx[ref_idx >= 0]
        rows_c = O.round_to(WL.rows(w, "kv_cmp", b * w.N + torch.as_tensor(sel)), "bf16")
        raw = WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.c_src0, w.c_src0 + w.T_c))
        gate = WL.rows(w, "gate", b * w.T_c + torch.arange(w.T_c))
        rows_c[sel == w.c_dst0] = O.round_to(O.compress(raw, gate, ape, np.ones(w.D), w.win, w.stride), "bf16")[0]
        rows_w = O.as_f64(WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.T_raw)))
        qh = WL.rows(w, "q", q * w.H + torch.arange(w.H))
        ref = O.attend(qh, np.concatenate([rows_c, rows_w]), sink, w.scale)[0]
        assert_close(out[q], ref, torch.bfloat16, f"FP8 decode chain q={q}")
        compared += 1
    assert compared >= 3


def test_status_word_flags_bad_device_values(cuda_device):
    # Out-of-range counts, indices and window ends are clamped/skipped on the
    # device and reported through the workspace status word; no fault.
    Q, B, N, T_raw, H, D = 4, 1, 50, 20, 4, 16
    q = torch.randn(Q, H, D, device=cuda_device)
    kv = torch.randn(B, N, D, device=cuda_device)
    kw = torch.randn(B, T_raw, D, device=cuda_device)
    sink = torch.zeros(H, device=cuda_device)
    ws = ops.Workspace(cuda_device)
    idx = torch.tensor([[0, 1, 2, 3]] * Q, dtype=torch.int32, device=cuda_device)
    idx[1, 2] = N + 5
    idx[2, 0] = -7
    we = torch.tensor([0, 5, 19, 3], dtype=torch.int32, device=cuda_device)
    ops.sparse_mqa(q, kv, idx, kw, we, sink, 0.25, 4, q_per_seq=Q, ws=ws)
    assert ws.status() == 2  # CSA_STATUS_BAD_INDEX
    we[3] = T_raw + 1
    ops.sparse_mqa(q, kv, torch.zeros_like(idx), kw, we, sink, 0.25, 4, q_per_seq=Q, ws=ws)
    assert ws.status() == 4  # CSA_STATUS_BAD_WINDOW
    n = torch.tensor([N, N + 1, -1, 3], dtype=torch.int32, device=cuda_device)
    ops.hca_mqa(q, kv, n, kw, torch.zeros_like(we), sink, 0.25, 4, q_per_seq=Q, ws=ws)
    assert ws.status() == 1  # CSA_STATUS_BAD_COUNT
    qi = torch.randn(Q, 4, 16, device=cuda_device)
    ki = torch.randn(B, N, 16, device=cuda_device)
    ops.index_topk(qi, torch.rand(Q, 4, device=cuda_device), ki, n, 8, q_per_seq=Q, ws=ws)
    assert ws.status() == 1
    ops.sparse_mqa(q, kv, torch.zeros_like(idx), kw, torch.zeros_like(we), sink, 0.25, 4, q_per_seq=Q, ws=ws)
    assert ws.status() == 0
    torch.cuda.synchronize()
