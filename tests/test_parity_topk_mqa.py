"""A3 + A4 in one call (csa_topk_sparse_mqa): the top-k of given indexer
scores, selected inside the attention kernel where the launch plan allows,
against the fp64 oracle's selection and attention."""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import _lib, ops, synth, workloads as WL
from helpers import assert_close, check_topk_set

pytestmark = pytest.mark.gpu

SCORES_TID = 40  # seeded stream of the synthetic indexer scores


def _scores(w, ties=False):
    s = synth.normal(w.seed, SCORES_TID, (w.Q, w.N))
    if ties:  # a coarse grid: long runs of equal scores at every boundary
        s = torch.round(s * 4) / 4
    return s


def _w(**changes):
    """A variant of the 64K decode batch; the raw window buffer is placed so
    that every query's own token lies in it."""
    w = WL.small(BASE, **changes)
    return WL.small(w, raw0=w.pos0 - (w.T_raw - w.q_per_seq))


def _case(cuda_device, w, n, ties=False, check_every=1, launches=None):
    """Runs the call, checks every selection against the oracle's and the
    output of every check_every-th query; returns how many outputs were
    compared. launches: the expected number of kernels the call launches."""
    scores = _scores(w, ties)
    d = {t: WL.make(w, t, cuda_device) for t in ("q", "kv_cmp", "kv_win", "sink")}
    n = torch.as_tensor(n, dtype=torch.int32)
    win_end = w.win_end()
    args = (scores.to(cuda_device), n.to(cuda_device), w.k, d["q"], d["kv_cmp"], d["kv_win"], win_end.to(cuda_device),
            d["sink"], w.scale, w.W)
    ws = ops.Workspace(cuda_device)
    ops.topk_sparse_mqa(*args, q_per_seq=w.q_per_seq, ws=ws)  # sizes the workspace
    before = _lib.lib().csa_launch_count()
    out, idx = ops.topk_sparse_mqa(*args, q_per_seq=w.q_per_seq, ws=ws)
    n_launch = _lib.lib().csa_launch_count() - before
    if launches is not None:
        assert launches(n_launch), f"{n_launch} kernel launches"
    # the same selection through the stand-alone top-k kernel
    idx_sep = ops.topk(scores.to(cuda_device), n.to(cuda_device), w.k)
    torch.cuda.synchronize()
    del d
    idx_h, out_h = idx.cpu().numpy(), out.cpu()
    assert np.array_equal(idx_h, idx_sep.cpu().numpy()), "fused and stand-alone selections differ"
    sink = WL.make(w, "sink")
    compared = 0
    for q in range(w.Q):
        nv, b = int(n[q]), q // w.q_per_seq
        s = O.as_f64(scores[q, :nv])
        ref_idx = O.topk(s, w.k)
        if check_topk_set(idx_h[q], ref_idx, s, w.k, nv) or q % check_every:
            continue
        sel = np.sort(ref_idx[ref_idx >= 0])
        rows_c = O.as_f64(WL.rows(w, "kv_cmp", b * w.N + torch.as_tensor(sel, dtype=torch.int64)))
        kv_win_b = WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.T_raw))
        rows = np.concatenate([rows_c.reshape(-1, w.D), O.window_rows(kv_win_b, int(win_end[q]), w.W)])
        qh = WL.rows(w, "q", q * w.H + torch.arange(w.H))
        ref = O.attend(qh, rows, sink, w.scale)[0]
        assert_close(out_h[q], ref, w.dtype, f"query {q} (n={nv})")
        compared += 1
    return compared


BASE = WL.WORKLOADS["csa_decode_64k"]


def test_full_size_decode_batch(cuda_device):
    # The 64K-context decode batch in the benchmark's launch configuration
    # (32 queries, 16,383 entries each, clusters of 4): every selection and
    # every output against the oracle.
    w = BASE
    assert _case(cuda_device, w, [w.N] * w.Q, launches=lambda c: c == 1) >= w.Q - 2


def test_pro_shape_128_heads_top_1024(cuda_device):
    w = WL.WORKLOADS["csa_decode_64k_pro"]
    assert _case(cuda_device, w, [w.N] * w.Q, check_every=4, launches=lambda c: c == 1) >= w.Q // 4 - 1


@pytest.mark.parametrize("Q,B,N,k", [
    (16, 4, 3000, 512),  # clusters of 5
    (8, 2, 3000, 256),   # clusters of up to 10 (where resident): slices of 32 leave some CTAs empty at n = k + 1
    (6, 3, 1001, 256),
])
def test_ragged_visible_counts(cuda_device, Q, B, N, k):
    # n below, at and just above k, zero and one entry, and the full list:
    # the n <= k queries take the no-selection branch in every CTA. (The
    # launch plan, fused or not, depends on cluster residency; both are
    # checked against the oracle.)
    w = _w(seed=5, Q=Q, B=B, N=N, k=k)
    n = [[N, k + 1, k, 0, 1, N - 1, 600, 1000][q % 8] for q in range(Q)]
    n = [min(v, N) for v in n]
    assert _case(cuda_device, w, n) >= Q - 1


def test_ties_resolve_to_the_smaller_index(cuda_device):
    # Scores on a coarse grid: many entries equal the k-th score and the
    # selection must keep the smallest indices among them, exactly.
    w = _w(seed=6, Q=8, B=8, N=4000, k=512)
    scores = _scores(w, ties=True)
    n = torch.full((w.Q,), w.N, dtype=torch.int32)
    d = {t: WL.make(w, t, cuda_device) for t in ("q", "kv_cmp", "kv_win", "sink")}
    _, idx = ops.topk_sparse_mqa(scores.to(cuda_device), n.to(cuda_device), w.k, d["q"], d["kv_cmp"], d["kv_win"],
                                 w.win_end().to(cuda_device), d["sink"], w.scale, w.W)
    idx_h = idx.cpu().numpy()
    for q in range(w.Q):
        ref = O.topk(O.as_f64(scores[q]), w.k)
        assert np.array_equal(idx_h[q], np.sort(ref)), f"query {q}"
    # the case is only meaningful when the boundary score is shared
    s0 = O.as_f64(scores[0])
    kth = s0[O.topk(s0, w.k)[-1]]
    assert np.sum(s0 == kth) > 1


def test_many_queries_take_the_two_kernel_path(cuda_device):
    # More queries than a cluster per query allows: the call runs the
    # stand-alone top-k, then the attention; the results are the same.
    w = _w(seed=7, Q=160, B=4, N=2000, k=64, W=16)
    assert _case(cuda_device, w, [w.N - (q % 5) * 300 for q in range(w.Q)], check_every=8,
                 launches=lambda c: c >= 2) >= 18


def test_decode_step_with_the_fused_selection(cuda_device):
    # DecodeStep(fuse_select=True), replayed from its CUDA graph on the 64K
    # decode batch: indexer scores, then the selection made inside the
    # attention kernel. The selections of 8 queries against the oracle's
    # indexer top-k, and their outputs against the oracle attention.
    from compressed_sparse_attention_15_b200.step import DecodeStep

    w = BASE
    d = {t: WL.make(w, t, cuda_device) for t in ("q", "kv_cmp", "kv_win", "qi", "wi", "ki", "sink", "gate", "ape")}
    n = ops.visible_entries(w.positions(), w.win, w.stride)
    ds = DecodeStep(q=d["q"], kv_cmp=d["kv_cmp"], kv_win=d["kv_win"], sink=d["sink"], scale=w.scale, win_len=w.W,
                    win_end=w.win_end().to(cuda_device), n_cmp=n.to(cuda_device), ape=d["ape"],
                    norm_w=WL.norm_w(w, cuda_device), gate=d["gate"], append_src0=w.c_src0, append_dst0=w.c_dst0,
                    win=w.win, stride=w.stride, qi=d["qi"], wi=d["wi"], ki=d["ki"], k=w.k, fuse_select=True,
                    fused=False)
    out = ds.run().cpu()
    assert ds.status() == 0
    idx_h = ds.idx.cpu().numpy()
    del d, ds
    ape, sink, wi = WL.make(w, "ape"), WL.make(w, "sink"), WL.make(w, "wi")
    compared = 0
    for q in range(0, w.Q, 4):
        b = q
        ki = WL.rows(w, "ki", torch.arange(b * w.N, (b + 1) * w.N))
        ref_idx, ref_s = O.index_topk(WL.rows(w, "qi", q * w.Hi + torch.arange(w.Hi)), wi[q], ki, w.pos0, w.k,
                                      w.win, w.stride)
        if check_topk_set(idx_h[q], ref_idx, ref_s, w.k, int(n[q])):
            continue
        sel = np.sort(ref_idx[ref_idx >= 0])
        rows_c = O.as_f64(WL.rows(w, "kv_cmp", b * w.N + torch.as_tensor(sel, dtype=torch.int64)))
        # the entry the step appended, from the raw window tokens
        raw = WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.c_src0, w.c_src0 + w.T_c))
        gate = WL.rows(w, "gate", b * w.T_c + torch.arange(w.T_c))
        new = O.round_to(O.compress(raw, gate, ape, np.ones(w.D), w.win, w.stride), "bf16")[0]
        rows_c[sel == w.c_dst0] = new
        rows_w = O.window_rows(WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.T_raw)), int(w.win_end()[q]), w.W)
        qh = WL.rows(w, "q", q * w.H + torch.arange(w.H))
        ref = O.attend(qh, np.concatenate([rows_c, rows_w]), sink, w.scale)[0]
        assert_close(out[q], ref, torch.bfloat16, f"fused decode step q={q}")
        compared += 1
    assert compared >= 6
