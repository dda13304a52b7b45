"""A2 indexer scores and A3 top-k: CUDA vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import ops, synth, workloads as WL
from helpers import check_topk_set, f64

pytestmark = pytest.mark.gpu


def _score_inputs(seed, Q, B, N, Hi, Di, dtype):
    qi = synth.normal(seed, 4, (Q, Hi, Di), dtype=dtype)
    wi = synth.uniform(seed, 5, (Q, Hi))
    ki = synth.normal(seed, 6, (B, N, Di), dtype=dtype)
    return qi, wi, ki


@pytest.mark.parametrize("Q,B,N,Hi,Di,dtype", [
    (256, 1, 63, 4, 16, torch.float32),      # the tiny configuration
    (6, 3, 1000, 64, 128, torch.bfloat16),   # Flash indexer shape, ragged tail
    (5, 5, 300, 8, 32, torch.bfloat16),
    (4, 2, 129, 64, 128, torch.float32),
    (16, 2, 1000, 64, 128, torch.bfloat16),  # 8 queries per sequence: groups of 4 share each key tile
    (8, 1, 129, 64, 128, torch.bfloat16),    # one group pair over a full tile + 1 entry
])
def test_index_scores_match_oracle(cuda_device, Q, B, N, Hi, Di, dtype):
    qi, wi, ki = _score_inputs(1, Q, B, N, Hi, Di, dtype)
    qps = Q // B
    # ragged visible counts, including 0, 1 and N
    n = torch.tensor([[N, 0, 1, N - 1, N // 2, 17][q % 6] for q in range(Q)], dtype=torch.int32)
    s = ops.index_scores(qi.to(cuda_device), wi.to(cuda_device), ki.to(cuda_device), n.to(cuda_device),
                         q_per_seq=qps).cpu()
    for q in range(Q):
        nv = int(n[q])
        ref = O.index_scores(qi[q], wi[q], ki[q // qps], nv)
        got = f64(s[q, :nv])
        scale = max(np.abs(ref).max(initial=0.0), 1.0)
        assert np.max(np.abs(got - ref), initial=0.0) <= 2e-5 * scale * (1 if dtype == torch.float32 else 5)
        assert torch.isnan(s[q, nv:]).all()  # untouched beyond the visible count


@pytest.mark.parametrize("N,k", [(1, 1), (100, 100), (101, 100), (1000, 16), (5000, 512), (20000, 2048),
                                 (49153, 512), (100000, 2048), (262143, 1024), (300000, 64)])
def test_topk_exact_on_given_scores(cuda_device, N, k):
    # (from 49153 entries up the selection is two-stage: segments, then a merge)
    # Both sides select from the same fp32 scores: bit-exact index sets.
    # Scores are quantised so that ties (including +0 / -0) are frequent.
    Q = 3
    u = synth.uniform(4, 12, (Q, N))
    s = torch.floor(u * 50) - 25.0
    s[s == 0] = -0.0
    s[1] = u[1]                          # a row without ties
    n = torch.tensor([N, max(0, N - 7), N // 2], dtype=torch.int32)
    got = ops.topk(s.to(cuda_device), n.to(cuda_device), k).cpu().numpy()
    for q in range(Q):
        nv = int(n[q])
        want = O.topk(f64(s[q, :nv]), k)
        m = min(k, nv)
        assert np.array_equal(np.sort(want[:m]), got[q, :m]), f"query {q}"
        assert np.all(got[q, m:] == -1)


@pytest.mark.parametrize("Q,N,k,shape", [
    (32, 16383, 512, "one CTA per query, 16 keys per thread in registers (64K-context decode batch)"),
    (3, 2000, 64, "one CTA per query, 4 keys per thread in registers"),
    (100, 5000, 512, "one CTA per query, 8 keys per thread in registers"),
    (8, 262143, 1024, "cluster of 8 CTAs per query, 32K entries each (1M-context decode batch)"),
    (5, 30000, 512, "cluster of 8, a short last slice"),
    (8, 262143, 64, "cluster of 8 sampling and filtering, a small k"),
    (100, 20000, 512, "one CTA per query, sample and filter over keys cached in shared memory"),
    (200, 33791, 512, "sample and filter over cached keys, the prefill chunk's list length"),
    (150, 40960, 2048, "sample and filter over cached keys, the longest such list"),
    (100, 60000, 64, "two stages: segment winners, then a merge"),
    (76, 1 << 20, 2048, "one CTA per query re-reading the scores (winners too many to merge)"),
])
def test_topk_every_launch_shape(cuda_device, Q, N, k, shape):
    # The launch shape follows from (Q, N, k) and the GPU's 148 SMs. Scores
    # are drawn on the device; the checked rows are drawn again on the host.
    u = synth.uniform(5, 13, (Q, N), device=cuda_device)
    s = torch.floor(u * 4096) - 2048.0              # ties at every threshold
    n = torch.tensor([N - (q % 5) * 3 for q in range(Q)], dtype=torch.int32)
    n[1] = min(N, k + 1)                             # just above k: one entry dropped
    got = ops.topk(s, n.to(cuda_device), k).cpu().numpy()
    del u, s
    for q in sorted({0, 1, Q // 2, Q - 1}):
        nv = int(n[q])
        row = synth.uniform_at(5, 13, q * N + torch.arange(nv, dtype=torch.int64))
        want = O.topk(f64(torch.floor(row * 4096) - 2048.0), k)
        m = min(k, nv)
        assert np.array_equal(np.sort(want[:m]), got[q, :m]), f"{shape}: query {q}"
        assert np.all(got[q, m:] == -1)


@pytest.mark.parametrize("Q,N", [(160, 30000), (8, 100000)])
@pytest.mark.parametrize("levels", [1, 4])
def test_topk_filter_falls_back_when_the_floor_admits_too_many(cuda_device, Q, N, levels):
    # Scores over 1 or 4 distinct values: the sampled floor admits far more
    # than the 4,096 candidates the filter holds (or the range is empty), so
    # the exact select decides, over the cached keys of one CTA per query
    # (160 queries) or of a cluster of 8 per query (8 queries); ties take the
    # smallest positions.
    k = 512
    u = synth.uniform(6, 14, (Q, N))
    s = torch.floor(u * levels) if levels > 1 else torch.zeros((Q, N))
    n = torch.tensor([N - (q % 4) for q in range(Q)], dtype=torch.int32)
    got = ops.topk(s.to(cuda_device), n.to(cuda_device), k).cpu().numpy()
    for q in (0, 1, Q - 1):
        nv = int(n[q])
        want = O.topk(f64(s[q, :nv]), k)
        assert np.array_equal(np.sort(want[:k]), got[q])


def test_topk_all_equal_scores_take_smallest_indices(cuda_device):
    s = torch.zeros((2, 5000))
    s[1, ::2] = -0.0
    n = torch.tensor([5000, 4000], dtype=torch.int32)
    got = ops.topk(s.to(cuda_device), n.to(cuda_device), 300).cpu().numpy()
    assert np.array_equal(got[0], np.arange(300)) and np.array_equal(got[1], np.arange(300))


@pytest.mark.parametrize("Q,B,N,Hi,Di,k,dtype", [
    (256, 1, 63, 4, 16, 16, torch.float32),    # tiny: causal, many exact-zero ties
    (4, 4, 3000, 64, 128, 512, torch.bfloat16),
    (3, 1, 700, 64, 128, 2048, torch.bfloat16),  # k > n: everything kept, padded
])
def test_index_topk_matches_oracle(cuda_device, Q, B, N, Hi, Di, k, dtype):
    qi, wi, ki = _score_inputs(2, Q, B, N, Hi, Di, dtype)
    qps = Q // B
    if Q == 256:
        n = ops.visible_entries(torch.arange(Q), 8, 4)   # causal prefill positions 0..255
    else:
        n = torch.full((Q,), N, dtype=torch.int32)
    idx = ops.index_topk(qi.to(cuda_device), wi.to(cuda_device), ki.to(cuda_device), n.to(cuda_device), k,
                         q_per_seq=qps).cpu().numpy()
    swaps = 0
    for q in range(Q):
        nv = int(n[q])
        ref_idx, ref_s = O.index_topk(qi[q], wi[q], ki[q // qps], q if Q == 256 else 4 * (N - 1) + 7, k, 8, 4)
        assert O.n_visible(q if Q == 256 else 4 * (N - 1) + 7, 8, 4) == nv
        swaps += check_topk_set(idx[q], ref_idx, ref_s, k, nv)
    assert swaps <= max(2, Q // 8)


@pytest.mark.parametrize("name,nq", [("csa_decode_64k", 32), ("csa_decode_1m", 8), ("csa_prefill_chunk_4k", 24)])
def test_index_topk_full_size(cuda_device, name, nq):
    # Full-size workloads in the benchmark's launch configuration; the
    # oracle checks nq queries (all of them for the decode batches).
    w = WL.WORKLOADS[name]
    qi, wi, ki = (WL.make(w, t, cuda_device) for t in ("qi", "wi", "ki"))
    p = w.positions()
    n = ops.visible_entries(p, w.win, w.stride)
    ws = ops.Workspace(cuda_device)
    idx = ops.index_topk(qi, wi, ki, n.to(cuda_device), w.k, q_per_seq=w.q_per_seq, ws=ws).cpu().numpy()
    assert ws.status() == 0
    del ki
    qs = np.unique(np.linspace(0, w.Q - 1, nq).round().astype(int))
    seqs = sorted({int(q) // w.q_per_seq for q in qs})
    ki_h = {b: WL.rows(w, "ki", torch.arange(b * w.N, (b + 1) * w.N)) for b in seqs}
    qi_h, wi_h = WL.make(w, "qi"), WL.make(w, "wi")
    swaps = 0
    for q in qs:
        b = int(q) // w.q_per_seq
        ref_idx, ref_s = O.index_topk(qi_h[q], wi_h[q], ki_h[b], int(p[q]), w.k, w.win, w.stride)
        swaps += check_topk_set(idx[q], ref_idx, ref_s, w.k, int(n[q]))
    assert swaps <= max(2, len(qs) // 4)


@pytest.mark.parametrize("Q,N", [(32, 16383), (4, 300), (3, 129)])
def test_scores_repeat_exactly_on_one_workspace(cuda_device, Q, N):
    # Three calls on one workspace give bit-identical scores equal to the
    # oracle's, a clean status, and leave the workspace header (status word,
    # wait limit, reserved bytes) at zero for the next call.
    qi = synth.normal(11, 1, (Q, 64, 128), dtype=torch.bfloat16)
    wi = synth.uniform(11, 2, (Q, 64))
    ki = synth.normal(11, 3, (Q, N, 128), dtype=torch.bfloat16)
    n = torch.tensor([N - (q % 3) * 7 for q in range(Q)], dtype=torch.int32)
    d = [t.to(cuda_device) for t in (qi, wi, ki, n)]
    ws = ops.Workspace(cuda_device)
    runs = []
    for _ in range(3):
        out = torch.zeros((Q, N), dtype=torch.float32, device=cuda_device)
        ops.index_scores(*d, out=out, ws=ws)
        torch.cuda.synchronize()
        assert int(ws.buf[:256].count_nonzero()) == 0
        runs.append(out.cpu().numpy())
    assert np.array_equal(runs[0], runs[1]) and np.array_equal(runs[0], runs[2])
    for q in range(Q):
        nv = int(n[q])
        ref = O.index_scores(qi[q], wi[q], ki[q], nv)
        scale = max(np.abs(ref).max(initial=0.0), 1.0)
        assert np.max(np.abs(f64(runs[0][q, :nv]) - ref), initial=0.0) <= 1e-4 * scale
