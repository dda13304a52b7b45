"""A2 / A3 on FP8 E4M3 indexer inputs (reading R18): CUDA vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import ops, synth, workloads as WL
from helpers import check_topk_set, f64

pytestmark = pytest.mark.gpu


def _fp8_inputs(seed, Q, B, N, Hi, Di):
    w = WL.small(WL.WORKLOADS["csa_decode_64k"], seed=seed, Q=Q, B=B, N=N, Hi=Hi, Di=Di)
    return [WL.make(w, t) for t in ("qi8", "sq", "wi", "ki8", "sk")]


@pytest.mark.parametrize("Q,B,N,Hi,Di", [
    (6, 3, 1000, 64, 128),    # tensor-core path, ragged last tile
    (4, 2, 129, 64, 128),     # one full tile + 1 entry
    (5, 5, 300, 8, 32),       # generic kernel
    (256, 1, 63, 4, 16),      # the tiny shape
])
def test_index_scores_fp8_match_oracle(cuda_device, Q, B, N, Hi, Di):
    qi8, sq, wi, ki8, sk = _fp8_inputs(3, Q, B, N, Hi, Di)
    qps = Q // B
    n = torch.tensor([[N, 0, 1, N - 1, N // 2, 17][q % 6] for q in range(Q)], dtype=torch.int32)
    d = lambda t: t.to(cuda_device)
    s = ops.index_scores_fp8(d(qi8), d(sq), d(wi), d(ki8), d(sk), d(n), q_per_seq=qps).cpu()
    for q in range(Q):
        nv = int(n[q])
        b = q // qps
        ref = O.index_scores_fp8(qi8[q].numpy(), sq[q], wi[q], ki8[b].numpy(), sk[b], nv)
        got = f64(s[q, :nv])
        scale = max(np.abs(ref).max(initial=0.0), 1.0)
        # exact code products, fp32 sums over Di and Hi: a few ulp of the largest term
        assert np.max(np.abs(got - ref), initial=0.0) <= 1e-5 * scale, f"query {q}"
        assert torch.isnan(s[q, nv:]).all()


@pytest.mark.parametrize("Q,B,N,k", [(4, 4, 3000, 512), (3, 1, 700, 2048)])
def test_index_topk_fp8_matches_oracle(cuda_device, Q, B, N, k):
    qi8, sq, wi, ki8, sk = _fp8_inputs(4, Q, B, N, 64, 128)
    qps = Q // B
    n = torch.full((Q,), N, dtype=torch.int32)
    d = lambda t: t.to(cuda_device)
    idx = ops.index_topk_fp8(d(qi8), d(sq), d(wi), d(ki8), d(sk), d(n), k, q_per_seq=qps).cpu().numpy()
    swaps = 0
    for q in range(Q):
        b = q // qps
        ref_s = O.index_scores_fp8(qi8[q].numpy(), sq[q], wi[q], ki8[b].numpy(), sk[b], N)
        swaps += check_topk_set(idx[q], O.topk(ref_s, k), ref_s, k, N)
    assert swaps <= 2


def test_index_topk_fp8_full_size(cuda_device):
    # The 64K-context decode batch with FP8 indexer keys, in the benchmark's
    # launch configuration; the oracle checks every query.
    w = WL.WORKLOADS["csa_decode_64k"]
    t = {name: WL.make(w, name, cuda_device) for name in ("qi8", "sq", "wi", "ki8", "sk")}
    p = w.positions()
    n = ops.visible_entries(p, w.win, w.stride)
    idx = ops.index_topk_fp8(t["qi8"], t["sq"], t["wi"], t["ki8"], t["sk"], n.to(cuda_device), w.k,
                             q_per_seq=w.q_per_seq).cpu().numpy()
    del t
    qi8, sq, wi = (WL.make(w, name) for name in ("qi8", "sq", "wi"))
    swaps = 0
    for q in range(w.Q):
        b = q // w.q_per_seq
        rows = torch.arange(b * w.N, (b + 1) * w.N)
        ki8_b, sk_b = WL.rows(w, "ki8", rows).numpy(), WL.rows(w, "sk", rows)
        nv = int(n[q])
        ref_s = O.index_scores_fp8(qi8[q].numpy(), sq[q], wi[q], ki8_b, sk_b, nv)
        swaps += check_topk_set(idx[q], O.topk(ref_s, w.k), ref_s, w.k, nv)
    assert swaps <= w.Q // 4

