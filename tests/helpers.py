"""Shared test utilities: tolerances, top-k set comparison, seeded index
lists. Nothing here computes a step of the method."""
from __future__ import annotations

import numpy as np
import torch

from compressed_sparse_attention_15_b200 import synth

# Acceptance bars: bf16 inputs with fp32 accumulation, and exact fp32.
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_REL = 1e-5
TIE_REL = 1e-4


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def assert_close(gpu, ref, dtype, what=""):
    """GPU output vs fp64 oracle, with the bar of the input dtype."""
    g, r = f64(gpu), f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - r)
    if dtype == torch.float32:
        rel = err.max() / max(np.abs(r).max(), 1e-30)
        assert rel <= FP32_REL, f"{what}: max rel err {rel:.3e} > {FP32_REL}"
    else:
        assert err.max() <= BF16_MAX_ABS, f"{what}: max abs err {err.max():.3e} > {BF16_MAX_ABS}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e} > {BF16_MEAN_ABS}"
    return err.max()


def check_topk_set(gpu_idx, oracle_idx, oracle_scores, k, n):
    """GPU selection vs oracle selection for one query.

    Exact set equality, except swaps at the selection boundary where the
    oracle scores of the swapped entries differ from the k-th score by at
    most TIE_REL relative. Returns the number of swapped entries."""
    g = np.asarray(gpu_idx)
    o = np.asarray(oracle_idx)
    m = min(k, n)
    gv, ov = g[g >= 0], o[o >= 0]
    assert np.all(g[m:] == -1) and gv.size == m, f"expected {m} selected then -1 padding"
    assert np.all(np.diff(gv) > 0), "selection must be ascending and unique"
    assert gv.min(initial=0) >= 0 and gv.max(initial=0) < max(n, 1)
    gs, os_ = set(gv.tolist()), set(ov.tolist())
    only_g, only_o = gs - os_, os_ - gs
    if not only_g:
        return 0
    s = np.asarray(oracle_scores)
    tau = s[ov[-1]]  # the oracle's k-th best score (best-first order)
    tol = TIE_REL * max(abs(tau), 1e-30)
    for j in only_g:
        assert s[j] >= tau - tol, f"GPU kept j={j} (score {s[j]!r}) well below the boundary {tau!r}"
    for j in only_o:
        assert s[j] <= tau + tol, f"GPU dropped j={j} (score {s[j]!r}) well above the boundary {tau!r}"
    return len(only_g)


def seeded_idx(seed: int, Q: int, N: int, k: int, n_sel=None, n_vis=None) -> torch.Tensor:
    """int32 [Q, k]: for query q, min(k, n_sel[q], n_vis[q]) distinct entries
    of [0, n_vis[q]) drawn from the seeded stream, ascending, then -1."""
    u = synth.uniform_at(seed, 100, torch.arange(Q * N, dtype=torch.int64)).reshape(Q, N)
    j = torch.arange(N).reshape(1, N)
    if n_vis is not None:
        u[j >= torch.as_tensor(n_vis).reshape(Q, 1).long()] = 2.0
    m = min(k, N)
    vals, pick = torch.topk(u, m, dim=1, largest=False)
    pick[vals >= 2.0] = -1
    if n_sel is not None:
        pick[torch.arange(m).reshape(1, m) >= torch.as_tensor(n_sel).reshape(Q, 1).long()] = -1
    pick = torch.where(pick < 0, torch.full_like(pick, 1 << 40), pick).sort(dim=1).values
    pick[pick == (1 << 40)] = -1
    out = torch.full((Q, k), -1, dtype=torch.int32)
    out[:, :m] = pick.to(torch.int32)
    return out
