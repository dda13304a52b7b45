"""Bounded waits end with a status bit, not a hang.

Every wait of a tensor-core kernel on its own pipeline gives up after a limit
(2 s, or the number of nanoseconds in bytes 8..15 of the workspace). Here the
indexer scorer runs with a 1 ns limit: some wait of its pipeline runs out, the
kernel raises CSA_STATUS_WAIT_TIMEOUT, drains the copies and tensor-core work
it has in flight, frees its tensor memory and returns. The context stays
usable: the next call with the default limit is clean and matches the oracle.
No GPU fault is caused: the limit is an ordinary argument of the wait.
"""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import _lib, ops, synth
from helpers import f64

pytestmark = pytest.mark.gpu

CSA_STATUS_WAIT_TIMEOUT = 8


def _inputs(dev, Q=4, N=65536, Hi=64, Di=128):
    # indexer shape of the Flash model (64 heads x 128 dims, bf16): the
    # tensor-core scorer serves it
    qi = synth.normal(3, 4, (Q, Hi, Di), dtype=torch.bfloat16)
    wi = synth.uniform(3, 5, (Q, Hi))
    ki = synth.normal(3, 6, (Q, N, Di), dtype=torch.bfloat16)
    n = torch.tensor([N, N - 5, N // 2 + 3, 1000][:Q], dtype=torch.int32)
    return qi, wi, ki, n, [t.to(dev) for t in (qi, wi, ki, n)]


def _set_limit(ws: ops.Workspace, ns: int):
    buf = ws.get(256)
    buf[8:16].copy_(torch.tensor([ns], dtype=torch.int64).view(torch.uint8).to(buf.device))


def test_scorer_wait_timeout_raises_status_and_returns(cuda_device):
    qi, wi, ki, n, (dqi, dwi, dki, dn) = _inputs(cuda_device)
    ws = ops.Workspace(cuda_device)
    _set_limit(ws, 1)
    ops.index_scores(dqi, dwi, dki, dn, ws=ws)
    torch.cuda.synchronize()  # the call returned: every wait ended
    st = ws.status()
    assert st & CSA_STATUS_WAIT_TIMEOUT, f"status {st:#x}"

    # the same context, a fresh workspace (default limit): clean and correct
    ws2 = ops.Workspace(cuda_device)
    s = ops.index_scores(dqi, dwi, dki, dn, ws=ws2).cpu()
    assert ws2.status() == 0
    rng = np.random.default_rng(0)
    for q in range(qi.shape[0]):
        nv = int(n[q])
        js = np.unique(np.concatenate([rng.integers(0, nv, 300), [0, nv - 1]]))
        ref = O.index_scores(qi[q], wi[q], ki[q][js], len(js))
        got = f64(s[q, js])
        scale = max(np.abs(ref).max(initial=0.0), 1.0)
        assert np.max(np.abs(got - ref)) <= 1e-4 * scale
        assert torch.isnan(s[q, nv:]).all()


def test_limit_is_read_per_call(cuda_device):
    # a workspace whose limit is set back to zero takes the default again
    _, _, _, _, (dqi, dwi, dki, dn) = _inputs(cuda_device, Q=2, N=4096)
    ws = ops.Workspace(cuda_device)
    _set_limit(ws, 1)
    ops.index_scores(dqi, dwi, dki, dn, ws=ws)
    ws.status()  # (read and cleared; the bit may or may not be up on so short a call)
    _set_limit(ws, 0)
    ops.index_scores(dqi, dwi, dki, dn, ws=ws)
    assert ws.status() == 0
    assert _lib.lib().csa_last_cuda_error() == 0
