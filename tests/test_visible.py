"""Causal visibility (reading R6) and entry counts come from the library
(csa_visible_counts / csa_visible_counts_host / csa_num_entries), checked
against the oracle's own definitions: n_visible(p) and n_entries(T)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_attention_15_b200 import _lib, ops
from compressed_sparse_attention_15_b200.build import build

GEOMS = [(8, 4), (128, 128), (1, 1), (4, 4), (16, 4), (7, 3)]


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def _positions():
    p = list(range(-3, 300)) + [65535, 131072, 135167, 1048575, 2**31 + 5]
    return torch.tensor(p, dtype=torch.int64)


@pytest.mark.parametrize("win,stride", GEOMS)
def test_host_counts_match_oracle(L, win, stride):
    p = _positions()
    n = ops.visible_entries(p, win, stride)
    assert n.dtype == torch.int32 and n.device.type == "cpu"
    ref = [O.n_visible(int(x), win, stride) if x >= 0 else 0 for x in p]
    ref = [min(r, 2**31 - 1) for r in ref]
    assert n.tolist() == ref


@pytest.mark.parametrize("win,stride", GEOMS)
def test_num_entries_matches_oracle(L, win, stride):
    for T in list(range(0, 200)) + [4100, 65536, 1048576]:
        assert ops.num_entries(T, win, stride) == O.n_entries(T, win, stride), (T, win, stride)


def test_workload_counts(L):
    # the entry counts the workloads state (decode: all entries visible)
    assert ops.num_entries(65536, 8, 4) == 16383
    assert ops.num_entries(1048576, 8, 4) == 262143
    assert ops.num_entries(1048576, 128, 128) == 8192
    n = ops.visible_entries(torch.tensor([131072, 135167]), 8, 4)
    assert n.tolist() == [32767, 33791]


def test_rejects_bad_arguments(L):
    P = ctypes.c_void_p(4096)
    assert L.csa_num_entries(100, 0, 4) == -1
    assert L.csa_num_entries(100, 8, 0) == -1
    assert L.csa_num_entries(-1, 8, 4) == -1
    assert L.csa_visible_counts_host(P, -1, 8, 4, P) == 1
    assert L.csa_visible_counts_host(P, 4, 0, 4, P) == 1
    assert L.csa_visible_counts_host(ctypes.c_void_p(0), 4, 8, 4, P) == 1
    assert L.csa_visible_counts_host(ctypes.c_void_p(4100), 4, 8, 4, P) == 1  # int64 array not 8-byte aligned
    assert L.csa_visible_counts(P, 4, 8, 0, P, ctypes.c_void_p(0)) == 1
    assert L.csa_visible_counts(P, 4, 8, 4, ctypes.c_void_p(4098), ctypes.c_void_p(0)) == 1
    assert L.csa_visible_counts_host(ctypes.c_void_p(0), 0, 8, 4, ctypes.c_void_p(0)) == 0  # nothing to do


@pytest.mark.gpu
@pytest.mark.parametrize("win,stride", GEOMS)
def test_device_counts_match_oracle(cuda_device, win, stride):
    p = _positions()
    n = ops.visible_entries(p.to(cuda_device), win, stride)
    assert n.is_cuda and n.dtype == torch.int32
    torch.cuda.synchronize()
    ref = np.array([min(O.n_visible(int(x), win, stride), 2**31 - 1) if x >= 0 else 0 for x in p])
    assert np.array_equal(n.cpu().numpy(), ref)


@pytest.mark.gpu
def test_device_counts_large_batch(cuda_device):
    # many blocks and the grid-stride loop: every causal prefill position of a 300K-token chunk
    p = torch.arange(300_000, dtype=torch.int64)
    n = ops.visible_entries(p.to(cuda_device), 8, 4).cpu()
    ref = ops.visible_entries(p, 8, 4)
    assert torch.equal(n, ref)
    assert int(n[-1]) == O.n_visible(299_999, 8, 4)
