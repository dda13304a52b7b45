"""The C ABI: the library loads, exports every function include/csa.h
declares, and rejects bad arguments on the host before any launch (these
calls return before touching the GPU, so they run without one)."""
import ctypes
import os
import re

import pytest

from compressed_sparse_attention_15_b200 import _lib
from compressed_sparse_attention_15_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa_\w+|hca_\w+)\s*\(", src)))


def test_header_declares_the_four_calls():
    names = _declared()
    for n in ("csa_compress", "csa_index_topk", "csa_sparse_mqa", "hca_mqa"):
        assert n in names


def test_every_declared_symbol_is_exported_and_bound(L):
    names = _declared()
    assert names
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, f"{n} has no ctypes signature"


def test_strerror(L):
    for c in range(7):
        assert _lib.strerror(c).startswith("CSA_")
    assert "unknown" in _lib.strerror(99)


NULL = ctypes.c_void_p(0)
P = ctypes.c_void_p(4096)  # a non-null, aligned placeholder; never dereferenced


def test_compress_rejects_bad_arguments(L):
    def call(kv=P, ratio=4, win=8, stride=4, T=64, D=16, B=1, dtype=1):
        return L.csa_compress(kv, P, P, P, ratio, win, stride, P, B, T, D, 0, 0, 0, dtype, NULL)
    assert call(kv=NULL) == 1
    assert call(ratio=8) == 1          # ratio must equal stride
    assert call(T=7) == 1              # fewer tokens than one window
    assert call(win=129, stride=129, ratio=129, T=300) == 1
    assert call(dtype=7) == 1
    assert call(B=0) == 1
    assert call(kv=ctypes.c_void_p(4097)) == 1   # misaligned bf16


def test_index_topk_rejects_bad_arguments(L):
    ws_ok = L.csa_index_topk_workspace_bytes(4, 100, 16)
    assert ws_ok >= 256 + 4 * 100 * 4

    def call(k=16, Hi=4, Di=16, q_per_seq=4, B=1, ws=P, ws_bytes=ws_ok):
        return L.csa_index_topk(P, P, P, P, k, P, 4, B, Hi, Di, 100, q_per_seq, 1, ws, ws_bytes, NULL)
    assert call(k=0) == 1
    assert call(k=4097) == 1
    assert call(Hi=129) == 1
    assert call(q_per_seq=1) == 1      # 1 sequence x 1 query < 4 queries
    assert call(ws_bytes=ws_ok - 1) == 3
    assert call(ws=ctypes.c_void_p(4096 + 128)) == 3  # not 256-byte aligned


def test_index_fp8_rejects_bad_arguments(L):
    ws_ok = L.csa_index_topk_workspace_bytes(4, 100, 16)

    def topk(k=16, Hi=4, Di=16, q_per_seq=4, sq=P, sk=P, ws_bytes=ws_ok):
        return L.csa_index_topk_fp8(P, sq, P, P, sk, P, k, P, 4, 1, Hi, Di, 100, q_per_seq, P, ws_bytes, NULL)
    assert topk(k=0) == 1
    assert topk(Hi=129) == 1
    assert topk(Di=257) == 1
    assert topk(q_per_seq=1) == 1
    assert topk(sq=NULL) == 1 and topk(sk=NULL) == 1          # the scales are required
    assert topk(sk=ctypes.c_void_p(4096 + 2)) == 1           # misaligned float array
    assert topk(ws_bytes=ws_ok - 1) == 3

    def scores(scores_ptr=P, ws_bytes=256):
        return L.csa_index_scores_fp8(P, P, P, P, P, P, scores_ptr, 4, 1, 4, 16, 100, 4, P, ws_bytes, NULL)
    assert scores(scores_ptr=NULL) == 1
    assert scores(ws_bytes=255) == 3


def test_mqa_rejects_bad_arguments(L):
    ws = L.csa_mqa_workspace_bytes(2, 4, 16, 32)
    assert ws >= 256

    def sparse(idx=P, k=16, W=16, H=4, D=16, ws_bytes=ws):
        return L.csa_sparse_mqa(P, P, idx, P, P, 0.25, P, 2, 1, H, D, 63, k, W, P, 256, 2, 0, P, ws_bytes, NULL)
    assert sparse(idx=NULL) == 1
    assert sparse(W=0) == 1
    assert sparse(H=129) == 1
    assert sparse(D=1025) == 1
    assert sparse(ws_bytes=255) == 3
    assert L.hca_mqa(P, P, P, P, 0.25, P, 2, 1, 4, 16, 63, NULL, 16, P, 256, 2, 0, P, ws, NULL) == 1


def test_topk_rejects_bad_arguments(L):
    assert L.csa_topk(P, P, 0, P, 2, 10, P, 256, NULL) == 1
    assert L.csa_topk(NULL, P, 4, P, 2, 10, P, 256, NULL) == 1
    assert L.csa_topk(P, P, 4, P, 2, 10, P, 0, NULL) == 3


def test_topk_sparse_mqa_rejects_bad_arguments(L):
    # scores [2, 63], k 16, window 16, 4 heads x 16 dims, one sequence of 2 queries
    ws = L.csa_topk_sparse_mqa_workspace_bytes(2, 4, 16, 63, 16, 16)
    assert ws >= L.csa_topk_workspace_bytes(2, 63, 16)
    assert ws >= L.csa_mqa_workspace_bytes(2, 4, 16, 16 + 16)

    def call(scores=P, n=P, k=16, idx_out=P, W=16, H=4, ws_bytes=ws, ws_ptr=P):
        return L.csa_topk_sparse_mqa(scores, n, k, idx_out, P, P, P, P, 0.25, P, 2, 1, H, 16, 63, W, P, 256, 2, 0,
                                     ws_ptr, ws_bytes, NULL)
    assert call(scores=NULL) == 1
    assert call(n=NULL) == 1
    assert call(idx_out=NULL) == 1
    assert call(k=0) == 1
    assert call(k=4097) == 1
    assert call(idx_out=ctypes.c_void_p(4096 + 2)) == 1  # misaligned int32 array
    assert call(W=0) == 1
    assert call(H=129) == 1
    assert call(ws_bytes=ws - 1) == 3
    assert call(ws_ptr=ctypes.c_void_p(4096 + 128)) == 3  # not 256-byte aligned
