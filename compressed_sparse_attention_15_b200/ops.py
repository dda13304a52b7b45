"""Torch-facing wrappers of the C ABI (include/csa.h).

These functions only check tensor metadata, allocate outputs / workspaces
with torch (PyTorch is the device-memory allocator and stream provider) and
pass raw pointers, sizes and the current CUDA stream to libcsa.so. They do no
arithmetic of the method. Names follow the C entry points.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

_DT = {torch.float32: _lib.CSA_DTYPE_F32, torch.bfloat16: _lib.CSA_DTYPE_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; use torch.float32 or torch.bfloat16") from None


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, device=None, contiguous=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class Workspace:
    """A reusable device workspace (first 256 bytes: the status word)."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor:
        nbytes = max(256, int(nbytes))
        if self.buf is None or self.buf.numel() < nbytes:
            # zero-filled: the status word, and the counters of csa_decode_step
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf

    def status(self) -> int:
        """Synchronise, return and clear the status word (0 = clean)."""
        if self.buf is None:
            return 0
        return workspace_status(self.buf)


def workspace_status(ws: torch.Tensor) -> int:
    v = ctypes.c_uint32(0)
    rc = _lib.lib().csa_workspace_status(_ptr(ws), _stream(ws.device), ctypes.byref(v))
    if rc not in (_lib.CSA_OK, 5):
        _lib.check("csa_workspace_status", rc)
    return int(v.value)


def visible_entries(p: torch.Tensor, win: int, stride: int) -> torch.Tensor:
    """int32 count of compressed entries visible at each position p
    (csa_visible_counts on a CUDA tensor, one kernel on the current stream;
    csa_visible_counts_host on a CPU tensor). Returns a tensor on p's device."""
    p = torch.as_tensor(p, dtype=torch.int64).contiguous()
    out = torch.empty(p.shape, dtype=torch.int32, device=p.device)
    L = _lib.lib()
    if p.is_cuda:
        rc = L.csa_visible_counts(_ptr(p), p.numel(), int(win), int(stride), _ptr(out), _stream(p.device))
        _lib.check("csa_visible_counts", rc)
    else:
        rc = L.csa_visible_counts_host(_ptr(p), p.numel(), int(win), int(stride), _ptr(out))
        _lib.check("csa_visible_counts_host", rc)
    return out


def num_entries(T: int, win: int, stride: int) -> int:
    """Entries a compressor run over T raw tokens makes (csa_num_entries)."""
    n = _lib.lib().csa_num_entries(int(T), int(win), int(stride))
    if n < 0:
        raise ValueError(f"invalid window geometry win={win} stride={stride} T={T}")
    return int(n)


# ------------------------------------------------------------------ A1

def compress(kv, gate, ape, norm_w, win: int, stride: int, out=None, ratio=None, rope=None):
    """Gated-pooling compressor + RMSNorm (csa_compress); with
    rope = (rope_dims, theta, pos0 int64 [B] or None), RoPE on the entries'
    last rope_dims dims as well (csa_compress_rope).

    kv, gate: [B, T, D] (or [T, D]) with contiguous rows and any sequence
    stride; ape [win, D] fp32; norm_w [D] fp32. Returns / fills out
    [B, N, D] (rows contiguous, any sequence stride), N = (T - win)//stride + 1.
    """
    squeeze = kv.dim() == 2
    if squeeze:
        kv, gate = kv.unsqueeze(0), gate.unsqueeze(0)
    _need(kv, "kv", contiguous=False)
    _need(gate, "gate", dtype=kv.dtype, device=kv.device, contiguous=False)
    _need(ape, "ape", dtype=torch.float32, device=kv.device)
    _need(norm_w, "norm_w", dtype=torch.float32, device=kv.device)
    B, T, D = kv.shape
    for t, nm in ((kv, "kv"), (gate, "gate")):
        if t.shape != (B, T, D) or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{nm} must be [B, T, D] with contiguous [T, D] rows")
    N = num_entries(T, win, stride)
    if out is None:
        out = torch.empty((B, N, D), dtype=kv.dtype, device=kv.device)
    else:
        if out.dim() == 2:
            out = out.unsqueeze(0)
        _need(out, "out", dtype=kv.dtype, device=kv.device, contiguous=False)
        if out.shape != (B, N, D) or out.stride(2) != 1 or out.stride(1) != D:
            raise ValueError("out must be [B, N, D] with contiguous [N, D] rows")
    if rope is None:
        rc = _lib.lib().csa_compress(
            _ptr(kv), _ptr(gate), _ptr(ape), _ptr(norm_w), int(stride if ratio is None else ratio), int(win),
            int(stride), _ptr(out), B, T, D, kv.stride(0), gate.stride(0), out.stride(0), _dtype_code(kv),
            _stream(kv.device))
        _lib.check("csa_compress", rc)
    else:
        rope_dims, theta, pos0 = rope
        if pos0 is not None:
            _need(pos0, "pos0", dtype=torch.int64, device=kv.device)
        rc = _lib.lib().csa_compress_rope(
            _ptr(kv), _ptr(gate), _ptr(ape), _ptr(norm_w), int(stride if ratio is None else ratio), int(win),
            int(stride), _ptr(out), B, T, D, kv.stride(0), gate.stride(0), out.stride(0), int(rope_dims),
            float(theta), _ptr(pos0) if pos0 is not None else None, _dtype_code(kv), _stream(kv.device))
        _lib.check("csa_compress_rope", rc)
    return out[0] if squeeze else out


def index_compress(kv, gate, ape, norm_w, win: int, stride: int, fp8: bool = False):
    """The indexer's own compressor (csa_index_compress): csa_compress's
    entries rotated by the orthonormal Hadamard matrix. Returns [B, N, D] in
    the input dtype, or (E4M3 codes uint8 [B, N, D], scales fp32 [B, N])."""
    squeeze = kv.dim() == 2
    if squeeze:
        kv, gate = kv.unsqueeze(0), gate.unsqueeze(0)
    _need(kv, "kv")
    _need(gate, "gate", dtype=kv.dtype, device=kv.device)
    _need(ape, "ape", dtype=torch.float32, device=kv.device)
    _need(norm_w, "norm_w", dtype=torch.float32, device=kv.device)
    B, T, D = kv.shape
    N = num_entries(T, win, stride)
    out = torch.empty((B, N, D), dtype=torch.uint8 if fp8 else kv.dtype, device=kv.device)
    scales = torch.empty((B, N), dtype=torch.float32, device=kv.device) if fp8 else None
    rc = _lib.lib().csa_index_compress(
        _ptr(kv), _ptr(gate), _ptr(ape), _ptr(norm_w), int(stride), int(win), int(stride), _ptr(out),
        _ptr(scales) if fp8 else None, B, T, D, 0, 0, 0, _dtype_code(kv),
        _lib.CSA_DTYPE_E4M3 if fp8 else _dtype_code(kv), _stream(kv.device))
    _lib.check("csa_index_compress", rc)
    if squeeze:
        return (out[0], scales[0]) if fp8 else out[0]
    return (out, scales) if fp8 else out


def hadamard_rows(x, fp8: bool = False):
    """Orthonormal Hadamard rotation of the last dimension of x (csa_hadamard_rows):
    same shape and dtype, or (E4M3 codes uint8, scales fp32 [x.shape[:-1]])."""
    _need(x, "x")
    D = x.shape[-1]
    rows = x.numel() // D
    out = torch.empty(x.shape, dtype=torch.uint8 if fp8 else x.dtype, device=x.device)
    scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device) if fp8 else None
    rc = _lib.lib().csa_hadamard_rows(_ptr(x), _ptr(out), _ptr(scales) if fp8 else None, rows, D, _dtype_code(x),
                                      _lib.CSA_DTYPE_E4M3 if fp8 else _dtype_code(x), _stream(x.device))
    _lib.check("csa_hadamard_rows", rc)
    return (out, scales) if fp8 else out


# ------------------------------------------------------------- A2 + A3

def _index_common(qi, wi, ki, n_cmp, q_per_seq):
    _need(qi, "qi")
    _need(wi, "wi", dtype=torch.float32, device=qi.device)
    _need(ki, "ki", dtype=qi.dtype, device=qi.device)
    _need(n_cmp, "n_cmp", dtype=torch.int32, device=qi.device)
    Q, Hi, Di = qi.shape
    B, N_max, Di2 = ki.shape
    if Di2 != Di or wi.shape != (Q, Hi) or n_cmp.shape != (Q,):
        raise ValueError("shape mismatch among qi [Q,Hi,Di], wi [Q,Hi], ki [B,N,Di], n_cmp [Q]")
    if q_per_seq is None:
        if Q % B:
            raise ValueError("q_per_seq is required when B does not divide Q")
        q_per_seq = Q // B
    return Q, Hi, Di, B, N_max, q_per_seq


def index_topk(qi, wi, ki, n_cmp, k: int, q_per_seq=None, out=None, ws: Workspace | None = None):
    """Indexer scores + top-k (csa_index_topk). Returns int32 [Q, k]."""
    Q, Hi, Di, B, N_max, qps = _index_common(qi, wi, ki, n_cmp, q_per_seq)
    if out is None:
        out = torch.empty((Q, k), dtype=torch.int32, device=qi.device)
    _need(out, "out", dtype=torch.int32, device=qi.device)
    L = _lib.lib()
    nbytes = L.csa_index_topk_workspace_bytes(Q, N_max, k)
    w = (ws or Workspace(qi.device)).get(nbytes)
    rc = L.csa_index_topk(_ptr(qi), _ptr(wi), _ptr(ki), _ptr(n_cmp), int(k), _ptr(out), Q, B, Hi, Di, N_max, qps,
                          _dtype_code(qi), _ptr(w), w.numel(), _stream(qi.device))
    _lib.check("csa_index_topk", rc)
    return out


def index_scores(qi, wi, ki, n_cmp, q_per_seq=None, out=None, ws: Workspace | None = None):
    """Indexer scores only (csa_index_scores): fp32 [Q, N_max]; entries
    j >= n_cmp[q] are left as they were in ``out`` (NaN when allocated here)."""
    Q, Hi, Di, B, N_max, qps = _index_common(qi, wi, ki, n_cmp, q_per_seq)
    if out is None:
        out = torch.full((Q, N_max), float("nan"), dtype=torch.float32, device=qi.device)
    _need(out, "out", dtype=torch.float32, device=qi.device)
    w = (ws or Workspace(qi.device)).get(256)
    rc = _lib.lib().csa_index_scores(_ptr(qi), _ptr(wi), _ptr(ki), _ptr(n_cmp), _ptr(out), Q, B, Hi, Di, N_max,
                                     qps, _dtype_code(qi), _ptr(w), w.numel(), _stream(qi.device))
    _lib.check("csa_index_scores", rc)
    return out


def topk(scores, n_cmp, k: int, out=None, ws: Workspace | None = None):
    """Top-k of given fp32 scores [Q, N_max] (csa_topk). Returns int32 [Q, k]."""
    _need(scores, "scores", dtype=torch.float32)
    _need(n_cmp, "n_cmp", dtype=torch.int32, device=scores.device)
    Q, N_max = scores.shape
    if out is None:
        out = torch.empty((Q, k), dtype=torch.int32, device=scores.device)
    _need(out, "out", dtype=torch.int32, device=scores.device)
    L = _lib.lib()
    w = (ws or Workspace(scores.device)).get(L.csa_topk_workspace_bytes(Q, N_max, k))
    rc = L.csa_topk(_ptr(scores), _ptr(n_cmp), int(k), _ptr(out), Q, N_max, _ptr(w), w.numel(),
                    _stream(scores.device))
    _lib.check("csa_topk", rc)
    return out


# ------------------------------------------------------- A2 / A3 on FP8 inputs

def _index_fp8_common(qi8, sq, wi, ki8, sk, n_cmp, q_per_seq):
    _need(qi8, "qi8", dtype=torch.uint8)
    dev = qi8.device
    for t, nm in ((sq, "sq"), (wi, "wi"), (sk, "sk")):
        _need(t, nm, dtype=torch.float32, device=dev)
    _need(ki8, "ki8", dtype=torch.uint8, device=dev)
    _need(n_cmp, "n_cmp", dtype=torch.int32, device=dev)
    Q, Hi, Di = qi8.shape
    B, N_max, Di2 = ki8.shape
    if Di2 != Di or wi.shape != (Q, Hi) or sq.shape != (Q, Hi) or sk.shape != (B, N_max) or n_cmp.shape != (Q,):
        raise ValueError("shape mismatch among qi8 [Q,Hi,Di], sq/wi [Q,Hi], ki8 [B,N,Di], sk [B,N], n_cmp [Q]")
    if q_per_seq is None:
        if Q % B:
            raise ValueError("q_per_seq is required when B does not divide Q")
        q_per_seq = Q // B
    return Q, Hi, Di, B, N_max, q_per_seq


def index_scores_fp8(qi8, sq, wi, ki8, sk, n_cmp, q_per_seq=None, out=None, ws: Workspace | None = None):
    """Indexer scores on FP8 E4M3 codes with per-row scales
    (csa_index_scores_fp8): fp32 [Q, N_max], entries past n_cmp untouched."""
    Q, Hi, Di, B, N_max, qps = _index_fp8_common(qi8, sq, wi, ki8, sk, n_cmp, q_per_seq)
    if out is None:
        out = torch.full((Q, N_max), float("nan"), dtype=torch.float32, device=qi8.device)
    _need(out, "out", dtype=torch.float32, device=qi8.device)
    w = (ws or Workspace(qi8.device)).get(256)
    rc = _lib.lib().csa_index_scores_fp8(_ptr(qi8), _ptr(sq), _ptr(wi), _ptr(ki8), _ptr(sk), _ptr(n_cmp), _ptr(out),
                                         Q, B, Hi, Di, N_max, qps, _ptr(w), w.numel(), _stream(qi8.device))
    _lib.check("csa_index_scores_fp8", rc)
    return out


def index_topk_fp8(qi8, sq, wi, ki8, sk, n_cmp, k: int, q_per_seq=None, out=None, ws: Workspace | None = None):
    """FP8 indexer scores + top-k (csa_index_topk_fp8). Returns int32 [Q, k]."""
    Q, Hi, Di, B, N_max, qps = _index_fp8_common(qi8, sq, wi, ki8, sk, n_cmp, q_per_seq)
    if out is None:
        out = torch.empty((Q, k), dtype=torch.int32, device=qi8.device)
    _need(out, "out", dtype=torch.int32, device=qi8.device)
    L = _lib.lib()
    w = (ws or Workspace(qi8.device)).get(L.csa_index_topk_workspace_bytes(Q, N_max, k))
    rc = L.csa_index_topk_fp8(_ptr(qi8), _ptr(sq), _ptr(wi), _ptr(ki8), _ptr(sk), _ptr(n_cmp), int(k), _ptr(out),
                              Q, B, Hi, Di, N_max, qps, _ptr(w), w.numel(), _stream(qi8.device))
    _lib.check("csa_index_topk_fp8", rc)
    return out


# ------------------------------------------------------------- A4 / A5

def _mqa_common(q, kv_cmp, kv_win, win_end, sink, q_per_seq):
    _need(q, "q")
    _need(kv_cmp, "kv_cmp", dtype=q.dtype, device=q.device)
    _need(kv_win, "kv_win", dtype=q.dtype, device=q.device)
    _need(win_end, "win_end", dtype=torch.int32, device=q.device)
    _need(sink, "sink", dtype=torch.float32, device=q.device)
    Q, H, D = q.shape
    B, N_max, D2 = kv_cmp.shape
    B2, T_raw, D3 = kv_win.shape
    if D2 != D or D3 != D or B2 != B or win_end.shape != (Q,) or sink.shape != (H,):
        raise ValueError("shape mismatch among q [Q,H,D], kv_cmp [B,N,D], kv_win [B,T,D], win_end [Q], sink [H]")
    if q_per_seq is None:
        if Q % B:
            raise ValueError("q_per_seq is required when B does not divide Q")
        q_per_seq = Q // B
    return Q, H, D, B, N_max, T_raw, q_per_seq


def sparse_mqa(q, kv_cmp, idx, kv_win, win_end, sink, scale: float, win_len: int, q_per_seq=None, out=None,
               ws: Workspace | None = None):
    """CSA attention over the selected entries + window + sink (csa_sparse_mqa)."""
    Q, H, D, B, N_max, T_raw, qps = _mqa_common(q, kv_cmp, kv_win, win_end, sink, q_per_seq)
    _need(idx, "idx", dtype=torch.int32, device=q.device)
    if idx.dim() != 2 or idx.shape[0] != Q:
        raise ValueError("idx must be [Q, k]")
    k = idx.shape[1]
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", dtype=q.dtype, device=q.device)
    L = _lib.lib()
    w = (ws or Workspace(q.device)).get(L.csa_mqa_workspace_bytes(Q, H, D, k + win_len))
    rc = L.csa_sparse_mqa(_ptr(q), _ptr(kv_cmp), _ptr(idx), _ptr(kv_win), _ptr(sink), float(scale), _ptr(out), Q, B,
                          H, D, N_max, k, int(win_len), _ptr(win_end), T_raw, qps, _dtype_code(q), _ptr(w),
                          w.numel(), _stream(q.device))
    _lib.check("csa_sparse_mqa", rc)
    return out


def topk_sparse_mqa(scores, n_cmp, k: int, q, kv_cmp, kv_win, win_end, sink, scale: float, win_len: int,
                    q_per_seq=None, out=None, idx_out=None, ws: Workspace | None = None):
    """Top-k of the indexer scores, then CSA attention over the selection
    (csa_topk_sparse_mqa: one kernel where the launch plan allows). Returns
    (out [Q, H, D], idx [Q, k] int32)."""
    Q, H, D, B, N_max, T_raw, qps = _mqa_common(q, kv_cmp, kv_win, win_end, sink, q_per_seq)
    _need(scores, "scores", dtype=torch.float32, device=q.device)
    _need(n_cmp, "n_cmp", dtype=torch.int32, device=q.device)
    if scores.shape != (Q, N_max) or n_cmp.shape != (Q,):
        raise ValueError("scores must be [Q, N_max] and n_cmp [Q]")
    if out is None:
        out = torch.empty_like(q)
    if idx_out is None:
        idx_out = torch.empty((Q, k), dtype=torch.int32, device=q.device)
    _need(out, "out", dtype=q.dtype, device=q.device)
    _need(idx_out, "idx_out", dtype=torch.int32, device=q.device)
    L = _lib.lib()
    w = (ws or Workspace(q.device)).get(L.csa_topk_sparse_mqa_workspace_bytes(Q, H, D, N_max, int(k), int(win_len)))
    rc = L.csa_topk_sparse_mqa(_ptr(scores), _ptr(n_cmp), int(k), _ptr(idx_out), _ptr(q), _ptr(kv_cmp), _ptr(kv_win),
                               _ptr(sink), float(scale), _ptr(out), Q, B, H, D, N_max, int(win_len), _ptr(win_end),
                               T_raw, qps, _dtype_code(q), _ptr(w), w.numel(), _stream(q.device))
    _lib.check("csa_topk_sparse_mqa", rc)
    return out, idx_out


def hca_mqa(q, kv_cmp, n_cmp, kv_win, win_end, sink, scale: float, win_len: int, q_per_seq=None, out=None,
            ws: Workspace | None = None):
    """HCA attention over every visible entry + window + sink (hca_mqa)."""
    Q, H, D, B, N_max, T_raw, qps = _mqa_common(q, kv_cmp, kv_win, win_end, sink, q_per_seq)
    _need(n_cmp, "n_cmp", dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", dtype=q.dtype, device=q.device)
    L = _lib.lib()
    w = (ws or Workspace(q.device)).get(L.csa_mqa_workspace_bytes(Q, H, D, N_max + win_len))
    rc = L.hca_mqa(_ptr(q), _ptr(kv_cmp), _ptr(kv_win), _ptr(sink), float(scale), _ptr(out), Q, B, H, D, N_max,
                   _ptr(n_cmp), int(win_len), _ptr(win_end), T_raw, qps, _dtype_code(q), _ptr(w), w.numel(),
                   _stream(q.device))
    _lib.check("hca_mqa", rc)
    return out


# ------------------------------------------------------- the whole decode step

def decode_step(q, kv_cmp, kv_win, win_end, sink, scale: float, win_len: int, n_cmp, *, qi=None, wi=None, ki=None,
                k: int | None = None, qi8=None, sq=None, ki8=None, sk=None, append=None, out=None, idx_out=None,
                q_per_seq=None, ws: Workspace | None = None, persistent: bool = False):
    """One decode step in one call (csa_decode_step): the cache append, then
    for CSA (qi or qi8 given) the indexer top-k and the sparse attention, for
    HCA the dense attention over the n_cmp visible entries. persistent=True
    asks for the one-persistent-kernel variant (CSA_STEP_PERSISTENT), else the
    chained kernels (CSA_STEP_CHAINED).

    append = None or a dict with kv, gate ([B, T, D], rows contiguous, any
    sequence stride), ape, norm_w, win, stride, row0 (first cache row written)
    and optionally rope = (rope_dims, theta, pos0 int64 [B] or None).
    Returns out [Q, H, D] (and fills idx_out [Q, k] for CSA)."""
    Q, H, D, B, N_max, T_raw, qps = _mqa_common(q, kv_cmp, kv_win, win_end, sink, q_per_seq)
    _need(n_cmp, "n_cmp", dtype=torch.int32, device=q.device)
    if n_cmp.shape != (Q,):
        raise ValueError("n_cmp must be [Q]")
    a = _lib.DecodeStepArgs()
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", dtype=q.dtype, device=q.device)
    a.q, a.kv_cmp, a.kv_win, a.win_end, a.sink, a.out, a.n_cmp = (
        _ptr(q), _ptr(kv_cmp), _ptr(kv_win), _ptr(win_end), _ptr(sink), _ptr(out), _ptr(n_cmp))
    a.scale = float(scale)
    a.Q, a.B, a.H, a.D, a.N_max, a.win_len, a.T_raw, a.q_per_seq = Q, B, H, D, N_max, int(win_len), T_raw, qps
    a.dtype = _dtype_code(q)
    a.variant = _lib.CSA_STEP_PERSISTENT if persistent else _lib.CSA_STEP_CHAINED
    fp8 = qi8 is not None
    if qi is not None or fp8:
        if k is None:
            raise ValueError("k is required for a CSA step")
        if fp8:
            _index_fp8_common(qi8, sq, wi, ki8, sk, n_cmp, qps)
            a.qi, a.sq, a.wi, a.ki, a.sk = _ptr(qi8), _ptr(sq), _ptr(wi), _ptr(ki8), _ptr(sk)
            a.index_dtype = _lib.CSA_DTYPE_E4M3
            a.Hi, a.Di = qi8.shape[1], qi8.shape[2]
        else:
            _index_common(qi, wi, ki, n_cmp, qps)
            a.qi, a.wi, a.ki = _ptr(qi), _ptr(wi), _ptr(ki)
            a.index_dtype = _dtype_code(qi)
            a.Hi, a.Di = qi.shape[1], qi.shape[2]
        if idx_out is None:
            idx_out = torch.empty((Q, int(k)), dtype=torch.int32, device=q.device)
        _need(idx_out, "idx_out", dtype=torch.int32, device=q.device)
        if idx_out.shape != (Q, int(k)):
            raise ValueError("idx_out must be [Q, k]")
        a.idx_out = _ptr(idx_out)
        a.k = int(k)
    if append is not None:
        kv, gate = append["kv"], append["gate"]
        _need(kv, "append kv", dtype=q.dtype, device=q.device, contiguous=False)
        _need(gate, "append gate", dtype=q.dtype, device=q.device, contiguous=False)
        _need(append["ape"], "ape", dtype=torch.float32, device=q.device)
        _need(append["norm_w"], "norm_w", dtype=torch.float32, device=q.device)
        if kv.dim() != 3 or kv.shape[0] != B or kv.shape[2] != D or kv.stride(2) != 1 or kv.stride(1) != D:
            raise ValueError("append kv must be [B, T, D] with contiguous [T, D] rows")
        if gate.shape != kv.shape or gate.stride(2) != 1 or gate.stride(1) != D:
            raise ValueError("append gate must match append kv")
        a.app_kv, a.app_gate, a.ape, a.norm_w = _ptr(kv), _ptr(gate), _ptr(append["ape"]), _ptr(append["norm_w"])
        a.app_win, a.app_stride, a.app_T = int(append["win"]), int(append["stride"]), kv.shape[1]
        a.app_kv_seq_stride, a.app_gate_seq_stride = kv.stride(0), gate.stride(0)
        a.app_row0 = int(append["row0"])
        rope = append.get("rope")
        if rope is not None:
            rope_dims, theta, pos0 = rope
            if pos0 is not None:
                _need(pos0, "pos0", dtype=torch.int64, device=q.device)
                a.pos0 = _ptr(pos0)
            a.rope_dims, a.rope_theta = int(rope_dims), float(theta)
    L = _lib.lib()
    w = (ws or Workspace(q.device)).get(L.csa_decode_step_workspace_bytes(ctypes.byref(a)))
    rc = L.csa_decode_step(ctypes.byref(a), _ptr(w), w.numel(), _stream(q.device))
    _lib.check("csa_decode_step", rc)
    return out
