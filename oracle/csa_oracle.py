"""fp64 CPU oracle for the hybrid compressed-sparse attention (CSA/HCA) path.

TEST INFRASTRUCTURE ONLY. This module is the independent, slow, obviously
correct statement of what the path computes. Only the test suite, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import
or run it. It shares no code with the CUDA library or its Python binding and
imports neither; the two sides meet only in the seeded input generator.

Every function takes plain arrays, converts them exactly to float64, and does
all arithmetic in float64 with numpy. There is no blocking, fusion or
reordering beyond what each definition states.

Sources (the pages describe the method only in prose):

* "DeepSeek-V4 Architecture Analysis" (architecture_analysis.py),
  INNOVATIONS section 1, "COMPRESSED SPARSE ATTENTION (CSA)": sliding window of
  the nearest 128 tokens; learned gated pooling 4 tokens -> 1 with overlapping
  windows, using absolute position embeddings within the window and an RMSNorm
  on the compressed output; HCA 128 tokens -> 1; an indexer that scores
  compressed positions by dot products with per-head importance weights and
  keeps the top-k; a learnable per-head scalar attention sink.
* same page, INNOVATIONS section 2, "UNIFIED HEAD DIMENSION": keys and values
  share one head_dim = 512 representation (K = V); the RoPE dimensions are
  rotated separately (pre-applied to the inputs here).
* "DeepSeek-V4-Flash" (llm-atlas model card), table "Champs bruts du
  config.json": head_dim 512, index_n_heads 64, index_head_dim 128,
  index_topk 512, sliding_window 128, rms_norm_eps 1e-6,
  num_attention_heads 64, num_key_value_heads 1.

Readings taken where the pages are silent (each is listed with its reason in
the design notes):

* R1 CSA windows are 8 tokens long with stride 4: entry j covers tokens
  [4j, 4j + 7]; a trailing partial window makes no entry. HCA uses window =
  stride = 128.
* R2 the pool is a per-dimension softmax over the window positions of
  (gate + ape[i]), ape indexed by position i inside the window.
* R4 RMSNorm: y = c / sqrt(mean(c^2) + eps) * norm_w, eps = 1e-6.
* R6 entry j is visible at position p iff its last token j*stride + win - 1
  is <= p.
* R8 the window is tokens max(0, p - W + 1) .. p, not de-duplicated against
  compressed entries.
* R9 indexer score s_j = sum_h w_h * max(0, qi_h . ki_j), unscaled.
* R10 top-k orders by (score descending, index ascending); fewer than k
  visible entries are all kept and the rest padded with -1.
* R11 the sink is a per-head logit (not multiplied by the softmax scale) in
  the denominator, carrying a zero value vector.
* R12 K = V: one row serves as key and value.
* R18 FP8 indexer (the next row after the bf16 path): indexer keys and
  queries are OCP FP8 E4M3 codes ("fmt": "e4m3", "quant_method": "fp8" in the
  quantization_config of "deepseek-ai/DeepSeek-V4-Flash-0731", table "Config
  changes"; the indexer is trained with quantization-aware training,
  Architecture analysis INNOVATIONS section 1) with one positive fp32 scale
  per row: per compressed entry for the keys, per (query, head) for the
  queries; value = scale * decoded code. The score is R9 on those values.
* R19 the indexer's own compressor (the next row f2; Architecture analysis
  INNOVATIONS section 1: "its own dedicated KV compressor with Hadamard
  rotation"): the A1 pool + RMSNorm at the indexer head dim, followed by the
  orthonormal Sylvester-Hadamard rotation x -> x H_n / sqrt(n) of each row; the
  queries take the same rotation, so scores are unchanged in exact
  arithmetic. Rows become FP8 codes with one scale per row, amax / 448
  (dynamic scaling; a zero row gets scale 1), each value rounded to the
  nearest E4M3 value, ties to even, magnitudes above 448 saturating to 448.
* R20 RoPE on the compressed entries (the next row f3; Architecture analysis,
  INNOVATIONS section 1: "RoPE on rope dimensions of compressed KV", section
  2: the last 64 of the 512 dims are the rope dims; ARCHITECTURE_SPEC:
  compress_rope_theta 160000): after the pool + RMSNorm, the last 64 dims of
  entry j are rotated in adjacent pairs (d, d + 1) by the angle
  p_j * theta^(-2i / 64) for pair i, with p_j = pos0 + j * stride + win - 1,
  the absolute position of the entry's last token (pos0: the position of the
  sequence's raw token 0). Plain RoPE, no frequency scaling.

Pins (tests/test_oracle_pins.py) tie every function to something other than
itself: closed forms, textbook/library special cases (torch rms_norm,
avg_pool1d, scaled_dot_product_attention), invariants and brute force.
"""
from __future__ import annotations

import numpy as np

RMS_EPS = 1e-6


def as_f64(x) -> np.ndarray:
    """Exact conversion to float64 (bf16 and fp32 values are representable)."""
    try:  # torch tensors (bf16 has no numpy dtype): widen in torch first
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# A1: gated-pooling compressor + RMSNorm
# ---------------------------------------------------------------------------

def n_entries(T: int, win: int, stride: int) -> int:
    """Number of complete windows of length ``win`` at stride ``stride`` that
    fit in T tokens (reading R1: a trailing partial window makes no entry)."""
    if T < win:
        return 0
    return (T - win) // stride + 1


def rms_norm(c: np.ndarray, norm_w: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """RMSNorm over the last axis (model card: rms_norm_eps = 1e-6; the
    architecture analysis, INNOVATIONS section 1: "RMSNorm on compressed
    output")."""
    c = as_f64(c)
    rms = np.sqrt(np.mean(c * c, axis=-1, keepdims=True) + eps)
    return c / rms * as_f64(norm_w)


def compress(kv, gate, ape, norm_w, win: int, stride: int, eps: float = RMS_EPS,
             pre_norm: bool = False) -> np.ndarray:
    """Compress one sequence of raw per-token KV into one entry per window.

    kv, gate: [T, D] (the wkv / wgate projections, RoPE already applied);
    ape: [win, D] absolute position embedding indexed by the position inside
    the window; norm_w: [D]. Returns [n_entries(T), D] in float64.

    Follows the architecture analysis, INNOVATIONS section 1: learned gated
    pooling over (overlapping, for CSA) windows, position embeddings within
    the window, RMSNorm on the compressed output. For entry j over tokens
    t = j*stride + i, i = 0..win-1, and every dimension d:
        a[i, d] = softmax over i of (gate[t, d] + ape[i, d])
        c[d]    = sum_i a[i, d] * kv[t, d]
        out     = RMSNorm(c) * norm_w
    With ``pre_norm`` the pooled c is returned without the norm.
    """
    kv = as_f64(kv)
    gate = as_f64(gate)
    ape = as_f64(ape)
    T, D = kv.shape
    assert gate.shape == (T, D) and ape.shape == (win, D)
    N = n_entries(T, win, stride)
    out = np.empty((N, D), dtype=np.float64)
    block = max(1, (1 << 22) // max(1, win * D))  # bounds the temporaries
    for j0 in range(0, N, block):
        j1 = min(N, j0 + block)
        tok = (np.arange(j0, j1)[:, None] * stride + np.arange(win)[None, :])  # [n, win]
        logits = gate[tok] + ape[None, :, :]                # [n, win, D]
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        a = e / e.sum(axis=1, keepdims=True)                # softmax over the window axis
        out[j0:j1] = (a * kv[tok]).sum(axis=1)
    if pre_norm:
        return out
    return rms_norm(out, norm_w, eps)


# ---------------------------------------------------------------------------
# Causal visibility of compressed entries
# ---------------------------------------------------------------------------

def rope_last_dims(x, positions, theta: float, rope_dims: int = 64) -> np.ndarray:
    """Rotate the last `rope_dims` dims of each row of x in adjacent pairs
    (reading R20): pair i = (d, d + 1), d = D - rope_dims + 2 i, by the angle
    positions[row] * theta^(-2 i / rope_dims)."""
    y = as_f64(x).copy()
    pos = np.asarray(positions, dtype=np.float64)
    D = y.shape[-1]
    i = np.arange(rope_dims // 2, dtype=np.float64)
    ang = pos[:, None] * theta ** (-2.0 * i / rope_dims)[None, :]        # [rows, pairs]
    c, s_ = np.cos(ang), np.sin(ang)
    a = y[:, D - rope_dims::2].copy()
    b = y[:, D - rope_dims + 1::2].copy()
    y[:, D - rope_dims::2] = a * c - b * s_
    y[:, D - rope_dims + 1::2] = a * s_ + b * c
    return y


def compress_rope(kv, gate, ape, norm_w, win: int, stride: int, pos0: int, theta: float, rope_dims: int = 64,
                  eps: float = RMS_EPS) -> np.ndarray:
    """A1 followed by RoPE on the entries' last dims (reading R20): entry j at
    the position of its last token, pos0 + j * stride + win - 1."""
    c = compress(kv, gate, ape, norm_w, win, stride, eps)
    p = pos0 + np.arange(c.shape[0]) * stride + win - 1
    return rope_last_dims(c, p, theta, rope_dims)


def n_visible(p: int, win: int, stride: int) -> int:
    """Entries whose every token is at or before position p (reading R6):
    entry j is visible iff j*stride + win - 1 <= p, i.e. the number of complete
    windows in the prefix of p + 1 tokens."""
    return n_entries(p + 1, win, stride)


# ---------------------------------------------------------------------------
# A2 + A3: indexer scores and top-k selection
# ---------------------------------------------------------------------------

def index_scores(qi, wi, ki, n_vis: int) -> np.ndarray:
    """Indexer score of every visible compressed entry for one query.

    qi: [Hi, Di] indexer query heads; wi: [Hi] per-head importance weights;
    ki: [>= n_vis, Di] indexer keys of the query's sequence.
    Architecture analysis, INNOVATIONS section 1 (indexer: "dot-product
    attention + per-head importance weights"); reading R9:
        s_j = sum_h wi[h] * max(0, qi[h] . ki[j]),  j < n_vis.
    """
    qi = as_f64(qi)
    wi = as_f64(wi)
    ki = as_f64(ki)[:n_vis]
    dots = ki @ qi.T                     # [n_vis, Hi]
    return np.maximum(dots, 0.0) @ wi    # [n_vis]


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of OCP FP8 E4M3 codes (uint8), written from the format's
    definition: bit 7 sign, bits 6-3 exponent (bias 7), bits 2-0 mantissa;
    exponent 0 is subnormal, m/8 * 2^-6; otherwise (1 + m/8) * 2^(e - 7);
    S.1111.111 is NaN and there are no infinities (the "fn" variant, largest
    finite value 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    return np.where((c & 0x7F) == 0x7F, np.nan, sign * mag)


def e4m3_encode(x) -> np.ndarray:
    """Nearest OCP FP8 E4M3 code of each value (ties to the even code),
    magnitudes above 448 saturating to 448, the sign kept (a negative value
    that rounds to zero gives -0, 0x80); written from the format's value set:
    the 127 non-negative finite codes 0x00..0x7E in increasing order."""
    x = np.asarray(x, dtype=np.float64)
    pos = e4m3_decode(np.arange(0x7F, dtype=np.uint8))          # 0 .. 448, increasing
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(pos, a, side="left"), 0, 0x7E)   # first value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - pos[lo], pos[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))   # ties: even code (even mantissa)
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a == pos[hi], hi, code).astype(np.uint8)      # exact values
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)  # the sign is kept, zero included


def quantize_rows_e4m3(x):
    """Per-row dynamic FP8 quantization (reading R19), in fp32 like the GPU
    (the codes are integers decided by fp32 arithmetic on both sides):
        scale = fp32(amax_row / 448) (1 for an all-zero row),
        code  = e4m3_encode(fp32(x_f32 / scale)).
    x: [rows, n]. Returns (codes uint8 [rows, n], scales float32 [rows])."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    amax = np.abs(x32).max(axis=1)
    scale = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0)).astype(np.float32)
    y = (x32 / scale[:, None]).astype(np.float32)
    return e4m3_encode(y), scale


def hadamard_matrix(n: int) -> np.ndarray:
    """Sylvester's Hadamard matrix: H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]]."""
    assert n >= 1 and n & (n - 1) == 0
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_rotate(x) -> np.ndarray:
    """Orthonormal Hadamard rotation of each row (reading R19): x H_n / sqrt(n)."""
    x = as_f64(x)
    n = x.shape[-1]
    return x @ hadamard_matrix(n) / np.sqrt(n)


def index_compress(kv, gate, ape, norm_w, win: int, stride: int, eps: float = RMS_EPS) -> np.ndarray:
    """The indexer's keys from its own raw KV (reading R19): the A1 pool +
    RMSNorm at the indexer head dim, then the Hadamard rotation of each entry."""
    return hadamard_rotate(compress(kv, gate, ape, norm_w, win, stride, eps))


def index_scores_fp8(qi8, sq, wi, ki8, sk, n_vis: int) -> np.ndarray:
    """Indexer scores on FP8 inputs (reading R18), for one query:
        qi[h] = sq[h] * e4m3(qi8[h]),  ki[j] = sk[j] * e4m3(ki8[j]),
        s_j = sum_h wi[h] * max(0, qi[h] . ki[j]),  j < n_vis.
    qi8: [Hi, Di] uint8 codes, sq: [Hi]; ki8: [>= n_vis, Di] uint8 codes,
    sk: [>= n_vis]; wi: [Hi]."""
    qi = e4m3_decode(qi8) * as_f64(sq)[:, None]
    ki = e4m3_decode(np.asarray(ki8)[:n_vis]) * as_f64(sk)[:n_vis, None]
    return index_scores(qi, wi, ki, n_vis)


def index_topk_fp8(qi8, sq, wi, ki8, sk, p: int, k: int, win: int, stride: int):
    """FP8 scores and the selected index list for one query at position p."""
    nv = n_visible(p, win, stride)
    s = index_scores_fp8(qi8, sq, wi, ki8, sk, nv)
    return topk(s, k), s


def topk(scores, k: int) -> np.ndarray:
    """Indices of the min(k, n) best scores, best first, padded with -1 to k.

    Order (reading R10): score descending, ties by index ascending. A full
    stable sort is the definition (model card: index_topk = 512).
    """
    s = as_f64(scores)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))   # last key is primary
    out = np.full(k, -1, dtype=np.int64)
    m = min(k, n)
    out[:m] = order[:m]
    return out


def index_topk(qi, wi, ki, p: int, k: int, win: int, stride: int):
    """Scores and the selected index list for one query at position p."""
    nv = n_visible(p, win, stride)
    s = index_scores(qi, wi, ki, nv)
    return topk(s, k), s


# ---------------------------------------------------------------------------
# A4 / A5: MQA over selected rows + sliding window + sink
# ---------------------------------------------------------------------------

def attend(q, rows, sink, scale: float):
    """Softmax attention of H query heads over R shared rows plus a sink.

    q: [H, D]; rows: [R, D] used as both key and value (architecture analysis,
    INNOVATIONS section 2: keys and values share one representation);
    sink: [H] per-head logit with a zero value (INNOVATIONS section 1,
    "Attention sink"; reading R11); scale multiplies q . row only.
    For head h: logits_r = scale * q_h . row_r, plus sink_h;
        p_r = exp(logit_r - m) / Z,  p_sink = exp(sink_h - m) / Z,
        out_h = sum_r p_r * row_r.
    Returns (out [H, D], p [H, R], p_sink [H]).
    """
    q = as_f64(q)
    rows = as_f64(rows)
    sink = as_f64(sink)
    H = q.shape[0]
    R = rows.shape[0]
    logits = scale * (q @ rows.T) if R else np.zeros((H, 0))
    m = np.maximum(logits.max(axis=1) if R else -np.inf, sink)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(logits - m[:, None])
    e_sink = np.exp(sink - m)
    Z = e.sum(axis=1) + e_sink
    p = e / Z[:, None]
    out = p @ rows if R else np.zeros_like(q)
    return out, p, e_sink / Z


def window_rows(kv_win, win_end: int, W: int) -> np.ndarray:
    """Raw rows max(0, e - W + 1) .. e of one sequence's raw-KV buffer, where e
    is the buffer row of the query's own token (architecture analysis,
    INNOVATIONS section 1: each token attends to its nearest 128 tokens;
    reading R8: the query's own token is included)."""
    kv_win = as_f64(kv_win)
    lo = max(0, win_end - W + 1)
    return kv_win[lo:win_end + 1]


def sparse_mqa(q, kv_cmp, idx, kv_win, win_end: int, W: int, sink, scale: float):
    """CSA attention for one query: the selected compressed rows (entries
    idx >= 0 of this sequence's compressed cache), the sliding window and
    the sink. Returns out [H, D] (float64)."""
    kv_cmp = as_f64(kv_cmp)
    idx = np.asarray(idx)
    sel = kv_cmp[idx[idx >= 0]]
    rows = np.concatenate([sel, window_rows(kv_win, win_end, W)], axis=0)
    return attend(q, rows, sink, scale)[0]


def hca_mqa(q, kv_cmp, n_cmp: int, kv_win, win_end: int, W: int, sink, scale: float):
    """HCA attention for one query: every visible compressed entry
    (architecture analysis, INNOVATIONS section 1: HCA, 128 tokens -> 1, for
    global context, with no indexer), the sliding window and the sink."""
    kv_cmp = as_f64(kv_cmp)[:n_cmp]
    rows = np.concatenate([kv_cmp, window_rows(kv_win, win_end, W)], axis=0)
    return attend(q, rows, sink, scale)[0]


# ---------------------------------------------------------------------------
# Storage rounding (the compressed cache is stored in the input dtype)
# ---------------------------------------------------------------------------

def round_to(x, dtype: str) -> np.ndarray:
    """Round float64 values once to 'fp32' or 'bf16' (round to nearest even)
    and return them as float64. bf16 is a single rounding from fp64 to 8
    significant bits (normal range only)."""
    x = as_f64(x)
    if dtype == "fp64":
        return x.copy()
    if dtype == "fp32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        # Round fp64 -> bf16 directly: keep 8 significant bits, ties to even.
        m, e = np.frexp(x)                  # x = m * 2**e, 0.5 <= |m| < 1
        scaled = np.ldexp(m, 8)             # 8 significant bits in the integer part
        r = np.round(scaled)                # numpy rounds half to even
        return np.ldexp(r, e - 8)
    raise ValueError(dtype)
