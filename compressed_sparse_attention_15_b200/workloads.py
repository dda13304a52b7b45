"""The synthetic workloads of the CSA/HCA path: shapes, positions, buffer
layout and the seeded recipe of every input tensor.

Pure data: nothing here computes any step of the method. Every tensor is
drawn by ``synth`` from (seed, tensor id, element index), so the host can
regenerate any slice the fp64 oracle needs.

Recipe (tensor id: distribution):
  1 q      [Q, H, D]      N(0,1)      query heads (RoPE already applied)
  2 kv_cmp [B, N, D]      N(0,1)      compressed KV cache
  3 kv_win [B, T_raw, D]  N(0,1)      raw-KV buffer holding the window tokens
  4 qi     [Q, Hi, Di]    N(0,1)      indexer query heads
  5 wi     [Q, Hi]        U(0,1)      indexer per-head weights (fp32)
  6 ki     [B, N, Di]     N(0,1)      indexer key cache
  7 sink   [H]            N(0,1)      per-head sink logit (fp32)
  8 kv_raw [1, bulk_T, D] N(0,1)     raw KV of a whole sequence (1 M-token bulk compression)
  9 gate   [B, T_c, D]    N(0,1)      gate logits of the tokens compressed in a step
 10 ape    [win, D]       N(0,0.1)    in-window position embedding (fp32)
 12 gate_raw [1, bulk_T, D] N(0,1)    gate logits of the bulk-compressed sequence
 13 qi8    [Q, Hi, Di]    E4M3 codes of 64 * N(0,1)   FP8 indexer queries (|64 x| <= 384 < 448)
 14 sq     [Q, Hi]        U(0,1)/64 + 1/256            their per-row scales (fp32)
 15 ki8    [B, N, Di]     E4M3 codes of 64 * N(0,1)   FP8 indexer keys
 16 sk     [B, N]         U(0,1)/64 + 1/256            their per-row scales (fp32)
 17 ikv_raw   [1, bulk_T, Di] N(0,1)   raw indexer KV of the bulk-compressed sequence
 18 igate_raw [1, bulk_T, Di] N(0,1)   its gate logits
 19 iape   [win, Di]      N(0,0.1)    the indexer compressor's position embedding (fp32)
    norm_w [D]            1.0         RMSNorm weight (fp32)
bf16 tensors are drawn in fp32 and rounded once to bf16 (RNE); FP8 codes are
fp32 draws rounded once to E4M3 (RNE, torch's float8_e4m3fn conversion).
"""
from __future__ import annotations

import dataclasses
import math

import torch

from . import synth

TID = {"q": 1, "kv_cmp": 2, "kv_win": 3, "qi": 4, "wi": 5, "ki": 6, "sink": 7, "kv_raw": 8, "gate": 9, "ape": 10,
       "gate_raw": 12, "qi8": 13, "sq": 14, "ki8": 15, "sk": 16, "ikv_raw": 17, "igate_raw": 18, "iape": 19}
FP8_CODE_STD = 64.0  # FP8 code draws are FP8_CODE_STD * N(0,1), inside the E4M3 range (448)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str            # "csa" (indexer + top-k + sparse MQA) or "hca" (dense MQA)
    dtype: torch.dtype
    B: int               # independent sequences
    Q: int               # queries
    H: int               # query heads (one shared KV head)
    D: int               # head dim (K = V)
    Hi: int              # indexer heads
    Di: int              # indexer head dim
    k: int               # top-k
    W: int               # sliding window
    win: int             # compressor window
    stride: int          # compressor stride (= ratio)
    N: int               # compressed entries per sequence (cache rows)
    T_raw: int           # rows of the raw-KV window buffer per sequence
    pos0: int            # absolute position of query 0 (queries of one sequence are consecutive)
    raw0: int            # absolute position of kv_win row 0
    # compressor run inside each step: raw tokens [c_src0, c_src0 + T_c) of
    # kv_win -> cache rows [c_dst0, c_dst0 + n) of every sequence
    T_c: int = 0
    c_src0: int = 0
    c_dst0: int = 0
    # one-off bulk compression of a whole raw sequence (kv_raw / gate_raw) into
    # sequence 0's cache, reported apart from the decode step
    bulk_T: int = 0
    seed: int = 0
    index_fmt: str = "bf16"  # indexer keys / queries: "bf16", or "e4m3" FP8 codes with per-row scales

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def q_per_seq(self) -> int:
        return self.Q // self.B

    def positions(self) -> torch.Tensor:
        """Absolute token position p of every query (int64 [Q])."""
        i = torch.arange(self.Q, dtype=torch.int64)
        return self.pos0 + i % self.q_per_seq

    def win_end(self) -> torch.Tensor:
        """Row of kv_win holding each query's own token (int32 [Q])."""
        return (self.positions() - self.raw0).to(torch.int32)


def _csa(**kw):
    return Workload(mode="csa", win=8, stride=4, **kw)


WORKLOADS = {
    # Tiny CSA prefill, fp32: every token of a 256-token sequence is a query.
    "tiny_csa_prefill_fp32": _csa(
        name="tiny_csa_prefill_fp32", dtype=torch.float32, B=1, Q=256, H=4, D=16, Hi=4, Di=16, k=16, W=16,
        N=63, T_raw=256, pos0=0, raw0=0, T_c=256, c_src0=0, c_dst0=0),
    # CSA decode at 64 K context, 32 sequences; the decode step also folds the
    # newest window (tokens L-8 .. L-1) into the last cache row.
    "csa_decode_64k": _csa(
        name="csa_decode_64k", dtype=torch.bfloat16, B=32, Q=32, H=64, D=512, Hi=64, Di=128, k=512, W=128,
        N=16383, T_raw=128, pos0=65535, raw0=65408, T_c=8, c_src0=120, c_dst0=16382),
    # HCA decode at 1 M context, 16 sequences, dense over all 8,192 entries.
    "hca_decode_1m": Workload(
        name="hca_decode_1m", mode="hca", dtype=torch.bfloat16, B=16, Q=16, H=64, D=512, Hi=64, Di=128, k=0,
        W=128, win=128, stride=128, N=8192, T_raw=128, pos0=1048575, raw0=1048448, T_c=128, c_src0=0,
        c_dst0=8191),
    # CSA prefill chunk: 4,096 new tokens after a 131,072-token context.
    "csa_prefill_chunk_4k": _csa(
        name="csa_prefill_chunk_4k", dtype=torch.bfloat16, B=1, Q=4096, H=64, D=512, Hi=64, Di=128, k=512,
        W=128, N=33791, T_raw=4223, pos0=131072, raw0=130945, T_c=4100, c_src0=123, c_dst0=32767),
    # CSA decode at 1 M context, 8 sequences, top-1024; sequence 0's cache can
    # be produced by compressing its 1,048,576 raw tokens (the bulk run).
    "csa_decode_1m": _csa(
        name="csa_decode_1m", dtype=torch.bfloat16, B=8, Q=8, H=64, D=512, Hi=64, Di=128, k=1024, W=128,
        N=262143, T_raw=128, pos0=1048575, raw0=1048448, T_c=8, c_src0=120, c_dst0=262142, bulk_T=1048576),
}
# The 64K decode batch in the V4-Pro attention shape: 128 query heads, top-1024
# ("DeepSeek-V4 Architecture Analysis", ARCHITECTURE_SPEC["DeepSeek-V4-Pro"]:
# num_heads 128, index_topk 1024, the same 512-dim head and 64 x 128 indexer).
WORKLOADS["csa_decode_64k_pro"] = dataclasses.replace(WORKLOADS["csa_decode_64k"], name="csa_decode_64k_pro",
                                                      H=128, k=1024)
# The 64K decode batch with the FP8 (E4M3) indexer.
WORKLOADS["csa_decode_64k_fp8"] = dataclasses.replace(WORKLOADS["csa_decode_64k"], name="csa_decode_64k_fp8",
                                                      index_fmt="e4m3")


def tensor_shape(w: Workload, name: str):
    return {
        "q": (w.Q, w.H, w.D), "kv_cmp": (w.B, w.N, w.D), "kv_win": (w.B, w.T_raw, w.D),
        "qi": (w.Q, w.Hi, w.Di), "wi": (w.Q, w.Hi), "ki": (w.B, w.N, w.Di), "sink": (w.H,),
        "kv_raw": (1, w.bulk_T, w.D), "gate_raw": (1, w.bulk_T, w.D), "ape": (w.win, w.D),
        "gate": (w.B, w.T_c, w.D), "qi8": (w.Q, w.Hi, w.Di), "sq": (w.Q, w.Hi), "ki8": (w.B, w.N, w.Di),
        "sk": (w.B, w.N), "ikv_raw": (1, w.bulk_T, w.Di), "igate_raw": (1, w.bulk_T, w.Di), "iape": (w.win, w.Di),
    }[name]


def _dtype_of(w: Workload, name: str):
    if name in ("qi8", "ki8"):
        return torch.uint8
    return torch.float32 if name in ("wi", "sink", "ape", "iape", "norm_w", "sq", "sk") else w.dtype


def _codes(x: torch.Tensor) -> torch.Tensor:
    return (x * FP8_CODE_STD).to(torch.float8_e4m3fn).view(torch.uint8)


def make(w: Workload, name: str, device="cpu") -> torch.Tensor:
    """Materialise one input tensor of workload ``w`` on ``device``."""
    shape = tensor_shape(w, name)
    dt = _dtype_of(w, name)
    if name == "wi":
        return synth.uniform(w.seed, TID[name], shape, dtype=dt, device=device)
    if name in ("sq", "sk"):
        return synth.uniform(w.seed, TID[name], shape, device=device) / 64 + 1.0 / 256
    if name in ("qi8", "ki8"):
        return _codes(synth.normal(w.seed, TID[name], shape, device=device))
    std = 0.1 if name in ("ape", "iape") else 1.0
    return synth.normal(w.seed, TID[name], shape, std=std, dtype=dt, device=device)


def rows(w: Workload, name: str, flat_rows) -> torch.Tensor:
    """Rows of a tensor (index into its flattened leading dims), regenerated
    on the host in the workload dtype."""
    shape = tensor_shape(w, name)
    if name in ("qi8", "ki8"):
        return _codes(synth.normal_rows(w.seed, TID[name], shape, flat_rows))
    if name in ("sq", "sk"):
        flat = torch.as_tensor(flat_rows, dtype=torch.int64)
        return synth.uniform_at(w.seed, TID[name], flat) / 64 + 1.0 / 256
    std = 0.1 if name in ("ape", "iape") else 1.0
    return synth.normal_rows(w.seed, TID[name], shape, flat_rows, std=std, dtype=_dtype_of(w, name))


def norm_w(w: Workload, device="cpu") -> torch.Tensor:
    return torch.ones(w.D, dtype=torch.float32, device=device)


def shard(w: Workload, rank: int) -> Workload:
    """The batch that process ``rank`` serves when several GPUs each run their
    own independent sequences: the same shapes, its own draws (rank 0's batch
    is ``w`` itself)."""
    if rank < 0:
        raise ValueError("rank must be >= 0")
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def small(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some fields changed (test-size variants)."""
    return dataclasses.replace(w, **changes)
