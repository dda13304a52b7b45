"""A whole decode step of one CSA or HCA attention layer, replayed from a
CUDA graph.

The step over device-resident caches is:
  1. fold the newest raw window of every sequence into its compressed cache
     (csa_compress, or csa_compress_rope with RoPE on the new entry's rope
     dims; CSA every 4 tokens, HCA every 128) -- on a forked stream,
     concurrently with 2 when the layer is CSA;
  2. CSA only: score every visible compressed entry and select the top-k
     (csa_index_topk, or csa_index_topk_fp8 with FP8 indexer inputs);
  3. attend over the selected (CSA) or all visible (HCA) entries + the
     sliding window + the per-head sink (csa_sparse_mqa / hca_mqa).
With fused=True the whole step is one csa_decode_step call: by default the
same kernels chained by programmatic dependent launch on one stream (CSA:
the scorer first, the append running in its tail, then the top-k, then the
attention, which computes its window tiles before the top-k is done), with
no second stream; persistent=True asks instead for the one persistent kernel in which
the selection and attention of some queries overlap the key scan of others
(measured slower: its per-query chains are latency-bound). With fused=False
(the default) the parts are separate calls, the append on a forked stream;
there, fuse_select=True makes a CSA step only score in 2
(csa_index_scores(_fp8)) and run 3 as csa_topk_sparse_mqa, the selection
inside the attention kernel where its launch plan allows.
The library never allocates or synchronises, so the launches are captured
once into a CUDA graph and each step is one graph launch. Buffers are bound
at construction; later steps see whatever the caller wrote into them.
"""
from __future__ import annotations

import torch

from . import ops


class DecodeStep:
    def __init__(self, *, q, kv_cmp, kv_win, sink, scale: float, win_len: int, win_end, n_cmp,
                 ape, norm_w, gate, append_src0: int, append_dst0: int, win: int, stride: int,
                 qi=None, wi=None, ki=None, k: int | None = None, out=None, graph: bool = True,
                 qi8=None, sq=None, ki8=None, sk=None, append_rope=None, fuse_select: bool = False,
                 fused: bool = False, persistent: bool = False):
        self.fp8 = qi8 is not None
        self.csa = qi is not None or self.fp8
        self.q, self.kv_cmp, self.kv_win, self.sink = q, kv_cmp, kv_win, sink
        self.scale, self.win_len, self.win_end, self.n_cmp = float(scale), int(win_len), win_end, n_cmp
        self.ape, self.norm_w, self.gate = ape, norm_w, gate
        self.win, self.stride = int(win), int(stride)
        T_c = gate.shape[1]
        n_new = ops.num_entries(T_c, self.win, self.stride)
        self.kv_src = kv_win[:, append_src0:append_src0 + T_c]
        self.cmp_dst = kv_cmp[:, append_dst0:append_dst0 + n_new]
        self.qi, self.wi, self.ki, self.k = qi, wi, ki, k
        self.qi8, self.sq, self.ki8, self.sk = qi8, sq, ki8, sk
        self.append_rope = append_rope  # (rope_dims, theta, pos0 int64 [B]): RoPE fused into the append
        dev = q.device
        self.out = out if out is not None else torch.empty_like(q)
        self.idx = torch.empty((q.shape[0], k), dtype=torch.int32, device=dev) if self.csa else None
        self.fused = bool(fused)
        self.persistent = bool(persistent)
        self.fuse_select = bool(fuse_select) and self.csa and not self.fused
        self.append_src0, self.append_dst0 = int(append_src0), int(append_dst0)
        self.scores = (torch.empty((q.shape[0], kv_cmp.shape[1]), dtype=torch.float32, device=dev)
                       if self.fuse_select else None)
        self.ws_index = ops.Workspace(dev)
        self.ws_mqa = ops.Workspace(dev)
        self.side = torch.cuda.Stream(dev)
        self.graph = None
        self.run_eager()  # sizes the workspaces and sets kernel attributes
        torch.cuda.synchronize(dev)
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._launch()
            self.graph = g

    # -- the parts, on the current stream --------------------------------
    def append(self):
        ops.compress(self.kv_src, self.gate, self.ape, self.norm_w, self.win, self.stride, out=self.cmp_dst,
                     rope=self.append_rope)

    def select(self):
        if self.fuse_select:  # scores only; the selection is made with the attention
            if self.fp8:
                ops.index_scores_fp8(self.qi8, self.sq, self.wi, self.ki8, self.sk, self.n_cmp, out=self.scores,
                                     ws=self.ws_index)
            else:
                ops.index_scores(self.qi, self.wi, self.ki, self.n_cmp, out=self.scores, ws=self.ws_index)
        elif self.fp8:
            ops.index_topk_fp8(self.qi8, self.sq, self.wi, self.ki8, self.sk, self.n_cmp, self.k, out=self.idx,
                               ws=self.ws_index)
        else:
            ops.index_topk(self.qi, self.wi, self.ki, self.n_cmp, self.k, out=self.idx, ws=self.ws_index)

    def attend(self):
        if self.fuse_select:
            ops.topk_sparse_mqa(self.scores, self.n_cmp, self.k, self.q, self.kv_cmp, self.kv_win, self.win_end,
                                self.sink, self.scale, self.win_len, out=self.out, idx_out=self.idx, ws=self.ws_mqa)
        elif self.csa:
            ops.sparse_mqa(self.q, self.kv_cmp, self.idx, self.kv_win, self.win_end, self.sink, self.scale,
                           self.win_len, out=self.out, ws=self.ws_mqa)
        else:
            ops.hca_mqa(self.q, self.kv_cmp, self.n_cmp, self.kv_win, self.win_end, self.sink, self.scale,
                        self.win_len, out=self.out, ws=self.ws_mqa)

    def step(self):
        """The whole step as one csa_decode_step call."""
        append = {"kv": self.kv_src, "gate": self.gate, "ape": self.ape, "norm_w": self.norm_w, "win": self.win,
                  "stride": self.stride, "row0": self.append_dst0, "rope": self.append_rope}
        if self.fp8:
            ops.decode_step(self.q, self.kv_cmp, self.kv_win, self.win_end, self.sink, self.scale, self.win_len,
                            self.n_cmp, qi8=self.qi8, sq=self.sq, wi=self.wi, ki8=self.ki8, sk=self.sk, k=self.k,
                            append=append, out=self.out, idx_out=self.idx, ws=self.ws_index,
                            persistent=self.persistent)
        elif self.csa:
            ops.decode_step(self.q, self.kv_cmp, self.kv_win, self.win_end, self.sink, self.scale, self.win_len,
                            self.n_cmp, qi=self.qi, wi=self.wi, ki=self.ki, k=self.k, append=append, out=self.out,
                            idx_out=self.idx, ws=self.ws_index, persistent=self.persistent)
        else:
            ops.decode_step(self.q, self.kv_cmp, self.kv_win, self.win_end, self.sink, self.scale, self.win_len,
                            self.n_cmp, append=append, out=self.out, ws=self.ws_index, persistent=self.persistent)

    def parts(self):
        if self.fused:
            return [("decode_step", self.step)]
        p = [("compress", self.append)]
        if self.fuse_select:
            p += [("index_scores", self.select), ("topk_mqa", self.attend)]
            return p
        if self.csa:
            p.append(("index_topk", self.select))
        p.append(("mqa", self.attend))
        return p

    def _launch(self):
        if self.fused:
            self.step()
            return
        main = torch.cuda.current_stream()
        if self.csa:
            # the append only feeds the attention: overlap it with the indexer
            self.side.wait_stream(main)
            with torch.cuda.stream(self.side):
                self.append()
            self.select()
            main.wait_stream(self.side)
        else:
            self.append()
        self.attend()

    def run_eager(self):
        """The step as individual launches (no graph)."""
        self._launch()

    def run(self):
        """One step: a single graph launch on the current stream."""
        if self.graph is None:
            self._launch()
        else:
            self.graph.replay()
        return self.out

    def status(self) -> int:
        """Synchronise and return (and clear) the device status bits."""
        return self.ws_index.status() | self.ws_mqa.status()
