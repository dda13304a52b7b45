"""Benchmark of the CSA/HCA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload csa_decode_64k] [--no-secondary] [--no-cpu-baseline]

One step = one pass of the whole path over one batch of the workload: for
the CSA decode workloads, fold the newest raw window into the compressed
cache (csa_compress), score + select (csa_index_topk) and attend
(csa_sparse_mqa); for the HCA workload, append + hca_mqa. Inputs are seeded
synthetic tensors of the DeepSeek-V4-Flash shapes, resident in HBM. The step
is captured once in a CUDA graph and replayed; L2 is flushed (a 256 MB
write, then a 256 MB read of another buffer so that no dirty line is left to
write back) before every timed step, outside the step's events.

Multi-GPU (torchrun): one process per GPU, each serving its own batch of
independent sequences (weak scaling, no collective on the data path); the
step time is the max over ranks. Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores on the same
workload (rank 0 only) and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressed_sparse_attention_15_b200 import _lib, ops, workloads as WL  # noqa: E402
from compressed_sparse_attention_15_b200.step import DecodeStep  # noqa: E402

METRIC = "CSA/HCA decode queries/s at 64K–1M ctx; HBM GB/s and % of roofline"
UNIT = "queries/s"
FLUSH_BYTES = 256 << 20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------
# Algorithmic bytes / FLOPs (what the method must move; scratch excluded)
# --------------------------------------------------------------------------

def algo_bytes(w: WL.Workload):
    """Per-step algorithmic bytes of each kernel family (dtype sizes: bf16 2,
    fp32 4, int32 4)."""
    e = 2 if w.dtype == torch.bfloat16 else 4
    n_vis = w.N  # decode: every entry is visible
    b = {}
    b["compress"] = w.B * (2 * w.T_c * w.D * e + w.win * w.D * 4 + w.D * 4
                           + ((w.T_c - w.win) // w.stride + 1) * w.D * e)
    if w.mode == "csa":
        if w.index_fmt == "e4m3":
            # FP8 key rows + one fp32 scale per entry; FP8 query heads + scales + weights
            b["index_scores"] = w.Q * (n_vis * (w.Di + 4) + w.Hi * w.Di + 2 * w.Hi * 4)
        else:
            b["index_scores"] = w.Q * (n_vis * w.Di * e + w.Hi * w.Di * e + w.Hi * 4)
        b["topk"] = w.Q * w.k * 4
        rows = w.k + w.W
        b["mqa"] = w.Q * (rows * w.D * e + 2 * w.H * w.D * e + w.k * 4 + w.H * 4)
    else:
        rows = n_vis + w.W
        b["mqa"] = w.Q * (rows * w.D * e + 2 * w.H * w.D * e + w.H * 4)
    return b


def algo_flops(w: WL.Workload):
    """Per-step FLOPs of the contractions: the indexer's products over every
    visible entry of every query, and QK^T + PV over each query's rows."""
    n_vis = ops.visible_entries(w.positions(), w.win, w.stride).double()
    f = {}
    if w.mode == "csa":
        f["index_scores"] = float(n_vis.sum()) * w.Hi * w.Di * 2
        rows = float(torch.clamp(n_vis, max=w.k).sum()) + w.Q * w.W
    else:
        rows = float(n_vis.sum()) + w.Q * w.W
    f["mqa"] = rows * w.H * w.D * 4
    return f


# The other workloads, each one line of "secondary": (label, workload, append
# RoPE (rope_dims, theta) or None). The RoPE line is the 64 K decode step with
# the cache append rotating the new entry's last 64 dims (qk_rope_head_dim 64,
# compress_rope_theta 160000 of the Flash configuration).
SECONDARY = (("hca_decode_1m", "hca_decode_1m", None), ("csa_decode_1m", "csa_decode_1m", None),
             ("csa_decode_64k_fp8", "csa_decode_64k_fp8", None), ("csa_decode_64k_pro", "csa_decode_64k_pro", None),
             ("csa_prefill_chunk_4k", "csa_prefill_chunk_4k", None),
             ("csa_decode_64k_append_rope", "csa_decode_64k", (64, 160000.0)))

# A step part whose algorithmic bytes and FLOPs are another's: the attention
# with the selection made inside it moves what the attention moves.
PART_ALIAS = {"topk_mqa": "mqa"}
# One csa_decode_step call moves the whole step's bytes.
WHOLE_STEP = "decode_step"


def part_amount(table, name):
    """Algorithmic bytes (or FLOPs) of one step part."""
    if name == WHOLE_STEP:
        return sum(table.values())
    return table.get(PART_ALIAS.get(name, name))


def prefill(w: WL.Workload) -> bool:
    """Several queries of one sequence share its compressed keys (a causal
    prefill chunk): the indexer is then tensor-bound, not HBM-bound."""
    return w.q_per_seq > 1


# --------------------------------------------------------------------------
# The step
# --------------------------------------------------------------------------

class Step:
    """Device-resident inputs of one workload wrapped in the package's
    DecodeStep (graph-captured decode step)."""

    # inputs that change every decode step; they live in one staging buffer so
    # that the end-to-end run moves them with a single host-to-device copy
    PER_STEP = ("q", "gate", "qi", "wi")

    def __init__(self, w: WL.Workload, device, graph: bool = True, caches=None, fused: bool = True, rope=None):
        self.w = w
        self.dev = device
        self.graph = graph
        self.fused = fused
        self.rope = rope  # (rope_dims, theta): RoPE fused into the append
        fp8 = w.index_fmt == "e4m3"
        per_step = self.PER_STEP if not fp8 else ("q", "gate", "qi8", "sq", "wi")
        names = [n for n in per_step if w.mode == "csa" or n not in ("qi", "wi", "qi8", "sq")]
        shapes = {n: WL.tensor_shape(w, n) for n in names}
        shapes["kv_new"] = (w.B, w.D)  # the newest raw token of each sequence
        dts = {n: (torch.float32 if n in ("wi", "sq") else torch.uint8 if n == "qi8" else w.dtype) for n in shapes}
        offs, total = {}, 0
        for n, shp in shapes.items():
            offs[n] = total
            total += -(-math.prod(shp) * torch.empty((), dtype=dts[n]).element_size() // 256) * 256
        self.stage = torch.empty(total, dtype=torch.uint8, device=device)
        self.t = {}
        for n, shp in shapes.items():
            nb = math.prod(shp) * torch.empty((), dtype=dts[n]).element_size()
            self.t[n] = self.stage[offs[n]:offs[n] + nb].view(dts[n]).view(shp)
        if caches is None:
            caches = {n: WL.make(w, n, device) for n in ("kv_cmp", "kv_win", "sink", "ape")}
            if w.mode == "csa":
                for n in (("ki8", "sk") if fp8 else ("ki",)):
                    caches[n] = WL.make(w, n, device)
        self.caches = caches
        self.t.update(caches)
        for n in names:
            self.t[n].copy_(WL.make(w, n, device))
        self.t["kv_new"].copy_(self.t["kv_win"][:, -1])
        t = self.t
        self.ds = DecodeStep(
            q=t["q"], kv_cmp=t["kv_cmp"], kv_win=t["kv_win"], sink=t["sink"], scale=w.scale, win_len=w.W,
            win_end=w.win_end().to(device), n_cmp=ops.visible_entries(w.positions().to(device), w.win, w.stride),
            ape=t["ape"], norm_w=WL.norm_w(w, device), gate=t["gate"], append_src0=w.c_src0, append_dst0=w.c_dst0,
            win=w.win, stride=w.stride, qi=t.get("qi"), wi=t.get("wi"), ki=t.get("ki"),
            k=w.k if w.mode == "csa" else None, graph=graph,
            qi8=t.get("qi8"), sq=t.get("sq"), ki8=t.get("ki8"), sk=t.get("sk"), fused=fused,
            append_rope=None if rope is None else
            (rope[0], rope[1], torch.full((w.B,), w.raw0 + w.c_src0, dtype=torch.int64, device=device)))
        self.out = self.ds.out
        self._scores = None

    def twin(self):
        """A second step over the same caches with its own input staging
        buffer and output (double buffering for the end-to-end pipeline)."""
        return Step(self.w, self.dev, graph=self.graph, caches=self.caches, fused=self.fused, rope=self.rope)

    def parts(self):
        """The step's kernels one call at a time (per-kernel timing and the
        profiling aid). Without the fused selection, the CSA select call is
        split into its two kernels, scores then top-k, through their own entry
        points."""
        ds = self.ds
        if not ds.csa or ds.fuse_select or ds.fused:
            return ds.parts()
        if self._scores is None:
            self._scores = torch.empty((self.w.Q, self.w.N), dtype=torch.float32, device=self.dev)
            self._ws_s, self._ws_t = ops.Workspace(self.dev), ops.Workspace(self.dev)
        sc = self._scores
        if ds.fp8:
            score = lambda: ops.index_scores_fp8(ds.qi8, ds.sq, ds.wi, ds.ki8, ds.sk, ds.n_cmp, out=sc, ws=self._ws_s)
        else:
            score = lambda: ops.index_scores(ds.qi, ds.wi, ds.ki, ds.n_cmp, out=sc, ws=self._ws_s)
        return [("compress", ds.append),
                ("index_scores", score),
                ("topk", lambda: ops.topk(sc, ds.n_cmp, ds.k, out=ds.idx, ws=self._ws_t)),
                ("mqa", ds.attend)]

    def run(self):
        return self.ds.run()


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device, path=None):
        try:
            self.idx = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.idx = str(torch.cuda.current_device())
        self.proc = None
        # the raw samples (the JSON line carries their summary)
        self.path = path or os.path.join(tempfile.gettempdir(), f"csa_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            if os.path.dirname(self.path):
                os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 8:
                    try:
                        rows.append((float(p[0]), float(p[1]), p[3:8]))
                    except ValueError:
                        pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for _, _, r in rows:
            for n, v in zip(names, r[1:5]):
                if v.lower() == "active":
                    seen.add(n)
        loaded = sorted(r[0] for r in rows)
        top = loaded[len(loaded) // 2:]  # samples under load sit in the upper half
        return {"sm_mhz": statistics.median(top), "sm_max_mhz": max(r[1] for r in rows), "reasons": sorted(seen),
                "samples": len(rows)}


class L2Flush:
    """Evicts L2 between timed steps: a 256 MB write (twice the L2), then a
    256 MB read of another buffer, so that the write's dirty lines are written
    back here and not during the next timed step."""

    def __init__(self, device):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def _sync_barrier(dist_on):
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
        torch.cuda.synchronize()


def max_over_ranks(ms: float, dist_on: bool, device) -> float:
    """The job's step time: the slowest rank's mean step time."""
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if dist_on:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, q_per_rank: int, ms_max: float) -> float:
    """Whole-job queries/s: every rank serves q_per_rank queries per step."""
    return world * q_per_rank / (ms_max * 1e-3)


def _time_steps(step, flush, stream, K):
    """Mean device time (ms) of K graph replays, L2 flushed before each."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush()
        evs[i][0].record(stream)
        step.run()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / K


def time_ours(args, w: WL.Workload, device, dist_on, rank, world, secondary=False, rope=None):
    """Times the step on both paths (the whole step as one csa_decode_step
    call, its kernels chained on one stream; and the separate calls, the
    append on a forked stream), reports the faster; the other path's time and the
    separate kernels' per-kernel times are kept for the record."""
    flush = L2Flush(device)
    stream = torch.cuda.current_stream(device)
    steps, launches = {}, {}
    for fused in (True, False):
        if args.path != "both" and (args.path == "step_call") != fused:
            continue
        n0 = _lib.lib().csa_launch_count()
        caches = steps[True].caches if True in steps else None
        steps[fused] = Step(w, device, caches=caches, fused=fused, rope=rope)  # runs once eagerly, then captured
        launches[fused] = (_lib.lib().csa_launch_count() - n0) // 2
        for _ in range(max(3, args.warmup)):
            steps[fused].run()
    torch.cuda.synchronize()
    K0 = max(5, args.steps // 5)
    trial = {f: _time_steps(st, flush, stream, K0) for f, st in steps.items()}
    # the faster path (the per-kernel times come from the separate calls either way)
    fused = len(trial) == 1 and True in trial or (len(trial) == 2 and trial[True] <= trial[False])
    step = steps[fused]
    launches_per_step = launches[fused]

    K = args.steps if not secondary else max(10, args.steps // 4)
    for st in steps.values():
        if st is not step:
            st.ds.graph = None  # release the other path's graph before the timed region
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = Clocks(device, args.clock_log)
    _sync_barrier(dist_on)
    wall0 = time.perf_counter()
    with clocks:
        time.sleep(0.2)
        for i in range(K):
            flush()
            evs[i][0].record(stream)
            step.run()
            evs[i][1].record(stream)
        _sync_barrier(dist_on)
    wall = time.perf_counter() - wall0
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = sum(step_ms) / K
    ms_max = max_over_ranks(ms, dist_on, device)

    # Per-kernel durations: the same kernels launched one by one with events
    # between them (a host-side head start keeps the launches queued); for
    # both paths when both were built.
    per = {}
    for st in steps.values():
        parts = st.parts()
        names = [n for n, _ in parts]
        acc = {n: 0.0 for n in names}
        Kp = max(5, K // 2)
        for _ in range(Kp):
            flush()
            torch.cuda._sleep(2_000_000)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
            ev[0].record(stream)
            for i, (_, f) in enumerate(st.parts()):
                f()
                ev[i + 1].record(stream)
            torch.cuda.synchronize()
            for i, n in enumerate(names):
                acc[n] += ev[i].elapsed_time(ev[i + 1]) / Kp
        per.update(acc)
    status = step.ds.status()
    paths = {("step_call" if f else "separate"): round(v, 4) for f, v in trial.items()}
    return {"ms": ms_max, "ms_local": ms, "per_kernel_ms": per, "launches_per_step": int(launches_per_step),
            "wall_s": wall, "clocks": clocks.summary(), "status": status, "K": K, "step": step,
            "path": "step_call" if fused else "separate", "paths_ms": paths}


def time_bulk_compress(args, w: WL.Workload, device, hbm_gbs):
    """The one-off compression of a 1 M-token raw sequence (kv_raw, gate_raw
    [1, bulk_T, 512] bf16 -> [1, (bulk_T - 8)/4 + 1, 512]), timed alone."""
    kv = WL.make(w, "kv_raw", device)
    gate = WL.make(w, "gate_raw", device)
    ape = WL.make(w, "ape", device)
    nw = WL.norm_w(w, device)
    n = (w.bulk_T - w.win) // w.stride + 1
    out = torch.empty((1, n, w.D), dtype=w.dtype, device=device)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream(device)
    for _ in range(3):
        ops.compress(kv, gate, ape, nw, w.win, w.stride, out=out)
    K = max(5, args.steps // 4)
    ms = 0.0
    for _ in range(K):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ops.compress(kv, gate, ape, nw, w.win, w.stride, out=out)
        b.record(stream)
        torch.cuda.synchronize()
        ms += a.elapsed_time(b) / K
    nbytes = 2 * w.bulk_T * w.D * 2 + n * w.D * 2 + w.win * w.D * 4 + w.D * 4
    gbps = nbytes / (ms * 1e-3) / 1e9
    return {"tokens": w.bulk_T, "entries": n, "ms": round(ms, 4), "GBps": round(gbps, 1),
            "frac": round(gbps / hbm_gbs, 4), "bytes": nbytes, "tokens_per_s": round(w.bulk_T / (ms * 1e-3), 1)}


def time_index_compress(args, w: WL.Workload, device, hbm_gbs):
    """The indexer's own compressor over the 1 M-token indexer stream
    (ikv_raw, igate_raw [1, bulk_T, 128] bf16 -> Hadamard-rotated E4M3 codes
    [1, (bulk_T - 8)/4 + 1, 128] + one fp32 scale per entry), then the Hadamard
    rotation + E4M3 quantisation of one decode batch's indexer queries
    ([Q * Hi, 128] bf16), each timed alone."""
    kv = WL.make(w, "ikv_raw", device)
    gate = WL.make(w, "igate_raw", device)
    ape = WL.make(w, "iape", device)
    nw = torch.ones(w.Di, dtype=torch.float32, device=device)
    qi = WL.make(WL.WORKLOADS["csa_decode_64k"], "qi", device).reshape(-1, w.Di)
    n = ops.num_entries(w.bulk_T, w.win, w.stride)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream(device)

    def timed(f):
        for _ in range(3):
            f()
        K = max(5, args.steps // 4)
        ms = 0.0
        for _ in range(K):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            f()
            b.record(stream)
            torch.cuda.synchronize()
            ms += a.elapsed_time(b) / K
        return ms

    ms_c = timed(lambda: ops.index_compress(kv, gate, ape, nw, w.win, w.stride, fp8=True))
    ms_h = timed(lambda: ops.hadamard_rows(qi, fp8=True))
    by_c = 2 * w.bulk_T * w.Di * 2 + n * (w.Di + 4) + w.win * w.Di * 4 + w.Di * 4
    by_h = qi.shape[0] * (w.Di * 2 + w.Di + 4)
    gc, gh = by_c / (ms_c * 1e-3) / 1e9, by_h / (ms_h * 1e-3) / 1e9
    return {"csa_index_compress": {"tokens": w.bulk_T, "entries": n, "out": "e4m3 codes + fp32 scales",
                                   "ms": round(ms_c, 4), "GBps": round(gc, 1), "frac": round(gc / hbm_gbs, 4),
                                   "bytes": by_c, "tokens_per_s": round(w.bulk_T / (ms_c * 1e-3), 1)},
            "csa_hadamard_rows": {"rows": qi.shape[0], "dim": w.Di, "out": "e4m3 codes + fp32 scales",
                                  "ms": round(ms_h, 4), "GBps": round(gh, 1), "bytes": by_h,
                                  "note": "one decode batch's query rows: launch-latency bound"}}


def path_parts(per_kernel_ms, path):
    """The per-kernel times of one path (empty if it was not built): the step call, or
    the separate kernels."""
    if path == "step_call":
        return {k: v for k, v in per_kernel_ms.items() if k == WHOLE_STEP}
    return {k: v for k, v in per_kernel_ms.items() if k != WHOLE_STEP}


def roofline_of(w, per_kernel_ms, hbm_gbs, traffic=None, tflops=None):
    """Roofline of the kernel with the most algorithmic bytes in the step
    (decode: HBM-bound), or with the most FLOPs against the bf16 tensor peak
    (prefill, given ``tflops``). ``traffic`` maps a part name to its measured
    DRAM bytes per launch."""
    if prefill(w) and tflops:
        af = algo_flops(w)
        name, fl = max(((k, part_amount(af, k)) for k in per_kernel_ms if part_amount(af, k) is not None),
                       key=lambda x: x[1])
        achieved = fl / (per_kernel_ms[name] * 1e-3) / 1e12
        return {"kernel": name, "bound": "tensor", "achieved": round(achieved, 1), "peak": tflops, "unit": "TFLOP/s",
                "frac": round(achieved / tflops, 4), "traffic": (traffic or {}).get(name), "flops_per_launch": int(fl)}
    ab = algo_bytes(w)
    best = max(((k, part_amount(ab, k)) for k in per_kernel_ms if part_amount(ab, k) is not None),
               key=lambda x: x[1])
    name, nbytes = best
    traffic = (traffic or {}).get(name)
    ms = per_kernel_ms[name]
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_gbs, "unit": "GB/s",
            "frac": round(achieved / hbm_gbs, 4), "traffic": traffic, "bytes_per_launch": int(nbytes)}


def load_traffic(path, workload):
    """DRAM bytes per launch of each part, from the committed ncu summary
    (profiles/traffic.json): {part: bytes}, for the kernels as they stand."""
    try:
        with open(path) as f:
            entry = json.load(f).get(workload) or {}
    except (OSError, ValueError):
        return {}
    return {part: v["dram_bytes_per_launch"] for part, v in entry.items()
            if isinstance(v, dict) and v.get("dram_bytes_per_launch")}


def e2e_ours(args, w: WL.Workload, step: Step, device):
    """Same metric through the public API with host buffers, as a serving loop
    runs it: every step copies its per-step inputs (q, qi, wi, the window's
    gates and the newest raw token of each sequence, packed in one pinned
    staging buffer) to the device in one copy, places the new token in the
    raw-KV buffer, runs the step and reads its output back. Two input/output
    buffer sets alternate, so that step i's copies overlap the compute of its
    neighbours (copies on their own streams, ordered by events). The step's
    working set (the caches it reads) exceeds L2, so the steps run back to
    back; the timed region spans K whole steps, first copy to last read."""
    pair = [step, step.twin()]
    host = step.stage.cpu().pin_memory()
    outs = [torch.empty(st.out.shape, dtype=st.out.dtype, pin_memory=True) for st in pair]
    h2d = host.numel()
    d2h = outs[0].numel() * outs[0].element_size()
    comp = torch.cuda.current_stream(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in pair]
    ev_done = [torch.cuda.Event() for _ in pair]
    ev_out = [torch.cuda.Event() for _ in pair]
    kv_win = step.t["kv_win"]

    def one(i):
        b = i % 2
        st = pair[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])  # step i - 2 has consumed this staging buffer
            st.stage.copy_(host, non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])  # step i - 2's output has been read back
        kv_win[:, -1].copy_(st.t["kv_new"])
        st.run()
        ev_done[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            outs[b].copy_(st.out, non_blocking=True)
            ev_out[b].record(s_out)

    K = max(20, args.steps)
    for i in range(4):  # warm-up
        one(i)
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    s_in.wait_stream(comp)
    for i in range(K):
        one(i)
    comp.wait_stream(s_out)
    e.record(comp)
    torch.cuda.synchronize()
    ms = a.elapsed_time(e) / K
    return {"value": round(w.Q / (ms * 1e-3), 1), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 4),
            "pipelined": "two buffer sets; copies on their own streams overlap neighbouring steps"}


# --------------------------------------------------------------------------
# The oracle on the host (CPU baseline and --impl reference)
# --------------------------------------------------------------------------

def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def time_oracle(w: WL.Workload, steps: int, budget_s: float, queries=None, rope=None):
    """Time the fp64 oracle on the host over the step's work: per sequence the
    append (the compressor over the step's raw tokens, with RoPE when ``rope``
    = (rope_dims, theta) is given), per query the indexer top-k (CSA) and the
    attention. ``queries`` (default: all) is the subset run; the time is
    extrapolated to the whole batch (sequences x append time + queries x query
    time). Up to ``steps`` passes; stops once ``budget_s`` of oracle time is
    spent (after at least one query). Input regeneration and row gathering are
    not timed."""
    import numpy as np

    import oracle as O

    qs = list(range(w.Q)) if queries is None else list(queries)
    ape = WL.make(w, "ape")
    sink = WL.make(w, "sink")
    fp8 = w.mode == "csa" and w.index_fmt == "e4m3"
    if w.mode == "csa":
        iq = {n: WL.make(w, n) for n in (("sq", "wi") if fp8 else ("wi",))}
    knames = (("ki8", "sk") if fp8 else ("ki",)) if w.mode == "csa" else ()
    # every sequence's indexer keys at once when they fit in a few hundred MB
    keys_all = {n: WL.make(w, n) for n in knames} if w.B * w.N * w.Di <= (80 << 20) else None
    t_app, n_app, t_q, n_q = 0.0, 0, 0.0, 0
    seq_cache, q_cache, raw_cache = {}, {}, {}  # regenerated inputs, kept for the next pass
    for _ in range(max(1, steps)):
        for q in qs:
            b = q // w.q_per_seq
            if b not in seq_cache:
                seq_cache.clear()
                if b not in raw_cache:
                    raw_cache[b] = (WL.rows(w, "kv_win", b * w.T_raw + torch.arange(w.c_src0, w.c_src0 + w.T_c)),
                                    WL.rows(w, "gate", b * w.T_c + torch.arange(w.T_c)))
                raw, gate = raw_cache[b]
                t0 = time.perf_counter()
                if rope:
                    new = O.compress_rope(raw, gate, ape, np.ones(w.D), w.win, w.stride, w.raw0 + w.c_src0, rope[1],
                                          rope[0])
                else:
                    new = O.compress(raw, gate, ape, np.ones(w.D), w.win, w.stride)
                new = O.round_to(new, "bf16")
                t_app += time.perf_counter() - t0
                n_app += 1
                if keys_all is not None:
                    keys = {n: t[b] for n, t in keys_all.items()}
                else:
                    keys = {n: WL.rows(w, n, b * w.N + torch.arange(w.N)) for n in knames}
                seq_cache[b] = (new, keys)
            new, keys = seq_cache[b]
            p = int(w.positions()[q])
            if q not in q_cache:
                q_cache[q] = {"q": WL.rows(w, "q", q * w.H + torch.arange(w.H))}
                if w.mode == "csa":
                    q_cache[q]["qi"] = WL.rows(w, "qi8" if fp8 else "qi", q * w.Hi + torch.arange(w.Hi))
            qc = q_cache[q]
            q_rows, qi_rows = qc["q"], qc.get("qi")
            t0 = time.perf_counter()
            if fp8:
                idx, _ = O.index_topk_fp8(qi_rows.numpy(), iq["sq"][q], iq["wi"][q], keys["ki8"].numpy(),
                                          keys["sk"], p, w.k, w.win, w.stride)
                sel = idx[idx >= 0]
            elif w.mode == "csa":
                idx, _ = O.index_topk(qi_rows, iq["wi"][q], keys["ki"], p, w.k, w.win, w.stride)
                sel = idx[idx >= 0]
            else:
                sel = np.arange(O.n_visible(p, w.win, w.stride))
            t_q += time.perf_counter() - t0
            if "rows" not in qc:
                rows_c = O.round_to(WL.rows(w, "kv_cmp", b * w.N + torch.as_tensor(sel)), "bf16")
                fresh = (sel >= w.c_dst0) & (sel < w.c_dst0 + len(new))
                rows_c[fresh] = new[sel[fresh] - w.c_dst0]
                e = int(w.win_end()[q])
                rows_w = O.as_f64(WL.rows(w, "kv_win", b * w.T_raw + torch.arange(max(0, e - w.W + 1), e + 1)))
                qc["rows"] = np.concatenate([rows_c, rows_w])
            t0 = time.perf_counter()
            O.attend(q_rows, qc["rows"], sink, w.scale)
            t_q += time.perf_counter() - t0
            n_q += 1
            if t_app + t_q >= budget_s:
                break
        if t_app + t_q >= budget_s:
            break
    step_s = w.B * (t_app / n_app) + w.Q * (t_q / n_q)
    subset = "all queries" if queries is None else f"{len(qs)} evenly spaced queries"
    return {"value": w.Q / step_s, "unit": UNIT, "cores": int(_oracle_cores()), "kind": "oracle",
            "sample": f"{n_q} queries ({subset}, {n_app} appends) of {w.name}"
                      f"{' with RoPE append' if rope else ''}, fp64 numpy, extrapolated to the batch of {w.Q}; "
                      f"input regeneration untimed", "seconds": round(t_app + t_q, 2)}


def time_oracle_compress(w: WL.Workload, budget_s: float, indexer: bool = False):
    """Time the oracle's compressor over consecutive chunks of the 1 M-token
    raw sequence (4,096 entries a chunk) until ``budget_s`` is spent; tokens/s.
    ``indexer``: the indexer's compressor (Hadamard rotation, E4M3 codes) on
    its 128-dim stream."""
    import numpy as np

    import oracle as O

    D = w.Di if indexer else w.D
    names = ("ikv_raw", "igate_raw") if indexer else ("kv_raw", "gate_raw")
    ape = WL.make(w, "iape" if indexer else "ape")
    per = 4096 * w.stride + w.win - w.stride  # tokens of a 4,096-entry chunk
    t, toks, i = 0.0, 0, 0
    while t < budget_s and (i + 1) * 4096 * w.stride <= w.bulk_T:
        r = torch.arange(i * 4096 * w.stride, min(w.bulk_T, i * 4096 * w.stride + per))
        kv, gate = WL.rows(w, names[0], r), WL.rows(w, names[1], r)
        t0 = time.perf_counter()
        if indexer:
            O.quantize_rows_e4m3(O.index_compress(kv, gate, ape, np.ones(D), w.win, w.stride))
        else:
            O.round_to(O.compress(kv, gate, ape, np.ones(D), w.win, w.stride), "bf16")
        t += time.perf_counter() - t0
        toks += 4096 * w.stride
        i += 1
    return {"value": round(toks / t, 1), "unit": "tokens/s", "cores": int(_oracle_cores()), "kind": "oracle",
            "sample": f"{i} chunks of 4,096 entries ({toks} tokens) of the {w.bulk_T}-token "
                      f"{'indexer ' if indexer else ''}stream, fp64 numpy", "seconds": round(t, 2)}


# --------------------------------------------------------------------------

def workload_config(w: WL.Workload):
    return {"workload": w.name, "batch": w.Q, "context": w.pos0 + 1, "heads": f"{w.H}q:1kv", "head_dim": w.D,
            "indexer": f"{w.Hi}x{w.Di} {w.index_fmt}" if w.mode == "csa" else None, "topk": w.k or None, "window": w.W,
            "compress": f"win {w.win} stride {w.stride}", "l2": "flushed before every timed step: 256 MB write, then 256 MB read (clean eviction)",
            "inputs": "seeded synthetic (counter-based generator), resident in HBM"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="csa_decode_64k", choices=[n for n in WL.WORKLOADS if n != "tiny_csa_prefill_fp32"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-log", default=None,
                    help="file for the nvidia-smi samples taken during the timed region (default: a temporary file)")
    ap.add_argument("--traffic-json", default=os.path.join(ROOT, "profiles", "traffic.json"))
    ap.add_argument("--path", default="both", choices=["both", "step_call", "separate"],
                    help="the decode step as one csa_decode_step call (its kernels chained on one stream), as "
                         "separate calls, or the faster of both")
    ap.add_argument("--once", action="store_true",
                    help="profiling aid: build the step without a graph and launch each of its kernels once more")
    ap.add_argument("--once-bulk", default=None, choices=["compress", "index_compress"],
                    help="profiling aid: run the 1 M-token bulk compression (or the indexer's) twice, untimed")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = WL.WORKLOADS[args.workload]
    hbm, tflops, peak_kind = _peaks()

    if args.impl == "reference":
        if rank != 0:
            return 0
        base = time_oracle(w, max(1, args.steps), budget_s=60.0)
        line = {"metric": METRIC, "value": round(base["value"], 3), "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(w.Q / base["value"] * 1e3, 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": workload_config(w), "impl": "reference",
                "cpu_baseline": base, "e2e": {"value": round(base["value"], 3), "unit": UNIT,
                                              "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    if args.once_bulk:
        wb, dev = WL.WORKLOADS["csa_decode_1m"], torch.device("cuda", 0)
        ix = args.once_bulk == "index_compress"
        kv = WL.make(wb, "ikv_raw" if ix else "kv_raw", dev)
        gate = WL.make(wb, "igate_raw" if ix else "gate_raw", dev)
        ape = WL.make(wb, "iape" if ix else "ape", dev)
        nw = torch.ones(kv.shape[-1], dtype=torch.float32, device=dev)
        for _ in range(2):
            if ix:
                ops.index_compress(kv, gate, ape, nw, wb.win, wb.stride, fp8=True)
            else:
                ops.compress(kv, gate, ape, nw, wb.win, wb.stride)
        torch.cuda.synchronize()
        print(json.dumps({"once_bulk": args.once_bulk, "tokens": wb.bulk_T}))
        return 0
    if args.once:
        step = Step(w, torch.device("cuda", 0), graph=False, fused=args.path == "step_call")  # runs the step once
        torch.cuda.synchronize()
        for _, f in step.parts():
            f()
        torch.cuda.synchronize()
        print(json.dumps({"once": w.name, "status": step.ds.status()}))
        return 0
    dist_on = world > 1
    if dist_on:
        import datetime

        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", torch.cuda.current_device())

    w = WL.shard(w, rank)  # this rank's own sequences (same shapes)
    r = time_ours(args, w, device, dist_on, rank, world)
    traffic = load_traffic(args.traffic_json, w.name)
    # the dominant kernel's own timing (the chained step runs the same kernels)
    roof = roofline_of(w, path_parts(r["per_kernel_ms"], "separate") or path_parts(r["per_kernel_ms"], r["path"]),
                       hbm, traffic, tflops)
    roof["peak_kind"] = f"{peak_kind} HBM copy bandwidth"
    e2e = e2e_ours(args, w, r["step"], device)
    del r["step"]
    torch.cuda.empty_cache()

    secondary = {}
    if not args.no_secondary and rank == 0 and not dist_on:
        for label, name, rope in SECONDARY:
            if name == w.name and rope is None:
                continue
            sw = WL.WORKLOADS[name]
            try:
                s = time_ours(args, sw, device, False, 0, 1, secondary=True, rope=rope)
                del s["step"]
                rf = roofline_of(sw, path_parts(s["per_kernel_ms"], "separate") or
                                 path_parts(s["per_kernel_ms"], s["path"]), hbm,
                                 load_traffic(args.traffic_json, label), tflops)
                line = {"workload": name, "queries_per_s": round(sw.Q / (s["ms"] * 1e-3), 1),
                        "ms_per_step": round(s["ms"], 4), "path": s["path"], "paths_ms": s["paths_ms"],
                        "per_kernel_ms": {k: round(v, 4) for k, v in s["per_kernel_ms"].items()}}
                if rope:
                    line["append"] = f"csa_compress_rope: rope_dims {rope[0]}, theta {rope[1]:g}"
                if prefill(sw):  # tensor-bound: the step's FLOPs against the bf16 peak
                    step_tf = sum(algo_flops(sw).values()) / (s["ms"] * 1e-3) / 1e12
                    line.update(step_TFLOPs=round(step_tf, 1), step_frac=round(step_tf / tflops, 4))
                else:
                    step_gbs = sum(algo_bytes(sw).values()) / (s["ms"] * 1e-3) / 1e9
                    line.update(step_GBps=round(step_gbs, 1), step_frac=round(step_gbs / hbm, 4))
                line.update(roofline=rf, status=s["status"])
                secondary[label] = line
            except Exception as ex:  # report, do not hide
                secondary[label] = {"error": repr(ex)}
            torch.cuda.empty_cache()
        w1m = WL.WORKLOADS["csa_decode_1m"]
        for label, fn in (("compress_1m_tokens", time_bulk_compress), ("indexer_compress_1m_tokens", time_index_compress)):
            try:
                secondary[label] = fn(args, w1m, device, hbm)
            except Exception as ex:
                secondary[label] = {"error": repr(ex)}
            torch.cuda.empty_cache()
        if not args.no_cpu_baseline:  # the oracle on the host cores, per line (bounded samples)
            for label, name, rope in SECONDARY:
                if label not in secondary or "error" in secondary[label]:
                    continue
                sw = WL.WORKLOADS[name]
                qs = None if not prefill(sw) else [round(i * (sw.Q - 1) / 63) for i in range(64)]
                try:
                    secondary[label]["cpu_baseline"] = time_oracle(sw, 1, budget_s=60.0, queries=qs, rope=rope)
                except Exception as ex:
                    secondary[label]["cpu_baseline"] = {"error": repr(ex)}
            for label, ix in (("compress_1m_tokens", False), ("indexer_compress_1m_tokens", True)):
                if "error" not in secondary.get(label, {"error": 1}):
                    try:
                        secondary[label]["cpu_baseline"] = time_oracle_compress(w1m, 3.0, indexer=ix)
                    except Exception as ex:
                        secondary[label]["cpu_baseline"] = {"error": repr(ex)}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline and not dist_on:
        cpu = time_oracle(w, 1000, budget_s=12.0)

    if rank == 0:
        step_bytes = sum(algo_bytes(w).values())
        value = job_value(world, w.Q, r["ms"])
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": r["K"],
            "warmup": args.warmup, "ms_per_step": round(r["ms"], 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w),
            "parallelism": f"replicas x{world} (independent sequences per GPU, no collective)",
            "step_GBps": round(step_bytes / (r["ms"] * 1e-3) / 1e9, 1),
            "step_roofline_frac": round(step_bytes / (r["ms"] * 1e-3) / 1e9 / hbm, 4),
            "path": r["path"], "paths_ms": r["paths_ms"],
            "per_kernel_ms": {k: round(v, 4) for k, v in r["per_kernel_ms"].items()},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": r["launches_per_step"] * r["K"], "launches_per_step": r["launches_per_step"],
            "clocks": r["clocks"], "device_status": r["status"], "wall_s_timed_region": round(r["wall_s"], 3),
            "secondary": secondary or None,
        }
        print(json.dumps(line))
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
