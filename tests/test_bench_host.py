"""bench.py's bookkeeping on the host: the algorithmic bytes and FLOPs per
query of each workload (the quantities the roofline fractions divide by),
against the counts derived by hand from the workload shapes, and which
kernel each workload's roofline names. Runs without a GPU."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from compressed_sparse_attention_15_b200 import workloads as WL  # noqa: E402


def _per_query(name, parts):
    w = WL.WORKLOADS[name]
    b = bench.algo_bytes(w)
    return sum(b[p] for p in parts) / w.Q


def test_csa_64k_decode_bytes_per_query():
    # keys 16,383 x 128 bf16 + the 64 x 128 query block + 64 weights;
    # 512 selected + 128 window rows of 1 KB, q and out (64 x 512 bf16 each),
    # 512 indices read, 64 sink values; 512 indices written by the top-k.
    keys = 16383 * 128 * 2 + 64 * 128 * 2 + 64 * 4
    attn = 640 * 1024 + 2 * 64 * 512 * 2 + 512 * 4 + 64 * 4
    assert _per_query("csa_decode_64k", ("index_scores", "topk", "mqa")) == keys + 512 * 4 + attn == 5_001_472


def test_hca_1m_decode_bytes_per_query():
    assert _per_query("hca_decode_1m", ("mqa",)) == (8192 + 128) * 1024 + 2 * 64 * 512 * 2 + 64 * 4 == 8_651_008


def test_csa_1m_decode_bytes_per_query():
    keys = 262143 * 128 * 2 + 64 * 128 * 2 + 64 * 4
    attn = (1024 + 128) * 1024 + 2 * 64 * 512 * 2 + 1024 * 4 + 64 * 4
    assert _per_query("csa_decode_1m", ("index_scores", "topk", "mqa")) == keys + 1024 * 4 + attn == 68_444_416


def test_fp8_indexer_moves_132_bytes_per_entry():
    w = WL.WORKLOADS["csa_decode_64k_fp8"]
    per_q = bench.algo_bytes(w)["index_scores"] / w.Q
    assert per_q == 16383 * (128 + 4) + 64 * 128 + 2 * 64 * 4


def test_prefill_chunk_flops():
    # 4,096 causal queries at p = 131,072 .. 135,167 see 32,767 .. 33,790
    # entries: sum = 4,096 x 32,767 + (0 + 1 + ... + 1,023) (one more entry
    # every 4 tokens) -- counted through the visibility rule, products of
    # 64 heads x 128 dims; attention over 512 + 128 rows, 64 heads x 512 dims, QK and PV.
    w = WL.WORKLOADS["csa_prefill_chunk_4k"]
    f = bench.algo_flops(w)
    vis = sum(32767 + (i + 4 - 3) // 4 for i in range(4096))
    assert f["index_scores"] == vis * 64 * 128 * 2
    assert f["mqa"] == 4096 * 640 * 64 * 512 * 4
    assert f["index_scores"] == pytest.approx(2.233e12, rel=1e-3)
    assert f["mqa"] == pytest.approx(0.344e12, rel=2e-3)


@pytest.mark.parametrize("name,kernel,bound", [
    ("csa_decode_64k", "index_scores", "hbm"),
    ("csa_decode_1m", "index_scores", "hbm"),
    ("hca_decode_1m", "mqa", "hbm"),
    ("csa_prefill_chunk_4k", "index_scores", "tensor"),
])
def test_roofline_names_the_dominant_kernel(name, kernel, bound):
    w = WL.WORKLOADS[name]
    parts = [p for p in ("compress", "index_scores", "topk", "mqa") if w.mode == "csa" or p in ("compress", "mqa")]
    per_kernel_ms = {p: 0.01 for p in parts}
    rf = bench.roofline_of(w, per_kernel_ms, 6452.8, None, 1676.0)
    assert (rf["kernel"], rf["bound"]) == (kernel, bound)
    # the attention with the selection inside it counts as the attention
    if w.mode == "csa":
        fused = {"compress": 0.01, "index_scores": 0.01, "topk_mqa": 0.01}
        assert bench.roofline_of(w, fused, 6452.8, None, 1676.0)["kernel"] == kernel


def test_oracle_timing_on_a_query_subset():
    # the CPU-baseline leg: a subset of queries, extrapolated to the batch
    w = WL.WORKLOADS["tiny_csa_prefill_fp32"]
    r = bench.time_oracle(w, 1, 5.0, queries=[0, 100, 255], rope=(8, 10000.0))
    assert r["value"] > 0 and r["kind"] == "oracle"
    assert r["sample"].startswith("3 queries (3 evenly spaced queries, 1 appends)")


def test_secondary_lines_cover_the_other_workloads():
    names = {n for _, n, _ in bench.SECONDARY}
    assert names == set(WL.WORKLOADS) - {"tiny_csa_prefill_fp32"}
    assert any(rope for _, _, rope in bench.SECONDARY)


def test_committed_traffic_records_are_consistent():
    # profiles/traffic.json (the `traffic` of each bench line) holds, per
    # workload and bench part, positive DRAM bytes per launch whose source is
    # a committed summary that names the kernel; and bench.load_traffic reads
    # every bench workload's record.
    import json
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    bench_names = {n for _, n, _ in bench.SECONDARY} | {"csa_decode_64k"}
    for name, parts in rec.items():
        assert name in bench_names, name
        for part, v in parts.items():
            assert part in ("compress", "index_scores", "topk", "mqa"), (name, part)
            assert v["dram_bytes_per_launch"] > 0, (name, part)
            src = os.path.join(ROOT, v["source"])
            assert os.path.isfile(src), (name, part, v["source"])
            with open(src) as f:
                text = f.read()
            for kernel in v["kernel"].split(" + "):
                assert kernel in text, (name, part, kernel)
        assert bench.load_traffic(os.path.join(ROOT, "profiles", "traffic.json"), name) == {
            p: v["dram_bytes_per_launch"] for p, v in parts.items()}
    assert {"csa_decode_64k", "hca_decode_1m", "csa_decode_1m"} <= set(rec)
