"""Writes the hand-derived closed-form fixtures in this folder.

The pages print no worked example with numbers for any step of the path, so
these fixtures are the smallest cases whose results can be derived by hand
from the prose definitions; each carries its derivation and citation. The
script evaluates those closed forms with the math module only (it runs
neither the oracle nor the CUDA path). Run: python tests/golden/make_closed_forms.py
"""
import json
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
e = math.e

compress = {
    "citation": "DeepSeek-V4 Architecture Analysis, INNOVATIONS section 1 (gated pooling with "
                "in-window position embeddings, RMSNorm on the compressed output); DeepSeek-V4-Flash "
                "model card, config.json rms_norm_eps = 1e-6",
    "derivation": "One window of 2 tokens (win = stride = 2), D = 2, ape = 0. Dim 0: gate (0, ln 3) -> "
                  "softmax weights (1/4, 3/4); kv (1, 3) -> c0 = 1/4 + 9/4 = 5/2. Dim 1: gate (0, 0) -> "
                  "weights (1/2, 1/2); kv (2, -1) -> c1 = 1/2. mean(c^2) = (25/4 + 1/4)/2 = 13/4. "
                  "out = c / sqrt(13/4 + 1e-6) * norm_w with norm_w = (1, 2).",
    "win": 2, "stride": 2,
    "kv": [[1.0, 2.0], [3.0, -1.0]],
    "gate": [[0.0, 0.0], [math.log(3.0), 0.0]],
    "ape": [[0.0, 0.0], [0.0, 0.0]],
    "norm_w": [1.0, 2.0],
    "pooled": [[2.5, 0.5]],
    "out": [[2.5 / math.sqrt(3.25 + 1e-6), 2 * 0.5 / math.sqrt(3.25 + 1e-6)]],
}

attend = {
    "citation": "DeepSeek-V4 Architecture Analysis, INNOVATIONS section 1 (attention sink: a per-head "
                "scalar) and section 2 (keys and values share one representation)",
    "derivation": "H = 1, D = 2, q = (1, 0), rows (1, 0) and (0, 1), scale 1, sink 0. Logits 1 and 0, "
                  "sink 0: Z = e + 1 + 1. p = (e/(e+2), 1/(e+2)), p_sink = 1/(e+2). "
                  "out = p0 * (1, 0) + p1 * (0, 1) = (e/(e+2), 1/(e+2)).",
    "q": [[1.0, 0.0]], "rows": [[1.0, 0.0], [0.0, 1.0]], "sink": [0.0], "scale": 1.0,
    "p": [[e / (e + 2), 1 / (e + 2)]], "p_sink": [1 / (e + 2)],
    "out": [[e / (e + 2), 1 / (e + 2)]],
}

topk = {
    "citation": "DeepSeek-V4 Architecture Analysis, INNOVATIONS section 1 (indexer selects the top-k "
                "compressed positions); DeepSeek-V4-Flash model card, config.json index_topk",
    "derivation": "Scores (3, 5, 5, 1, 5, 0), k = 3: the three 5s (indices 1, 2, 4) are kept, best first, "
                  "ties by index ascending. k = 2 keeps 1 and 2 (the tie at 5 goes to the smaller "
                  "indices). k = 8 keeps all six, ordered 1, 2, 4, 0, 3, 5, then -1, -1.",
    "scores": [3.0, 5.0, 5.0, 1.0, 5.0, 0.0],
    "cases": [{"k": 3, "idx": [1, 2, 4]}, {"k": 2, "idx": [1, 2]},
              {"k": 8, "idx": [1, 2, 4, 0, 3, 5, -1, -1]}],
}

index_fp8 = {
    "citation": "deepseek-ai/DeepSeek-V4-Flash-0731, table 'Config changes': quantization_config fmt e4m3, "
                "quant_method fp8; DeepSeek-V4 Architecture Analysis, INNOVATIONS section 1 (indexer: "
                "dot products with per-head importance weights, trained with QAT); OCP FP8 E4M3 format "
                "(sign, 4-bit exponent with bias 7, 3-bit mantissa)",
    "derivation": "Codes: 0x38 = 2^(7-7) = 1, 0x40 = 2^(8-7) = 2, 0xB8 = -1. Queries (Hi = 2, Di = 2): "
                  "head 0 codes (0x38, 0x40) scale 2 -> (2, 4); head 1 codes (0x40, 0xB8) scale 1/2 -> "
                  "(1, -1/2). Keys: entry 0 codes (0x38, 0x38) scale 1/2 -> (1/2, 1/2); entry 1 codes "
                  "(0x40, 0x38) scale 1 -> (2, 1); entry 2 codes (0xB8, 0xB8) scale 1 -> (-1, -1). "
                  "Dots: entry 0: head 0 1 + 2 = 3, head 1 1/2 - 1/4 = 1/4; entry 1: head 0 4 + 4 = 8, "
                  "head 1 2 - 1/2 = 3/2; entry 2: head 0 -6, head 1 -1/2 (both ReLU 0). Weights (1, 1/4): "
                  "s = (3 + 1/16, 8 + 3/8, 0).",
    "qi8": [[0x38, 0x40], [0x40, 0xB8]], "sq": [2.0, 0.5], "wi": [1.0, 0.25],
    "ki8": [[0x38, 0x38], [0x40, 0x38], [0xB8, 0xB8]], "sk": [0.5, 1.0, 1.0],
    "scores": [3.0625, 8.375, 0.0],
}

for name, obj in (("compress_two_token.json", compress), ("attend_two_row_sink.json", attend),
                  ("index_fp8_two_entries.json", index_fp8),
                  ("topk_ties.json", topk)):
    with open(os.path.join(HERE, name), "w") as f:
        json.dump(obj, f, indent=1)
        f.write("\n")
