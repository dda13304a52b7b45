"""Pins for the fp64 oracle: each check ties an oracle function to something
other than itself -- a hand-derived closed form, a textbook/library routine the
definition reduces to, an invariant, or brute force on tiny inputs -- chosen so
that a plausible slip (wrong softmax axis, ape indexed by absolute token, a
dropped ReLU, a scaled sink, an off-by-one window) fails at least one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- compressor

def test_compress_closed_form_two_tokens():
    g = _golden("compress_two_token.json")
    pooled = O.compress(g["kv"], g["gate"], g["ape"], g["norm_w"], g["win"], g["stride"], pre_norm=True)
    out = O.compress(g["kv"], g["gate"], g["ape"], g["norm_w"], g["win"], g["stride"])
    np.testing.assert_allclose(pooled, g["pooled"], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(out, g["out"], rtol=1e-14)


@pytest.mark.parametrize("win,stride", [(8, 4), (128, 128), (5, 3)])
def test_compress_constant_kv_is_preserved_before_norm(win, stride):
    # A convex combination of equal rows returns the row, for any gate / ape.
    T, D = 3 * win + 7, 6
    c = rng.normal(size=D)
    kv = np.tile(c, (T, 1))
    gate = rng.normal(size=(T, D)) * 3
    ape = rng.normal(size=(win, D))
    w = rng.uniform(0.5, 2, size=D)
    pooled = O.compress(kv, gate, ape, w, win, stride, pre_norm=True)
    assert pooled.shape == ((T - win) // stride + 1, D)
    np.testing.assert_allclose(pooled, np.tile(c, (pooled.shape[0], 1)), rtol=1e-12, atol=1e-12)
    out = O.compress(kv, gate, ape, w, win, stride)
    want = c / math.sqrt(np.mean(c * c) + 1e-6) * w
    np.testing.assert_allclose(out, np.tile(want, (out.shape[0], 1)), rtol=1e-12)


def test_compress_window_one_is_torch_rms_norm():
    # win = stride = 1: the pool is the identity, so compress == RMSNorm.
    T, D = 37, 16
    kv = rng.normal(size=(T, D)) * 1e-3  # small enough that eps matters
    gate = rng.normal(size=(T, D))
    ape = rng.normal(size=(1, D))
    w = rng.normal(size=D)
    out = O.compress(kv, gate, ape, w, 1, 1)
    ref = F.rms_norm(torch.tensor(kv), (D,), weight=torch.tensor(w), eps=1e-6).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("win,stride,T", [(8, 4, 64), (8, 4, 67), (128, 128, 1000), (128, 128, 1024)])
def test_compress_uniform_logits_is_average_pooling(win, stride, T):
    # Equal gate + ape over a window: softmax is uniform, pool = window mean.
    D = 5
    kv = rng.normal(size=(T, D))
    gate = np.tile(rng.normal(size=D), (T, 1))
    ape = np.tile(rng.normal(size=D), (win, 1))
    pooled = O.compress(kv, gate, ape, np.ones(D), win, stride, pre_norm=True)
    ref = F.avg_pool1d(torch.tensor(kv.T)[None], kernel_size=win, stride=stride)[0].numpy().T
    assert pooled.shape == ref.shape
    np.testing.assert_allclose(pooled, ref, rtol=1e-12, atol=1e-14)


def test_compress_ape_is_indexed_within_the_window():
    # gate = 0 and ape strongly favouring in-window position 3: entry j pools
    # token 4j + 3 (not a token fixed in absolute position).
    win, stride, T, D = 8, 4, 48, 4
    kv = rng.normal(size=(T, D))
    ape = np.zeros((win, D))
    ape[3] = 60.0
    pooled = O.compress(kv, np.zeros((T, D)), ape, np.ones(D), win, stride, pre_norm=True)
    for j in range(pooled.shape[0]):
        np.testing.assert_allclose(pooled[j], kv[j * stride + 3], rtol=1e-20, atol=1e-20 + 1e-24)


def test_compress_per_window_shift_invariance():
    # Adding a per-dimension constant to every gate in the sequence or to ape
    # leaves the softmax weights, hence the output, unchanged.
    win, stride, T, D = 8, 4, 40, 7
    kv, gate = rng.normal(size=(T, D)), rng.normal(size=(T, D))
    ape = rng.normal(size=(win, D))
    w = np.ones(D)
    a = O.compress(kv, gate, ape, w, win, stride)
    b = O.compress(kv, gate + rng.normal(size=D) * 50, ape + rng.normal(size=D), w, win, stride)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_compress_short_sequence_has_no_entries():
    assert O.compress(np.zeros((7, 3)), np.zeros((7, 3)), np.zeros((8, 3)), np.ones(3), 8, 4).shape == (0, 3)


# ------------------------------------------------------------------ visibility

def test_visibility_matches_windows_produced_by_the_prefix():
    # n_visible(p) == number of entries compress() makes from tokens 0..p.
    D = 1
    for win, stride in ((8, 4), (128, 128)):
        kv = np.zeros((700, D))
        for p in list(range(0, 300)) + [511, 639, 640, 699]:
            rows = O.compress(kv[: p + 1], kv[: p + 1], np.zeros((win, D)), np.ones(D), win, stride).shape[0]
            assert O.n_visible(p, win, stride) == rows, (win, stride, p)


def test_visibility_matches_the_stated_workload_entry_counts():
    # Entry counts stated for the workloads: 65,536 tokens -> 16,383 CSA
    # entries; 1,048,576 -> 262,143 CSA and 8,192 HCA entries; the prefill
    # chunk after 131,072 tokens sees 32,767 .. 33,791 entries.
    assert O.n_visible(65535, 8, 4) == 16383
    assert O.n_visible(1048575, 8, 4) == 262143
    assert O.n_visible(1048575, 128, 128) == 8192
    assert O.n_visible(131072, 8, 4) == 32767
    assert O.n_visible(135167, 8, 4) == 33791
    assert O.n_entries(4100, 8, 4) == 1024
    assert [O.n_visible(p, 8, 4) for p in (0, 6, 7, 10, 11, 14, 15)] == [0, 0, 1, 1, 2, 2, 3]


# --------------------------------------------------------------------- indexer

def test_index_single_head_unit_weight_is_a_plain_dot():
    Di, N = 16, 40
    qi = np.abs(rng.normal(size=(1, Di)))
    ki = np.abs(rng.normal(size=(N, Di)))  # all dots > 0
    s = O.index_scores(qi, [1.0], ki, N)
    np.testing.assert_allclose(s, np.dot(ki, qi[0]), rtol=1e-14)
    # ... and the selection is then an argsort of the dot products.
    np.testing.assert_array_equal(O.topk(s, 7), np.argsort(-np.dot(ki, qi[0]), kind="stable")[:7])


def test_index_negative_dots_contribute_nothing():
    Hi, Di, N = 4, 8, 30
    qi = np.abs(rng.normal(size=(Hi, Di)))
    ki = np.abs(rng.normal(size=(N, Di)))
    s = O.index_scores(-qi, rng.uniform(size=Hi), ki, N)
    assert np.all(s == 0.0)


def test_index_one_hot_weight_selects_relu_of_that_head():
    Hi, Di, N = 4, 8, 50
    qi, ki = rng.normal(size=(Hi, Di)), rng.normal(size=(N, Di))
    for h in range(Hi):
        w = np.zeros(Hi)
        w[h] = 1.0
        np.testing.assert_allclose(O.index_scores(qi, w, ki, N), np.clip(ki @ qi[h], 0, None), rtol=1e-13, atol=1e-15)


def test_index_linear_in_weights_and_homogeneous_in_queries():
    Hi, Di, N = 6, 8, 33
    qi, ki = rng.normal(size=(Hi, Di)), rng.normal(size=(N, Di))
    w1, w2 = rng.uniform(size=Hi), rng.uniform(size=Hi)
    s = lambda q, w: O.index_scores(q, w, ki, N)  # noqa: E731
    np.testing.assert_allclose(s(qi, w1 + w2), s(qi, w1) + s(qi, w2), rtol=1e-13)
    np.testing.assert_allclose(s(2.5 * qi, w1), 2.5 * s(qi, w1), rtol=1e-13)
    # Negating the query is not a sign flip (the ReLU is not odd).
    assert not np.allclose(s(-qi, w1), -s(qi, w1))


def test_index_ignores_entries_past_the_visible_count():
    qi, ki = rng.normal(size=(3, 4)), rng.normal(size=(20, 4))
    w = rng.uniform(size=3)
    a = O.index_scores(qi, w, ki, 9)
    ki2 = ki.copy()
    ki2[9:] = 1e6
    assert a.shape == (9,)
    np.testing.assert_array_equal(a, O.index_scores(qi, w, ki2, 9))


# ----------------------------------------------------------- FP8 indexer (R18)

def test_e4m3_decode_matches_torch_float8_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))  # -0 is 0x80


def test_e4m3_decode_values_from_the_format_definition():
    cases = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 / 8 * 2.0 ** -6, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3F: 1.875,
             0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    got = O.e4m3_decode(list(cases))
    assert np.array_equal(got, np.array(list(cases.values())))
    assert np.isnan(O.e4m3_decode([0x7F, 0xFF])).all()


def test_index_fp8_closed_form_two_entries():
    g = _golden("index_fp8_two_entries.json")
    got = O.index_scores_fp8(np.array(g["qi8"], np.uint8), g["sq"], g["wi"], np.array(g["ki8"], np.uint8),
                             g["sk"], 3)
    assert np.array_equal(got, np.array(g["scores"]))


def test_index_fp8_scales_are_homogeneous():
    Hi, Di, n = 5, 24, 40
    qi8 = rng.integers(0, 0x7F, size=(Hi, Di), dtype=np.uint8) | (rng.integers(0, 2, (Hi, Di)) << 7).astype(np.uint8)
    ki8 = rng.integers(0, 0x7F, size=(n, Di), dtype=np.uint8) | (rng.integers(0, 2, (n, Di)) << 7).astype(np.uint8)
    sq, sk, wi = rng.uniform(0.1, 2, Hi), rng.uniform(0.1, 2, n), rng.uniform(0, 1, Hi)
    base = O.index_scores_fp8(qi8, sq, wi, ki8, sk, n)
    # one positive factor on every key scale scales every score by it
    assert np.allclose(O.index_scores_fp8(qi8, sq, wi, ki8, 3.0 * sk, n), 3.0 * base, rtol=1e-13)
    # per-entry key scales scale each entry's score
    f = rng.uniform(0.5, 4, n)
    assert np.allclose(O.index_scores_fp8(qi8, sq, wi, ki8, f * sk, n), f * base, rtol=1e-13)
    # a query scale folds into the head weight (max(0, a x) = a max(0, x) for a > 0)
    a = rng.uniform(0.5, 4, Hi)
    assert np.allclose(O.index_scores_fp8(qi8, a * sq, wi, ki8, sk, n), O.index_scores_fp8(qi8, sq, a * wi, ki8, sk, n),
                       rtol=1e-13)


def test_index_fp8_unit_scales_single_head_is_a_plain_dot_of_decoded_codes():
    # Hi = 1, w = 1, unit scales, codes of positive values only: s_j = qi . ki_j
    # with qi, ki the values the codes stand for (torch's float8 conversion).
    Di, n = 16, 12
    qi8 = rng.integers(0x08, 0x7E, size=(1, Di), dtype=np.uint8)
    ki8 = rng.integers(0x08, 0x7E, size=(n, Di), dtype=np.uint8)
    tq = torch.from_numpy(qi8).view(torch.float8_e4m3fn).to(torch.float64)
    tk = torch.from_numpy(ki8).view(torch.float8_e4m3fn).to(torch.float64)
    got = O.index_scores_fp8(qi8, [1.0], [1.0], ki8, np.ones(n), n)
    assert np.allclose(got, (tk @ tq[0]).numpy(), rtol=1e-15)


# ------------------------------------------- indexer compressor and FP8 codes (R19)

def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    assert np.array_equal(O.e4m3_encode(vals), codes)
    assert np.array_equal(O.e4m3_encode(-vals), codes | 0x80)


def test_e4m3_encode_matches_torch_float8_on_fp32_values_in_range():
    # torch's cast rounds to nearest, ties to even, on fp32 inputs
    x = np.linspace(-448, 448, 400001).astype(np.float32)
    x = np.concatenate([x, (rng.standard_normal(100000) * 30).astype(np.float32).clip(-448, 448)])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x.astype(np.float64)), ref)


def test_e4m3_encode_ties_saturation_and_underflow():
    # 84 lies halfway between 80 (mantissa 010) and 88 (011): the even one
    assert O.e4m3_decode(O.e4m3_encode([84.0, -84.0])).tolist() == [80.0, -80.0]
    # 1.0625 halfway between 1 (000) and 1.125 (001); 1.1875 between 1.125 and 1.25 (010)
    assert O.e4m3_decode(O.e4m3_encode([1.0625, 1.1875])).tolist() == [1.0, 1.25]
    assert O.e4m3_encode([448.0, 460.0, 1e6, -1e6]).tolist() == [0x7E, 0x7E, 0x7E, 0xFE]
    # half the smallest subnormal (2^-10) ties to 0 (even); just above it goes to 2^-9
    assert O.e4m3_encode([2.0 ** -10, 2.0 ** -10 * 1.01, -1e-30]).tolist() == [0x00, 0x01, 0x80]


def test_quantize_rows_maps_the_row_maximum_to_448_and_bounds_the_error():
    x = rng.standard_normal((20, 128)) * rng.uniform(0.01, 100, (20, 1))
    x[3] = 0.0
    codes, scales = O.quantize_rows_e4m3(x)
    assert scales.dtype == np.float32 and scales[3] == 1.0 and (codes[3] & 0x7F == 0).all()
    deq = O.e4m3_decode(codes) * scales[:, None].astype(np.float64)
    for r in range(20):
        if r == 3:
            continue
        j = np.argmax(np.abs(x[r]))
        assert codes[r, j] & 0x7F == 0x7E                     # the largest magnitude becomes +-448
        # nearest-value rounding: error at most half the E4M3 spacing at that magnitude (<= 2^-4 relative),
        # or half the smallest subnormal step
        err = np.abs(deq[r] - x[r])
        assert np.all(err <= np.maximum(np.abs(x[r]) * 2.0 ** -4, 2.0 ** -10 * scales[r]) * 1.0001)


def test_quantize_rows_scale_reproduces_the_row_maximum():
    # Reading R19: the scale maps each row's largest magnitude onto the largest
    # finite E4M3 value (448, S.1111.110), so decoding that code and
    # multiplying by the scale gives the row maximum back, up to fp32
    # rounding. A scale with another denominator (amax / 440, amax / 512)
    # misses it by 2 % or more.
    x = rng.standard_normal((64, 128)) * rng.uniform(1e-3, 1e3, (64, 1))
    codes, scales = O.quantize_rows_e4m3(x)
    amax = np.abs(x.astype(np.float32)).max(axis=1).astype(np.float64)
    top = O.e4m3_decode(np.array([0x7E], dtype=np.uint8))[0]
    assert top == 448.0
    assert np.all(np.abs(top * scales.astype(np.float64) - amax) <= amax * 2.0 ** -22)


def test_quantize_rows_hand_example():
    # Row (3.5, -7, 1, 0): amax 7, scale 7 / 448 = 2^-6 exactly; the scaled
    # values 224, -448, 64, 0 are all E4M3 values:
    #   224 = 1.75 * 2^7 -> exponent field 7 + 7 = 14, mantissa .110 -> 0 1110 110 = 0x76
    #  -448 = -1.75 * 2^8 -> 1 1111 110 = 0xFE;   64 = 2^6 -> 0 1101 000 = 0x68;   0 -> 0x00
    codes, scales = O.quantize_rows_e4m3(np.array([[3.5, -7.0, 1.0, 0.0]]))
    assert scales[0] == np.float32(2.0 ** -6)
    assert codes[0].tolist() == [0x76, 0xFE, 0x68, 0x00]


def test_hadamard_is_sylvester_and_orthonormal():
    import scipy.linalg
    for n in (1, 2, 16, 128):
        assert np.array_equal(O.hadamard_matrix(n), scipy.linalg.hadamard(n))
    h = O.hadamard_matrix(128)
    assert np.array_equal(h @ h.T, 128 * np.eye(128))
    x = rng.standard_normal((7, 128))
    y = O.hadamard_rotate(x)
    assert np.allclose(O.hadamard_rotate(y), x, atol=1e-12)                 # H / sqrt(n) is its own inverse
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1))
    e0 = np.zeros((1, 128))
    e0[0, 0] = 1
    assert np.allclose(O.hadamard_rotate(e0), np.full((1, 128), 1 / np.sqrt(128)))


def test_rotation_leaves_indexer_scores_unchanged():
    Hi, n = 4, 30
    qi, ki, wi = rng.standard_normal((Hi, 128)), rng.standard_normal((n, 128)), rng.uniform(0, 1, Hi)
    assert np.allclose(O.index_scores(O.hadamard_rotate(qi), wi, O.hadamard_rotate(ki), n),
                       O.index_scores(qi, wi, ki, n), rtol=1e-12, atol=1e-12)


def test_index_compress_is_the_rotated_pool():
    # constant raw KV rows: the pool returns the row before the norm, so each
    # entry is the rotation of norm(c) -- an explicit closed form through H
    T, D = 20, 128
    c = rng.standard_normal(D)
    kv = np.tile(c, (T, 1))
    gate, ape = rng.standard_normal((T, D)), rng.standard_normal((8, D)) * 0.1
    out = O.index_compress(kv, gate, ape, np.ones(D), 8, 4)
    want = (c / np.sqrt(np.mean(c * c) + 1e-6)) @ scipy_hadamard(D) / np.sqrt(D)
    assert out.shape == (O.n_entries(T, 8, 4), D)
    assert np.allclose(out, np.tile(want, (out.shape[0], 1)), rtol=1e-12, atol=1e-12)


def scipy_hadamard(n):
    import scipy.linalg
    return scipy.linalg.hadamard(n).astype(np.float64)


# ------------------------------------------------------- RoPE on compressed entries (R20)

def test_rope_closed_form_one_pair():
    # rope_dims 2: the single pair rotates by the angle p * theta^0 = p
    x = np.array([[0.0, 0.0, 3.0, 4.0]])
    for p in (0.0, 1.0, 2.5):
        y = O.rope_last_dims(x, [p], 160000.0, rope_dims=2)
        assert np.allclose(y[0], [0.0, 0.0, 3 * math.cos(p) - 4 * math.sin(p), 3 * math.sin(p) + 4 * math.cos(p)],
                           rtol=0, atol=1e-15)


def test_rope_frequencies_follow_theta():
    # pair i of 64 rope dims turns by p * theta^(-i/32): a unit vector on pair i
    # ends at angle p * theta^(-i/32) (complex multiplication by e^{i angle})
    theta, p = 160000.0, 37.0
    for i in (0, 1, 17, 31):
        x = np.zeros((1, 512))
        x[0, 448 + 2 * i] = 1.0
        y = O.rope_last_dims(x, [p], theta)
        z = complex(y[0, 448 + 2 * i], y[0, 449 + 2 * i])
        ang = p * theta ** (-i / 32)
        assert abs(z - complex(math.cos(ang), math.sin(ang))) < 1e-12


def test_rope_dot_products_depend_only_on_the_offset():
    q, k = rng.standard_normal((1, 512)), rng.standard_normal((1, 512))
    dots = [float((O.rope_last_dims(q, [p + 100.0], 160000.0) @ O.rope_last_dims(k, [p], 160000.0).T)[0, 0])
            for p in (0.0, 1000.0, 123456.0)]
    assert np.allclose(dots, dots[0], rtol=1e-9)
    assert np.allclose(np.linalg.norm(O.rope_last_dims(q, [5e5], 160000.0)), np.linalg.norm(q))


def test_compress_rope_positions_are_the_last_tokens():
    T, D = 40, 128
    kv, gate = rng.standard_normal((T, D)), rng.standard_normal((T, D))
    ape = rng.standard_normal((8, D)) * 0.1
    base = O.compress(kv, gate, ape, np.ones(D), 8, 4)
    got = O.compress_rope(kv, gate, ape, np.ones(D), 8, 4, pos0=1000, theta=160000.0)
    assert np.array_equal(got[:, :64], base[:, :64])
    want = O.rope_last_dims(base, 1000 + 4 * np.arange(base.shape[0]) + 7, 160000.0)
    assert np.allclose(got, want, rtol=0, atol=1e-15)


def test_topk_closed_form_ties():
    g = _golden("topk_ties.json")
    for case in g["cases"]:
        np.testing.assert_array_equal(O.topk(g["scores"], case["k"]), case["idx"])


@pytest.mark.parametrize("n,k", [(6, 3), (8, 4), (9, 2), (10, 5), (7, 7)])
def test_topk_brute_force_subsets(n, k):
    # Among all k-subsets: maximal score sum, then the lexicographically
    # smallest sorted index tuple (== ties go to smaller indices).
    for trial in range(20):
        s = rng.integers(0, 4, size=n).astype(float)  # many ties
        best = None
        for sub in itertools.combinations(range(n), k):
            key = (-sum(s[list(sub)]), sub)
            if best is None or key < best:
                best = key
        got = O.topk(s, k)
        assert sorted(got.tolist()) == list(best[1])
        # best-first order
        assert all(s[got[i]] >= s[got[i + 1]] for i in range(k - 1))


def test_topk_short_list_is_padded():
    s = rng.normal(size=5)
    got = O.topk(s, 8)
    assert sorted(got[:5].tolist()) == list(range(5)) and list(got[5:]) == [-1, -1, -1]
    assert list(O.topk(np.zeros(0), 3)) == [-1, -1, -1]


# --------------------------------------------------------------------- attention

def test_attend_closed_form_with_sink():
    g = _golden("attend_two_row_sink.json")
    out, p, ps = O.attend(g["q"], g["rows"], g["sink"], g["scale"])
    np.testing.assert_allclose(out, g["out"], rtol=1e-14)
    np.testing.assert_allclose(p, g["p"], rtol=1e-14)
    np.testing.assert_allclose(ps, g["p_sink"], rtol=1e-14)


def _sdpa_with_sink(q, rows, sink, scale):
    """torch scaled_dot_product_attention (fp64) with the sink as an extra key
    of value zero whose logit is set through an additive per-head bias."""
    H, D = q.shape
    R = rows.shape[0]
    K = np.concatenate([rows, np.zeros((1, D))], 0)
    bias = np.zeros((H, 1, R + 1))
    bias[:, 0, R] = sink
    qt = torch.tensor(q)[:, None, :]                       # [H, 1, D]
    kt = torch.tensor(K)[None].expand(H, R + 1, D)          # shared K = V
    return F.scaled_dot_product_attention(qt, kt, kt, attn_mask=torch.tensor(bias), scale=scale)[:, 0].numpy()


@pytest.mark.parametrize("H,D,R", [(4, 16, 1), (4, 16, 37), (8, 64, 200)])
def test_attend_matches_torch_sdpa(H, D, R):
    q, rows = rng.normal(size=(H, D)), rng.normal(size=(R, D))
    sink = rng.normal(size=H) * 2
    scale = 1 / math.sqrt(D)
    out, p, ps = O.attend(q, rows, sink, scale)
    np.testing.assert_allclose(out, _sdpa_with_sink(q, rows, sink, scale), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(p.sum(1) + ps, 1.0, rtol=1e-14)


def test_attend_zero_scale_closed_form():
    # scale 0: every row has logit 0, so out = sum(rows) / (R + exp(sink)).
    H, D, R = 3, 5, 11
    rows = rng.normal(size=(R, D))
    sink = np.array([-1.0, 0.0, 2.0])
    out, _, _ = O.attend(rng.normal(size=(H, D)), rows, sink, 0.0)
    want = rows.sum(0)[None, :] / (R + np.exp(sink))[:, None]
    np.testing.assert_allclose(out, want, rtol=1e-13)


def test_attend_sink_limits():
    q, rows = rng.normal(size=(2, 4)), rng.normal(size=(1, 4))
    out, _, _ = O.attend(q, rows, np.full(2, -np.inf), 0.7)
    np.testing.assert_allclose(out, np.tile(rows, (2, 1)), rtol=1e-15)  # one row, no sink: out = row
    out, _, ps = O.attend(q, rows, np.full(2, 800.0), 0.7)
    assert np.all(np.abs(out) < 1e-300) and np.all(ps == 1.0)
    out, _, _ = O.attend(q, np.zeros((0, 4)), np.zeros(2), 0.7)
    assert np.all(out == 0.0)


def test_window_rows_clip_at_sequence_start():
    kv = rng.normal(size=(200, 3))
    assert O.window_rows(kv, 3, 16).shape == (4, 3)
    np.testing.assert_array_equal(O.window_rows(kv, 100, 16), kv[85:101])


def test_sparse_mqa_without_entries_and_sink_is_sliding_window_attention():
    # Sink at -inf and no compressed entries: plain causal sliding-window
    # softmax attention, as torch SDPA with a banded causal mask.
    T, H, D, W = 70, 4, 16, 16
    kv, q = rng.normal(size=(T, D)), rng.normal(size=(T, H, D))
    scale = 0.25
    band = np.full((T, T), -np.inf)
    for p in range(T):
        band[p, max(0, p - W + 1): p + 1] = 0.0
    qt = torch.tensor(q).permute(1, 0, 2)                   # [H, T, D]
    kt = torch.tensor(kv)[None].expand(H, T, D)
    ref = F.scaled_dot_product_attention(qt, kt, kt, attn_mask=torch.tensor(band), scale=scale)
    ref = ref.permute(1, 0, 2).numpy()
    idx = np.full(4, -1)
    for p in range(T):
        got = O.sparse_mqa(q[p], np.zeros((3, D)), idx, kv, p, W, np.full(H, -np.inf), scale)
        np.testing.assert_allclose(got, ref[p], rtol=1e-12, atol=1e-13)


def test_sparse_with_topk_covering_all_entries_equals_dense_hca():
    N, H, D, Hi, Di, W = 25, 4, 16, 4, 8, 16
    kv_cmp, kv_win = rng.normal(size=(N, D)), rng.normal(size=(300, D))
    qi, ki, w = rng.normal(size=(Hi, Di)), rng.normal(size=(N, Di)), rng.uniform(size=Hi)
    q, sink = rng.normal(size=(H, D)), rng.normal(size=H)
    p = 4 * (N - 1) + 7 + 2  # every entry visible
    idx, _ = O.index_topk(qi, w, ki, p, 32, 8, 4)
    a = O.sparse_mqa(q, kv_cmp, idx, kv_win, 250, W, sink, 0.25)
    b = O.hca_mqa(q, kv_cmp, N, kv_win, 250, W, sink, 0.25)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_sparse_mqa_is_order_free_and_skips_padding():
    N, H, D = 40, 4, 16
    kv_cmp, kv_win = rng.normal(size=(N, D)), rng.normal(size=(50, D))
    q, sink = rng.normal(size=(H, D)), rng.normal(size=H)
    idx = rng.permutation(N)[:12]
    a = O.sparse_mqa(q, kv_cmp, idx, kv_win, 20, 16, sink, 0.3)
    b = O.sparse_mqa(q, kv_cmp, np.concatenate([[-1], idx[::-1], [-1, -1]]), kv_win, 20, 16, sink, 0.3)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_attend_split_rows_merge_by_log_sum_exp():
    # Splitting the row set in two and merging the partial (max, sum, out)
    # by log-sum-exp reproduces the whole: the basis of a split-K combine.
    H, D, R = 4, 8, 30
    q, rows, sink = rng.normal(size=(H, D)), rng.normal(size=(R, D)), rng.normal(size=H)
    full, _, _ = O.attend(q, rows, sink, 0.4)
    parts = []
    for part in (rows[:13], rows[13:]):
        lg = 0.4 * q @ part.T
        m = lg.max(1)
        e = np.exp(lg - m[:, None])
        parts.append((m, e.sum(1), e @ part))
    M = np.maximum(np.maximum(parts[0][0], parts[1][0]), sink)
    Z = sum(l * np.exp(m - M) for m, l, _ in parts) + np.exp(sink - M)
    merged = sum(o * np.exp(m - M)[:, None] for m, _, o in parts) / Z[:, None]
    np.testing.assert_allclose(full, merged, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------- rounding

def test_round_to_bf16_matches_torch_on_fp32_values():
    x32 = (rng.normal(size=20000) * np.exp(rng.uniform(-20, 20, size=20000))).astype(np.float32)
    ref = torch.tensor(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_to(x32.astype(np.float64), "bf16"), ref)
