"""The seeded generator: a counter-based stream, identical bytes for a slice
and for the whole tensor, and the published SplitMix64 finaliser."""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_15_b200 import synth

M64 = (1 << 64) - 1


def _py_hash(seed, tid, c):
    key = synth.stream_key(seed, tid)
    return synth.mix_int((key + (c + 1) * synth.GAMMA) & M64)


def test_splitmix_finaliser_known_values():
    # SplitMix64 with state 0 stepped once by GAMMA: the published first
    # outputs of the generator seeded with 0.
    outs, state = [], 0
    for _ in range(3):
        state = (state + synth.GAMMA) & M64
        outs.append(synth.mix_int(state))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_torch_hash_matches_python_reference():
    c = torch.tensor([0, 1, 2, 12345, (1 << 40) + 7], dtype=torch.int64)
    got = synth._hash(7, 3, c)
    for i, ci in enumerate(c.tolist()):
        assert (int(got[i]) & M64) == _py_hash(7, 3, ci)


def test_uniform_and_normal_values_from_reference():
    idx = torch.tensor([0, 5, 999], dtype=torch.int64)
    u = synth.uniform_at(11, 2, idx)
    n = synth.normal_at(11, 2, idx)
    for i, ci in enumerate(idx.tolist()):
        assert float(u[i]) == (_py_hash(11, 2, ci) >> 40) * 2.0 ** -24
        acc = 0
        for m in range(6):
            h = _py_hash(11, 2, 6 * ci + m)
            acc += (h >> 40) + ((h >> 8) & 0xFFFFFF)
        assert float(n[i]) == float(np.float32(acc * 2.0 ** -24 - 6.0))


def test_slices_equal_whole_tensor():
    full = synth.normal(3, 9, (40, 24), dtype=torch.bfloat16)
    rows = [0, 7, 39, 8]
    np.testing.assert_array_equal(
        synth.normal_rows(3, 9, (40, 24), rows, dtype=torch.bfloat16).float().numpy(),
        full[rows].float().numpy())


def test_moments_and_bounds():
    x = synth.normal(0, 1, (1 << 18,))
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1) < 0.01
    assert float(x.abs().max()) <= 6.0
    u = synth.uniform(0, 5, (1 << 16,))
    assert 0.0 <= float(u.min()) and float(u.max()) < 1.0 and abs(float(u.mean()) - 0.5) < 0.01
    s = synth.normal(0, 1, (1 << 16,), std=0.1)
    assert abs(float(s.std()) - 0.1) < 0.002


def test_streams_differ_by_seed_and_tensor():
    a = synth.normal(0, 1, (1000,))
    assert not torch.equal(a, synth.normal(1, 1, (1000,)))
    assert not torch.equal(a, synth.normal(0, 2, (1000,)))
    assert torch.equal(a, synth.normal(0, 1, (1000,)))


@pytest.mark.gpu
def test_device_bytes_equal_host_bytes(cuda_device):
    for dt in (torch.float32, torch.bfloat16):
        h = synth.normal(5, 4, (3, 1000, 17), dtype=dt)
        d = synth.normal(5, 4, (3, 1000, 17), dtype=dt, device=cuda_device).cpu()
        assert torch.equal(h.view(torch.int16 if dt == torch.bfloat16 else torch.int32),
                           d.view(torch.int16 if dt == torch.bfloat16 else torch.int32))
    assert torch.equal(synth.uniform(5, 4, (999,)), synth.uniform(5, 4, (999,), device=cuda_device).cpu())


def test_fp8_code_draws_stay_inside_the_e4m3_range():
    import numpy as np

    import oracle as O
    from compressed_sparse_attention_15_b200 import workloads as WL
    w = WL.small(WL.WORKLOADS["csa_decode_64k"], Q=2, B=2, N=4096)
    for name in ("qi8", "ki8"):
        v = O.e4m3_decode(WL.make(w, name).numpy())
        assert np.isfinite(v).all() and np.abs(v).max() <= 448
    for name in ("sq", "sk"):
        s = WL.make(w, name)
        assert (s > 0).all()
