"""The seeded input generator (package ``synth``) against its published definition.

The generator is input plumbing shared by both sides, so it is pinned here
against an independent pure-Python restatement of its definition and against
the published SplitMix64 reference stream. The host==device check is a GPU test
(tests/test_gpu_parity.py).
"""
import os

import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splitmix64_state0.txt")
M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def py_mix64(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def py_value_bits(seed, tid, i, sigma, mean):
    key = py_mix64(py_mix64(seed) ^ tid)
    s = 0
    for j in range(3):
        w = py_mix64((key + (3 * i + j + 1) * GAMMA) & M64)
        s += sum((w >> (16 * q)) & 0xFFFF for q in range(4))
    z = np.float32(s - 393210) * np.float32(1.0 / 65536.0)
    v = np.float32(np.float32(mean) + np.float32(np.float32(sigma) * z))
    return int(synth.f32_to_bf16_bits(np.array([v]))[0])


def test_splitmix64_reference_stream():
    want = [int(line, 16) for line in open(GOLDEN) if line.startswith("0x")]
    got = [synth.mix64(((c + 1) * GAMMA) & M64) for c in range(len(want))]
    assert got == want
    # the stream of a key is the SplitMix64 stream whose state is that key
    words = synth.words_host(0, 0, 0, 3)
    key = py_mix64(py_mix64(0) ^ 0)
    assert [int(w) for w in words] == [py_mix64((key + (c + 1) * GAMMA) & M64) for c in range(3)]


@pytest.mark.parametrize("kind", [synth.KIND_GAMMA, synth.KIND_W_GATE, synth.KIND_W_DOWN,
                                  synth.KIND_X])
def test_host_fill_matches_python_definition(kind):
    rng = np.random.default_rng(kind)
    seed, tid = 1 + kind, synth.tensor_id(1, kind)
    sigma, mean = (np.float32(0.1), 1.0) if kind == synth.KIND_GAMMA else (synth.sigma_for(7168), 0.0)
    start = int(rng.integers(0, 1 << 33))
    got = synth.fill_host(seed, tid, start, 64, sigma, mean)
    want = [py_value_bits(seed, tid, start + i, sigma, mean) for i in range(64)]
    assert got.tolist() == want


def test_normal_moments_and_range():
    z = synth.z_host(5, synth.tensor_id(0, synth.KIND_X), 0, 1 << 20)
    assert abs(float(z.mean())) < 5e-3
    assert abs(float(z.std()) - 1.0) < 5e-3
    assert np.all(np.abs(z) <= 6.0) and np.all(np.isfinite(z))
    w = synth.bf16_bits_to_f32(synth.fill_host(5, synth.tensor_id(0, synth.KIND_W_UP), 0, 1 << 20,
                                                synth.sigma_for(7168)))
    assert abs(float(w.std()) * np.sqrt(7168) - 1.0) < 1e-2


def test_different_tensors_and_seeds_differ():
    a = synth.fill_host(1, synth.tensor_id(0, synth.KIND_W_GATE), 0, 256, 1.0)
    b = synth.fill_host(1, synth.tensor_id(0, synth.KIND_W_UP), 0, 256, 1.0)
    c = synth.fill_host(2, synth.tensor_id(0, synth.KIND_W_GATE), 0, 256, 1.0)
    d = synth.fill_host(1, synth.tensor_id(1, synth.KIND_W_GATE), 0, 256, 1.0)
    assert not np.array_equal(a, b) and not np.array_equal(a, c) and not np.array_equal(a, d)


def test_expert_slices_are_views_of_one_tensor():
    wl = synth.WORKLOADS[0]
    g3, _, d3 = wl.expert_host(0, 3)
    n = wl.I * wl.H
    whole = synth.fill_host(wl.seed, synth.tensor_id(0, synth.KIND_W_GATE), 0, 4 * n, synth.sigma_for(wl.H))
    assert np.array_equal(g3.ravel(), whole[3 * n:4 * n])


def test_router_bias_is_zipf_over_a_permutation():
    E = 896
    b = synth.router_bias(3, 0, E).astype(np.float64)
    want = np.sort(-2.2 * np.log(np.arange(1, E + 1)))
    np.testing.assert_allclose(np.sort(b), want.astype(np.float32), rtol=0, atol=0)
    b2 = synth.router_bias(4, 0, E)
    assert not np.array_equal(b, b2)


def test_correlated_rows_follow_their_sequence():
    x = synth.bf16_bits_to_f32(synth.rows_correlated(4, 0, 4, 8, 512))
    # rows of one sequence differ by 0.1 * noise; rows of different sequences by ~sqrt(2)
    within = np.std(x[0] - x[1])
    across = np.std(x[0] - x[8])
    assert 0.1 < within < 0.2 and 1.2 < across < 1.7


def test_workload_table():
    w = synth.WORKLOADS
    assert (w[1].B, w[1].H, w[1].E, w[1].k, w[1].I, w[1].Is) == (1, 7168, 896, 16, 1024, 2048)
    assert w[2].B == 8 and w[3].B == 64 and w[3].router == "zipf"
    assert w[4].B == 32 and w[4].layers == 2 and w[4].nseq * w[4].rows_per_seq == 32
    assert abs(w[1].weight_bytes_per_layer() / 1e9 - 39.56) < 0.05


def test_e4m3_encoder_is_nearest_ties_to_even_as_an_independent_conversion():
    """The generator's FP8 encoder against torch's float8_e4m3fn conversion on values
    inside the finite range (the generator clamps to +-448 first), ties included."""
    import torch

    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(50000) * 100, rng.standard_normal(50000) * 0.01,
                        np.array([0.0, -0.0, 448.0, -448.0, 2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875])])
    v = np.clip(v, -448, 448).astype(np.float32)
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(synth.e4m3_encode_host(v), want)
    # out-of-range values clamp to the largest finite code instead of NaN
    assert list(synth.e4m3_encode_host(np.array([500.0, -1e30], dtype=np.float32))) == [0x7E, 0xFE]


def test_fp8_block_scales_are_powers_of_two_around_the_weight_spread():
    wl = synth.WORKLOADS[1]
    s = wl.fp8_scales_host(0, "gate", [0, 1])
    e = np.log2(s)
    assert np.array_equal(e, np.round(e)) and s.shape == (2, wl.I // 128, wl.H // 128)
    s0 = synth.fp8_s0(wl.H)
    assert set(np.unique(e).astype(int)) <= {s0 - 1, s0, s0 + 1}
    assert len(np.unique(e)) == 3


def test_fp8_cover_codes_give_every_block_one_binade_and_every_code_full_weight():
    """Coverage codes: within a 128 x 128 block every code has the exponent field
    (b + phase) mod 16, all 16 fields appear across the blocks, no NaN code is drawn, and
    with the block scales every nonzero weight lies in [2^(t-3), 2^(t+1)) -- subnormal
    blocks included -- so a wrong decode of any code changes the layer visibly."""
    import torch

    wl = synth.Workload("cover", B=1, H=512, E=4, k=2, I=256, Is=128, seed=7, experts="fp8_cover")
    assert wl.is_fp8
    t = synth.cover_t(wl.H)
    fields = set()
    for e in range(wl.E):
        codes, scales = wl.expert_fp8_host(0, e)["gate"]
        rb, cb = wl.I // 128, wl.H // 128
        assert codes.shape == (wl.I, wl.H) and scales.shape == (rb, cb)
        assert not np.any((codes & 0x7F) == 0x7F)
        for r in range(rb):
            for c in range(cb):
                blk = codes[128 * r:128 * r + 128, 128 * c:128 * c + 128]
                f = (blk >> 3) & 15
                b = (e * rb + r) * cb + c
                want = (b + synth.cover_phase(wl.seed)) % 16
                assert np.all(f == want)
                fields.add(int(want))
                assert scales[r, c] == np.float32(2.0 ** (t + 7 - max(want, 1)))
                # all mantissas (field 15: 0..6, mantissa 7 there being NaN) and both signs
                assert len(np.unique(blk & 7)) == (7 if want == 15 else 8) and len(np.unique(blk >> 7)) == 2
        w = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
        w = w * np.kron(scales, np.ones((128, 128), dtype=np.float32))
        a = np.abs(w[w != 0])
        assert a.min() >= 2.0 ** (t - 3) and a.max() < 2.0 ** (t + 1)
    assert fields == set(range(16))
