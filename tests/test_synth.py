"""The seeded input generators: published splitmix64 values, determinism,
counter-based independence, and the workload recipes' shapes and statistics."""
import numpy as np

import synth


def test_splitmix64_published_sequence():
    # first outputs of splitmix64 seeded with 1234567 (reference implementation by S. Vigna)
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert [synth.splitmix64_at(1234567, i) for i in range(5)] == want


def test_counter_based_and_deterministic():
    a = synth.normal_bf16(7, 3, 1000)
    b = synth.normal_bf16(7, 3, 500, first=500)
    assert np.array_equal(a[500:], b)
    assert np.array_equal(a, synth.normal_bf16(7, 3, 1000))
    assert not np.array_equal(a, synth.normal_bf16(8, 3, 1000))


def test_normal_statistics():
    x = synth.bf16_bits_to_f32(synth.normal_bf16(1, 1, 200000)).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_activation_recipe():
    x = synth.activations(1, 256, 3072)
    xf = synth.bf16_bits_to_f32(x)
    mask = synth.outlier_mask(1, synth.S_ACT_PICK, 3072, 31)
    assert mask.sum() == 31
    big = np.abs(xf[:, mask == 1]).mean() / np.abs(xf[:, mask == 0]).mean()
    assert 20 < big < 40  # picked channels are scaled by 30


def test_kv_chunks_continue_the_stream():
    off = synth.kv_offsets(3, 2, 16)
    k0, v0 = synth.kv_chunk(3, 0, 8, 2, 16, off)
    k1, v1 = synth.kv_chunk(3, 1, 8, 2, 16, off)
    assert k0.shape == (8, 2, 16) and not np.array_equal(k0, k1)
    assert not np.array_equal(v0, v1)
