"""The seeded input generator (CPU only): slices, determinism, rounding, spikes, statistics."""
import numpy as np

import synth


def test_slices_are_independent():
    full = synth.normal_bf16(7, synth.TID_K, 1001)
    part = synth.normal_bf16(7, synth.TID_K, 300, start=501)
    assert np.array_equal(full[501:801], part)
    f = synth.normal_f32(7, synth.TID_K, 1001)
    assert np.array_equal(synth.bf16_bits_from_f32(f), full)


def test_streams_differ():
    a = synth.normal_f32(1, synth.TID_K, 64)
    b = synth.normal_f32(1, synth.TID_V, 64)
    c = synth.normal_f32(2, synth.TID_K, 64)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)


def test_bf16_round_to_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20], dtype=np.float32)
    want = np.array([0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F81], dtype=np.uint16)
    assert np.array_equal(synth.bf16_bits_from_f32(vals), want)


def test_normal_moments():
    x = synth.normal_f32(3, synth.TID_Q, 1 << 20).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3
    assert abs(np.mean(x ** 4) - 3.0) < 0.05  # normal kurtosis


def test_spikes_exact_count_and_factor():
    rows, dim = 5000, 8
    base = synth.normal_bf16(9, synth.TID_K, rows * dim).reshape(rows, dim)
    mat = base.copy()
    chosen = synth.spike_rows_bf16(mat, 9, 3, 5, 4.0)
    assert len(set(chosen.tolist())) == 5
    f = lambda b: (b.astype(np.uint32) << 16).view(np.float32)  # noqa: E731
    for r in range(rows):
        if r in set(chosen.tolist()):
            assert np.array_equal(f(mat[r]), 4.0 * f(base[r]))
        else:
            assert np.array_equal(mat[r], base[r])


def test_config_recipes():
    cfg = synth.decode_configs()
    assert cfg["long_1m"].n_spikes(1_048_576) == 1049
    assert cfg["llama3_8b_gqa"].kv_bytes == 2 * 8 * 32768 * 8 * 128 * 2
    assert cfg["extreme_ragged"].seqlens == [5_120_000, 1_048_576, 262_144, 4096]
    bif = synth.bifurcated_configs()["shared_prefix"]
    assert bif.n_samples == 64 and bif.prefix_len == 65536
