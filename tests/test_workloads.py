"""The seeded input generators: determinism, shapes and value laws."""
import numpy as np

from phase_aware_nvfp4_b200 import workloads as wl


def test_bf16_cast_round_to_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], dtype=np.float32)
    assert wl.f32_to_bf16_bits(v).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000]
    assert np.array_equal(wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(v[[0, 3]])), v[[0, 3]])


def test_generators_are_deterministic_and_chunk_independent():
    a = wl.heavy_tailed_bf16(3000, 64, 5)
    b = wl.heavy_tailed_bf16(3000, 64, 5)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, wl.heavy_tailed_bf16(3000, 64, 6))
    n = wl.normal_bf16(10, 32, 0.02, 1)
    assert n.shape == (10, 32) and n.dtype == np.uint16


def test_heavy_tailed_law_and_outlier_channels():
    x = wl.bf16_bits_to_f32(wl.heavy_tailed_bf16(8192, 400, 3)).astype(np.float64)
    ch = wl.outlier_channels(400, 0.01, 3)
    assert len(ch) == 4
    rest = np.setdiff1d(np.arange(400), ch)
    # Student-t(3): variance 3, heavy tails (kurtosis infinite -> large sample kurtosis)
    v = x[:, rest].var()
    assert 2.0 < v < 4.5
    ratio = np.median(np.abs(x[:, ch])) / np.median(np.abs(x[:, rest]))
    assert 18 < ratio < 22


def test_named_workloads():
    w = wl.qwen3_8b_projections()
    assert [(p.K, p.N) for p in w.projections] == [(4096, 4096), (4096, 1024), (4096, 12288), (12288, 4096)]
    assert abs(w.flops / 1e9 - (274.9 + 68.7 + 824.6 + 824.6)) < 1.0
    assert sum(wl.RAGGED_LENGTHS) == 131072
    x, off = wl.ragged_heavy_tailed_bf16([5, 7], 32, 1)
    assert x.shape == (12, 32) and off.tolist() == [0, 5, 12]
