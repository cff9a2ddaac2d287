"""The seeded input generators: deterministic, chunk-independent, and with the
stated distributions (CPU only)."""
import numpy as np

from engram_conditional_memory_hash_b200 import inputs


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-9, -2.0 - 2**-7], dtype=np.float32)
    b = inputs.f32_to_bf16_bits(f)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins;
    # 1 + 3*2^-8 ties between 1+2^-7 and 1+2^-6: even (1+2^-6) wins
    np.testing.assert_array_equal(inputs.bf16_bits_to_f32(b),
                                  np.array([1.0, 1.0, 1.0 + 2**-6, 1.0, -2.0], dtype=np.float32))


def test_normal_deterministic_and_prefix_stable():
    a = inputs.normal_bf16(7, 0, (3 * inputs.CHUNK + 5,))
    b = inputs.normal_bf16(7, 0, (3 * inputs.CHUNK + 5,))
    np.testing.assert_array_equal(a, b)
    c = inputs.normal_bf16(7, 0, (inputs.CHUNK + 3,))
    np.testing.assert_array_equal(a[: inputs.CHUNK + 3], c)
    f = inputs.bf16_bits_to_f32(a).astype(np.float64)
    assert abs(f.mean()) < 2e-3 and abs(f.std() - 1) < 2e-3


def test_weights_near_one():
    w = inputs.gate_inputs(inputs.WORKLOADS["tiny"], T=4)
    wh = inputs.bf16_bits_to_f32(w["wh"]).astype(np.float64)
    assert w["wh"].shape == (256,) and 0.95 < wh.mean() < 1.05 and 0.07 < wh.std() < 0.13


def test_zipf_ids():
    ids = inputs.zipf_ids(3, 6, (200000,), 129280, 1.1)
    assert ids.min() >= 0 and ids.max() < 129280
    counts = np.bincount(ids, minlength=129280)
    # P(rank 1) / P(rank 2) = 2^1.1
    assert abs(counts[0] / counts[1] - 2**1.1) < 0.1
    assert counts[0] > counts[10] > counts[1000]


def test_workload_shapes():
    w = inputs.WORKLOADS["full_path"]
    assert (w.T, w.H, w.D) == (65536, 7168, 64)
    h = inputs.hash_inputs(inputs.WORKLOADS["tiny"])
    assert h["tables"].shape == (int(h["table_sizes"].sum()), 32)
    assert np.all(h["multipliers"] & np.uint64(1) == 1)
    assert h["table_sizes"][0, 0] == 4099 and h["table_sizes"][1, 7] == 4231
    big = inputs.hash_inputs(inputs.WORKLOADS["hash_gather"], with_tables=False)
    assert big["table_sizes"][0, 0] == 1000003 and big["table_sizes"][1, 7] == 1000199
