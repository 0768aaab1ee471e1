"""The seeded input generator (host twin): reference outputs, slicing, moments."""
import numpy as np

import oracle_pins as P
import synth
from synth import workloads as W


def test_splitmix64_reference_outputs():
    g = P.golden("splitmix64_reference.json")
    got = synth.splitmix64_sequence(g["seed"], len(g["outputs"]))
    assert [int(v) for v in got] == [int(s) for s in g["outputs"]]


def test_slices_are_consistent_and_deterministic():
    k = synth.key(0, 7)
    a = synth.normal_bf16(k, 0, 100000, 0.02)
    assert np.array_equal(a[31337:31400], synth.normal_bf16(k, 31337, 63, 0.02))
    assert np.array_equal(a, synth.normal_bf16(k, 0, 100000, 0.02))
    assert not np.array_equal(a, synth.normal_bf16(synth.key(0, 8), 0, 100000, 0.02))


def test_irwin_hall_moments_and_support():
    z = synth.normal_f32(synth.key(0, 1), 0, 2_000_000, 1.0).astype(np.float64)
    assert abs(z.mean()) < 3e-3 and abs(z.std() - 1.0) < 3e-3
    assert z.min() >= -6.0 and z.max() < 6.0
    # Irwin-Hall(12) excess kurtosis is -0.1 (a normal's is 0).
    kurt = np.mean(z ** 4) / np.mean(z ** 2) ** 2 - 3
    assert -0.13 < kurt < -0.07
    # Values are multiples of 2^-16 (the integer sum scaled).
    assert np.all(z * 65536 == np.round(z * 65536))


def test_bf16_rounding_of_draws_matches_torch():
    import torch
    k = synth.key(0, 3)
    f = synth.normal_f32(k, 0, 50000, 0.02)
    b = synth.normal_bf16(k, 0, 50000, 0.02)
    want = torch.tensor(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, want)


def test_uniform_int_range():
    ids = synth.uniform_int(synth.key(0, 13), 0, 200000, 128000)
    assert ids.min() >= 0 and ids.max() < 128000
    assert abs(ids.mean() - 64000) < 600


def test_workload_shapes_and_flops():
    f = W.moe_flops(W.C2)
    assert f["routed"] == 2 * 4096 * 6 * 3 * 2048 * 1408
    assert abs(f["total"] / 1e9 - 568.0) < 1.0
    assert abs(W.moe_flops(W.C3)["total"] / 1e9 - 6524) < 3
    assert W.tensor_shape(W.C3, "w_down") == (256, 7168, 2048)


def test_zipf_bias_frozen():
    beta = W.zipf_beta()
    b = W.zipf_bias(128, beta)
    r = W.zipf_ranks(128)
    assert sorted(r) == list(range(1, 129))
    assert b[np.argmin(r)] == 0.0 and np.all(np.diff(b[np.argsort(r)]) < 0)


def test_f64_widening_matches_bf16_bits():
    """normal_bf16_as_f64 is the bf16 draws widened exactly (a storage format)."""
    k = synth.key(0, 77)
    bits = synth.normal_bf16(k, 1000, 50000, 0.7)
    wide = synth.normal_bf16_as_f64(k, 1000, 50000, 0.7)
    assert np.array_equal(synth.bf16_bits_to_f32(bits).astype(np.float64), wide)
