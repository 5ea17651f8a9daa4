"""The torch version of the input generator (used to draw the DiT stack on the
GPU) against the numpy definition, on the CPU."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from svdq_inputs import generator as g
from svdq_inputs import torch_gen as tg
from svdq_inputs import workloads as wl


def test_words_bit_identical():
    seed = g.stream_seed(0x5EED0000 + 5000 + 3, 1)
    ref = g.SplitMix64Stream(seed).take(4097)
    got = tg.words(seed, 0, 4097, "cpu").numpy().view(np.uint64)
    assert np.array_equal(ref, got)
    # a window further along the stream (the counter offset)
    s = g.SplitMix64Stream(seed)
    s.take(1000)
    assert np.array_equal(s.take(64), tg.words(seed, 1000, 64, "cpu").numpy().view(np.uint64))


def test_uniform_bit_identical():
    seed = g.stream_seed(12345, 7)
    ref = g.uniform(g.SplitMix64Stream(seed), 5000)
    got = tg.uniform(seed, 5000, "cpu").numpy()
    assert np.array_equal(ref, got)
    assert got.min() >= 0.0 and got.max() < 1.0


def test_bf16_rounding_matches_numpy_rule():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(size=20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.array([0.0, -0.0, 1.0, -1.0]),
                        # exact midpoints between bf16 neighbours: ties go to even
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)])])
    ref = g.bf16_bits_from_f64(x)
    got = tg.bf16_from_f64(torch.from_numpy(x)).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ref, got)


def _ulp_diff(a, b):
    a = a.astype(np.int32)
    b = b.astype(np.int32)
    return np.abs(a - b)


def test_stack_layer_matches_numpy_generator():
    # a narrow slice of a real stack layer's streams: same seeds and counters
    M = 8
    li = wl.make_stack_layer_inputs(1, M=M)          # 3072 -> 3072, outlier activations
    d = tg.make_stack_layer(1, M, "cpu")
    for name, ref, got in (("X", li.X, d["X"]), ("W", li.W, d["W"]),
                           ("A", li.lora_A, d["A"]), ("B", li.lora_B, d["B"])):
        got = got.view(torch.int16).numpy().view(np.uint16)
        assert got.shape == ref.shape, name
        same = np.mean(got == ref)
        # the integer streams are identical; fp64 transcendental ulps may flip
        # a bf16 rounding in a tiny fraction of elements, never by more than 1
        assert same >= 0.9999, (name, same)
        assert _ulp_diff(got, ref).max() <= 1, name


def test_gelu_activation_matches_numpy_generator():
    K, N, kind = wl.stack_layer_shapes()[3]
    assert kind == "gelu"
    li = wl.make_stack_layer_inputs(3, M=2)
    d = tg.make_stack_layer(3, 2, "cpu")
    got = d["X"].view(torch.int16).numpy().view(np.uint16)
    assert np.mean(got == li.X) >= 0.9999
    assert _ulp_diff(got, li.X).max() <= 1
