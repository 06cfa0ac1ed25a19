"""The seeded input generator: SplitMix64 outputs, normals, bf16 rounding, embedding."""
import math

import numpy as np

from vsa_synth import (bf16_bits_to_f32, f32_to_bf16_bits, get_config, make_layer_inputs,
                       position_embedding, splitmix64_outputs, standard_normal)


def test_splitmix64_published_outputs():
    # first outputs of SplitMix64 seeded with 0 (reference implementation by S. Vigna)
    got = [int(x) for x in splitmix64_outputs(np.uint64(0), 0, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_windows_agree():
    a = splitmix64_outputs(np.uint64(77), 0, 1000)
    b = splitmix64_outputs(np.uint64(77), 400, 100)
    assert np.array_equal(a[400:500], b)
    n = standard_normal(np.uint64(5), 0, 200_000)
    assert abs(n.mean()) < 0.01 and abs(n.std() - 1) < 0.01


def test_bf16_rounding():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 0.0, 3.0e38], dtype=np.float32)
    bits = f32_to_bf16_bits(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F81, 0xC020, 0x0000, 0x7F62]
    assert np.array_equal(bf16_bits_to_f32(bits)[:4], np.array([1.0, 1.0, 1.0 + 2 ** -7, -2.5], np.float32))


def test_position_embedding_smooth():
    pe = position_embedding(4, 8, 8, 12)
    assert pe.shape == (256, 12)
    # channel 0 follows t with wavelength 8, sine phase: token (t=2,0,0) -> sin(pi/2) = 1
    assert abs(pe[2 * 64, 0] - 1.0) < 1e-12
    # channel 3 follows t with cosine phase: token (0,0,0) -> 1
    assert abs(pe[0, 3] - 1.0) < 1e-12
    # channel 7 follows h with wavelength 16
    assert abs(pe[4 * 8, 7] - math.sin(2 * math.pi * 4 / 16)) < 1e-12


def test_layer_inputs_deterministic():
    cfg = get_config("tiny")
    a, b = make_layer_inputs(cfg), make_layer_inputs(cfg)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.gate, b.gate)
    assert a.q.shape == (1, 384, 2, 64) and a.q.dtype == np.uint16
    assert not np.array_equal(a.q, a.k)
