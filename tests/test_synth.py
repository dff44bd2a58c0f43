"""The seeded input recipe the tests and the oracle share (stated in the
design notes, reading s13): linear weights N(0, 0.02) rounded to bf16, biases
0, norm scales 1, tokens and conditioning N(0, 1); one independent stream per
(seed, tensor name); Flux position ids (0,0,0) for text and (0,h,w) row-major
for the image grid.  The generator holds none of the block's arithmetic."""
import numpy as np

from diffusion_transformer_block_flux_b200 import synth


def test_weights_follow_the_recipe():
    s = synth.TINY
    w = synth.single_block_weights(s)
    W1 = synth.bf16_bits_to_f64(w["W1"])
    assert W1.shape == (3 * s.D + s.M, s.D)
    assert abs(W1.mean()) < 1e-3 and abs(W1.std() - 0.02) < 5e-4
    assert not synth.bf16_bits_to_f64(w["b1"]).any() and not synth.bf16_bits_to_f64(w["b2"]).any()
    assert np.all(synth.bf16_bits_to_f64(w["q_scale"]) == 1.0)
    a = synth.block_activations(s)
    x = synth.bf16_bits_to_f64(a["x"])
    assert x.shape == (s.S, s.D) and abs(x.std() - 1.0) < 2e-2


def test_streams_are_seeded_per_tensor_and_deterministic():
    a = synth.normal_bf16(0, "t", (64, 64))
    assert np.array_equal(a, synth.normal_bf16(0, "t", (64, 64)))  # same seed and name: same bits
    assert not np.array_equal(a, synth.normal_bf16(0, "u", (64, 64)))  # another name: another stream
    assert not np.array_equal(a, synth.normal_bf16(1, "t", (64, 64)))  # another seed: another stream


def test_bf16_rounding_is_round_to_nearest_even():
    # 1 + 2^-8 lies halfway between bf16 1.0 and 1 + 2^-7: ties go to the even mantissa (1.0)
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], dtype=np.float32)
    got = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(x))
    assert got.tolist() == [1.0, 1.0 + 2 * 2.0 ** -7, -2.5, 0.0]


def test_flux_position_ids():
    ids = synth.flux_ids(3, 2, 4)
    assert ids.shape == (3 + 8, 3) and ids.dtype == np.int32
    assert not ids[:3].any()  # text tokens at (0, 0, 0)
    img = ids[3:]
    assert not img[:, 0].any()
    assert img[:, 1].tolist() == [0, 0, 0, 0, 1, 1, 1, 1] and img[:, 2].tolist() == [0, 1, 2, 3] * 2
