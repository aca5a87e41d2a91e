"""The seeded input generator: SplitMix64 against its published output sequence
(seed 1234567), split-independence of the threaded evaluation, and the
moments of the recipes."""
import numpy as np

import synth


def test_splitmix64_reference_sequence():
    # first outputs of SplitMix64 seeded with 1234567 (the reference sequence
    # published with the algorithm's C implementation)
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert [int(w) for w in synth.words(1234567, 5)] == want


def test_streams_are_split_independent(monkeypatch):
    key = synth.stream_key(3, 1, 2, synth.T_K)
    a = synth.normal(key, 3_000_001)
    monkeypatch.setattr(synth, "_PARALLEL_MIN", 1 << 40)
    b = synth.normal(key, 3_000_001)
    assert np.array_equal(a, b)
    assert np.array_equal(synth.words(key, 100, start=50), synth.words(key, 150)[50:])


def test_recipe_moments():
    z = synth.normal(synth.stream_key(1), 1_000_000)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    K, V, Q = synth.tiny_chunk(0)
    k = synth.bf16_bits_to_f32(K)
    assert abs(k[..., 7].mean() - 8) < 0.2 and abs(np.delete(k, 7, axis=2).mean()) < 0.05
    Kq = synth.bf16_bits_to_f32(synth.k_with_offsets_bf16(5, 0, 0, (512, 4, 128)))
    dev = Kq - Kq.mean(axis=0, keepdims=True)
    frac_big = (np.abs(dev) > 8).mean()           # outliers x20 on 1% of elements
    assert 0.005 < frac_big < 0.012


def test_device_generator_matches_the_host_one():
    """synth.device (torch, here on the CPU) draws the same bits as the host
    generator: words, uniforms, and the bf16 recipes of the quantize-only chunk."""
    import torch

    import synth.device as sd
    key = synth.stream_key(7, 1, 2, synth.T_K)
    assert np.array_equal(sd.words(key, 1000, "cpu").numpy().view(np.uint64),
                          synth.words(key, 1000))
    assert np.array_equal(sd.uniform(key, 999, "cpu").numpy(), synth.uniform(key, 999))
    shape = (96, 3, 128)
    K = sd.k_with_offsets_bf16(5, 0, 0, shape, "cpu")
    V = sd.gaussian_bf16(5, 0, 0, synth.T_V, shape, "cpu")
    assert K.dtype == torch.bfloat16 and tuple(K.shape) == shape
    assert np.array_equal(K.view(torch.int16).numpy().view(np.uint16),
                          synth.k_with_offsets_bf16(5, 0, 0, shape))
    assert np.array_equal(V.view(torch.int16).numpy().view(np.uint16),
                          synth.gaussian_bf16(5, 0, 0, synth.T_V, shape))
    Kq, Vq = sd.quant_chunk(3, "cpu", T_c=64, H=2)
    Kh, Vh = synth.quant_chunk(3, T_c=64, H=2)
    assert np.array_equal(Kq.view(torch.int16).numpy().view(np.uint16), Kh)
    assert np.array_equal(Vq.view(torch.int16).numpy().view(np.uint16), Vh)
