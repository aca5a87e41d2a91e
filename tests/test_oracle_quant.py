"""Pins for the oracle's chunk quantizer (K-smoothing + NVFP4 micro-blocks with
the Four-Over-Six choice) against what the pages and the mathematics fix:

* the pages' storage formula, (9/8)*T_c*H*d bytes against 4*T_c*H*d for bf16
  ("2605-LongLive2" DeepRead page, Method > 推理基础设施) -- golden fixture;
* a brute-force Four-Over-Six encoder built from nearest-value search
  (tests/brute.py) on every block of the tiny configuration and on whole heads
  of a full-size chunk;
* hand-made blocks whose encodings are known in closed form, one forcing each
  branch of the 6-vs-4 choice, the all-zero block and the underflowing block;
* K-smoothing closed forms: a per-channel constant chunk is reproduced exactly;
  integer-valued chunks give the exactly rounded mean; the 64-token segment
  order is observable and pinned;
* the reconstruction error bound and two exact invariances (sign flip,
  power-of-two scaling).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import synth
from brute import (e2m1_value, e4m3_value, four_over_six_blocks, pack_codes,
                   unpack_codes)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(x):
    return np.float32(x)


def bf16(x):
    return synth.to_bf16_bits(np.asarray(x, np.float64))


def smoothed(K_bits, mean):
    """fp32 K - mean (mean [H, d]), each element one IEEE subtraction."""
    return (synth.bf16_bits_to_f32(K_bits) - mean[None, :, :]).astype(np.float32)


# ------------------------------------------------------------------ storage

def test_storage_formula_matches_pages(orc):
    g = json.load(open(os.path.join(GOLDEN, "kv_storage.json")))
    for (T, H, d) in [(32, 2, 128), (7040, 24, 128), (48, 4, 64)]:
        n = T * H * d
        assert orc.payload_bytes(T, H, d) == g["nvfp4_kv_bytes_per_THd"] * n
        ratio = g["bf16_kv_bytes_per_THd"] * n / orc.payload_bytes(T, H, d)
        assert ratio == pytest.approx(32 / 9)
        assert round(ratio, 1) == g["compression_quoted"]
    # one chunk of 8 latent frames x 880 tokens at 1280x704
    assert 8 * 880 == 7040 and g["frames_per_chunk_quoted"] == 8


def test_output_sizes_are_the_byte_formula(orc):
    K, V, _ = synth.tiny_chunk(0)
    q = orc.quantize_chunk(K, V)
    T, H, d = K.shape
    total = sum(q[k].nbytes for k in ("k_codes", "k_scales", "v_codes", "v_scales"))
    assert total == 9 * T * H * d // 8


# ------------------------------------------------------------------ brute force

def _check_tensor_against_brute(q, X_bits, mean, heads=None):
    T, H, d = X_bits.shape
    x = smoothed(X_bits, mean) if mean is not None else synth.bf16_bits_to_f32(X_bits)
    A = np.abs(x).max()
    s = f32(A) / f32(2688) if A > 0 else f32(1)
    assert np.float32(q["s"]) == s
    heads = range(H) if heads is None else heads
    for h in heads:
        blocks = x[:, h, :].reshape(T * d // 16, 16)
        codes, sb, keep4 = four_over_six_blocks(blocks, s)
        assert np.array_equal(q["scales"][h].reshape(-1), sb), f"scales head {h}"
        assert np.array_equal(q["codes"][h].reshape(T, d // 2),
                              pack_codes(codes.reshape(T, d))), f"codes head {h}"
        assert np.array_equal(q["choice"][h].reshape(-1).astype(bool), keep4)


def test_tiny_config_all_blocks_match_brute_force(orc):
    for c in range(synth.TINY["chunks"]):
        K, V, _ = synth.tiny_chunk(c)
        qk = orc.quantize_tensor(K, smooth=True)
        qv = orc.quantize_tensor(V, smooth=False)
        _check_tensor_against_brute(qk, K, qk["mean"])
        _check_tensor_against_brute(qv, V, None)
        # both branches of the choice occur
        assert 0 < qk["choice"].mean() < 1 and 0 < qv["choice"].mean() < 1


def test_full_size_chunk_heads_match_brute_force(orc):
    K, V = synth.quant_chunk(0)
    qk = orc.quantize_tensor(K, smooth=True)
    qv = orc.quantize_tensor(V, smooth=False)
    _check_tensor_against_brute(qk, K, qk["mean"], heads=[0, 13, 23])
    _check_tensor_against_brute(qv, V, None, heads=[5, 23])


# ------------------------------------------------------------------ closed forms

def _two_block_row(block1):
    """[T=1, H=1, d=32]: block 0 holds the tensor maximum 2688 so s = 1 exactly."""
    row = np.zeros(32)
    row[0] = 2688.0
    row[16:] = block1
    return bf16(row.reshape(1, 1, 32))


def _codes_of(vals):
    lut = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    return np.array([lut[abs(v)] | (8 if (v < 0 or (v == 0 and np.signbit(v))) else 0)
                     for v in vals], np.uint8)


def test_block_exact_at_target_4_keeps_4(orc):
    b1 = [4, 3, 2, 1.5, 1, 0.5, 0, -4, -3, -2, -1.5, -1, -0.5, 0, 4, 1]
    q = orc.quantize_tensor(_two_block_row(b1), smooth=False)
    assert q["s"] == 1.0
    # block 0: 2688/(6*1) = 448 -> scale 448 (0x7E), 6 exactly; the 4-target
    # saturates to the same scale, a tie, so 6 is kept
    assert q["scales"][0, 0, 0] == 0x7E and q["choice"][0, 0, 0] == 0
    # block 1: 4/(4*1) = 1 -> scale 1.0 = 0x38, every element on the grid
    assert q["scales"][0, 0, 1] == 0x38 and q["choice"][0, 0, 1] == 1
    assert np.array_equal(q["codes"][0, 0, 8:], pack_codes(_codes_of(b1)))


def test_block_exact_at_target_6_keeps_6(orc):
    b1 = [6, 4, 3, 2, 1, 0.5, 0, -6, -4, -3, -2, -1, -0.5, 0, 6, 1.5]
    q = orc.quantize_tensor(_two_block_row(b1), smooth=False)
    # 6/(6*1) = 1 -> scale 1.0, exact (error 0); the 4-target (scale 1.5) is not
    assert q["scales"][0, 0, 1] == 0x38 and q["choice"][0, 0, 1] == 0
    assert np.array_equal(q["codes"][0, 0, 8:], pack_codes(_codes_of(b1)))


def test_target_6_scale_rounds_and_target_4_wins(orc):
    # block max 4: the 6-target ratio 4/6 rounds to the E4M3 value 0.6875 (0x33),
    # reconstructing 4 as 6*0.6875 = 4.125; the 4-target is exact
    b1 = [4, 1] + [0] * 14
    q = orc.quantize_tensor(_two_block_row(b1), smooth=False)
    assert q["choice"][0, 0, 1] == 1 and q["scales"][0, 0, 1] == 0x38
    assert orc.e4m3_encode(np.float32([4.0 / 6.0]))[0] == 0x33


def test_zero_and_underflowing_blocks(orc):
    # all-zero block: scale byte 0, codes +0, 6 kept
    q = orc.quantize_tensor(_two_block_row([0.0] * 16), smooth=False)
    assert q["scales"][0, 0, 1] == 0 and not q["codes"][0, 0, 8:].any()
    assert q["choice"][0, 0, 1] == 0
    # block max 1e-3 with s = 1: both ratios are below half the smallest E4M3
    # subnormal (2^-10), so both scales are 0, D = 0 and every code is +0 even
    # for negative inputs
    b1 = [-1e-3] * 8 + [1e-3] * 8
    q = orc.quantize_tensor(_two_block_row(b1), smooth=False)
    assert q["scales"][0, 0, 1] == 0 and not q["codes"][0, 0, 8:].any()


def test_all_zero_tensor_has_unit_scale(orc):
    q = orc.quantize_tensor(np.zeros((5, 2, 32), np.uint16), smooth=True)
    assert q["s"] == 1.0 and not q["codes"].any() and not q["scales"].any()
    assert not q["mean"].any()


# ------------------------------------------------------------------ K-smoothing

def test_constant_channels_reconstruct_exactly(orc):
    rng = np.random.default_rng(5)
    T, H, d = 100, 3, 32                          # 100 = 64 + 36: a ragged segment
    c = bf16(rng.standard_normal((1, H, d)) * 4)
    K = np.repeat(c, T, axis=0)
    q = orc.quantize_tensor(K, smooth=True)
    assert np.array_equal(q["mean"], synth.bf16_bits_to_f32(c)[0])
    assert q["s"] == 1.0 and not q["codes"].any() and not q["scales"].any()
    Kh = orc.dequantize_tensor(q["codes"], q["scales"], q["mean"], q["s"], T, H, d)
    assert np.array_equal(Kh, synth.bf16_bits_to_f32(K))


def rational_to_f32(fr: Fraction) -> np.float32:
    """Correctly rounded (nearest even) float32 of an exact rational."""
    f = np.float32(float(fr))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda v: (abs(Fraction(float(v)) - fr),
                                     int(np.float32(v).view(np.uint32)) & 1))
    return np.float32(best)


def test_mean_is_exactly_rounded_for_integer_chunks(orc):
    rng = np.random.default_rng(6)
    for T in (200, 7, 64, 129):
        K = bf16(rng.integers(-8, 9, size=(T, 2, 16)).astype(np.float64))
        mean = orc.k_mean(K)
        vals = synth.bf16_bits_to_f32(K).astype(np.int64)
        for h in range(2):
            for ch in range(16):
                want = rational_to_f32(Fraction(int(vals[:, h, ch].sum()), T))
                assert mean[h, ch] == want, (T, h, ch)


def test_mean_uses_64_token_segments(orc):
    # column: 2^25 then 63 ones | 64 ones.  In 64-token segments the second
    # segment's ones survive (2^25 + 64, mean 2^18 + 0.5); a single running sum
    # would lose every one (2^25 + 1 rounds back to 2^25, mean 2^18).
    col = np.ones(128)
    col[0] = 2.0 ** 25
    K = np.zeros((128, 1, 16))
    K[:, 0, 0] = col
    mean = orc.k_mean(bf16(K))
    assert mean[0, 0] == np.float32(2.0 ** 18 + 0.5)


# ------------------------------------------------------------------ bounds, invariants

def _element_bound(q, x, T, H, d):
    """Per-element reconstruction bound: half the widest grid gap (1) times D, or
    the overshoot above 6*D when the block scale rounded down."""
    D = e4m3_value(q["scales"]).astype(np.float64) * q["s"]            # [H, T, d/16]
    D = np.repeat(D, 16, axis=2).transpose(1, 0, 2)                     # [T, H, d]
    return np.maximum(D, np.abs(x) - 6 * D) * (1 + 1e-6) + 1e-30


def test_reconstruction_within_bound(orc):
    for c in range(synth.TINY["chunks"]):
        K, V, _ = synth.tiny_chunk(c)
        T, H, d = K.shape
        for X, smooth in ((K, True), (V, False)):
            q = orc.quantize_tensor(X, smooth=smooth)
            x = smoothed(X, q["mean"]) if smooth else synth.bf16_bits_to_f32(X)
            xh = orc.dequantize_tensor(q["codes"], q["scales"], None, q["s"], T, H, d)
            err = np.abs(x.astype(np.float64) - xh)
            assert np.all(err <= _element_bound(q, x, T, H, d))
            if smooth:          # dequant(K - mu) + mu against K itself
                Kh = orc.dequantize_tensor(q["codes"], q["scales"], q["mean"], q["s"], T, H, d)
                Kf = synth.bf16_bits_to_f32(X).astype(np.float64)
                slack = np.abs(q["mean"]).max() * 2.0 ** -22
                assert np.all(np.abs(Kf - Kh) <= _element_bound(q, x, T, H, d) + slack)


def test_sign_flip_flips_code_signs_only(orc):
    K, V, _ = synth.tiny_chunk(1)
    for X, smooth in ((K, True), (V, False)):
        q = orc.quantize_tensor(X, smooth=smooth)
        qn = orc.quantize_tensor(X ^ np.uint16(0x8000), smooth=smooth)
        assert qn["s"] == q["s"]
        assert np.array_equal(qn["scales"], q["scales"])
        assert np.array_equal(qn["choice"], q["choice"])
        if smooth:
            assert np.array_equal(qn["mean"], -q["mean"])
        x = smoothed(X, q["mean"]) if smooth else synth.bf16_bits_to_f32(X)
        nz = (x != 0).transpose(1, 0, 2)                       # [H, T, d]
        a, b = unpack_codes(q["codes"]), unpack_codes(qn["codes"])
        assert np.array_equal(b[nz], a[nz] ^ 8)
        assert np.array_equal(b[~nz], a[~nz])


@pytest.mark.parametrize("k", [3, -3])
def test_power_of_two_scaling_keeps_codes_and_scales(orc, k):
    K, V, _ = synth.tiny_chunk(2)
    for X, smooth in ((K, True), (V, False)):
        Xs = bf16(synth.bf16_bits_to_f32(X).astype(np.float64) * 2.0 ** k)
        q = orc.quantize_tensor(X, smooth=smooth)
        qs = orc.quantize_tensor(Xs, smooth=smooth)
        assert np.float32(qs["s"]) == np.float32(q["s"]) * np.float32(2.0 ** k)
        assert np.array_equal(qs["codes"], q["codes"])
        assert np.array_equal(qs["scales"], q["scales"])
        if smooth:
            assert np.array_equal(qs["mean"], q["mean"] * np.float32(2.0 ** k))


def test_dequantize_is_decode_times_scale(orc):
    K, V, _ = synth.tiny_chunk(3)
    T, H, d = V.shape
    q = orc.quantize_tensor(V, smooth=False)
    xh = orc.dequantize_tensor(q["codes"], q["scales"], None, q["s"], T, H, d)
    v = e2m1_value(unpack_codes(q["codes"]))                                # [H, T, d]
    D = np.repeat(e4m3_value(q["scales"]) * np.float32(q["s"]), 16, axis=2)
    assert np.array_equal(xh, (v * D).astype(np.float32).transpose(1, 0, 2))


def test_tiny_digest_unchanged(orc):
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_tiny_digest", os.path.join(GOLDEN, "make_tiny_digest.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert mod.digest() == json.load(open(os.path.join(GOLDEN, "tiny_chunk0_digest.json")))
