"""Pins for the oracle's number formats: E2M1 elements and E4M3 block scales.

The oracle writes its encoders as decision-point lists; these tests check them
against what the formats fix independently: the bit-field definitions
(sign / exponent / mantissa with their biases), nearest-value brute force over
the whole representable set with the even-code tie rule, and PyTorch's own
float8_e4m3fn conversion.  Sources: "2605-LongLive2" DeepRead page, Method >
训练基础设施 (E2M1 element, FP8 E4M3 block scale, FP32 tensor scale).
"""
import numpy as np
import pytest
import torch


from brute import (E2M1_MAGS, E4M3_POS, brute_e2m1, brute_e4m3, e2m1_from_bits,
                   e4m3_from_bits, midpoints_with_neighbours)


# ------------------------------------------------------------------ E2M1

def test_e2m1_decode_matches_bit_fields(orc):
    for c in range(16):
        assert orc.e2m1_decode(np.array([c], np.uint8))[0] == np.float32(e2m1_from_bits(c))
    # the grid named for the cache: {0, .5, 1, 1.5, 2, 3, 4, 6}
    assert list(E2M1_MAGS) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_round_trip_all_codes(orc):
    codes = np.arange(16, dtype=np.uint8)
    vals = orc.e2m1_decode(codes)
    # -0.0 decodes with its sign and re-encodes to 0x8
    assert np.array_equal(orc.e2m1_encode(vals), codes)


def test_e2m1_midpoints_and_neighbours_match_brute_force(orc):
    pts = midpoints_with_neighbours(E2M1_MAGS)
    pts = np.concatenate([pts, -pts, np.float32([7.0, 1e30, -1e30, 6.5, 1e-40, -1e-40, 0.0, -0.0])])
    assert np.array_equal(orc.e2m1_encode(pts), brute_e2m1(pts))


def test_e2m1_random_sweep_matches_brute_force(orc):
    rng = np.random.default_rng(11)
    y = np.concatenate([
        rng.uniform(-8, 8, 1_000_000),
        rng.standard_normal(500_000) * np.exp2(rng.integers(-12, 6, 500_000)),
    ]).astype(np.float32)
    assert np.array_equal(orc.e2m1_encode(y), brute_e2m1(y))


def test_e2m1_ties_go_to_even_code(orc):
    ties = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    want = np.uint8([0, 2, 2, 4, 4, 6, 6])          # even magnitude index
    assert np.array_equal(orc.e2m1_encode(ties), want)
    assert np.array_equal(orc.e2m1_encode(-ties), want | 8)


# ------------------------------------------------------------------ E4M3

def test_e4m3_decode_matches_bit_fields_and_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(codes).astype(np.float64)
    fields = np.array([e4m3_from_bits(c) for c in range(256)])
    assert np.array_equal(np.isnan(ours), np.isnan(fields))
    ok = ~np.isnan(fields)
    assert np.array_equal(ours[ok], fields[ok])
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(ours[ok], lib[ok])
    assert fields[0x7E] == 448.0 and np.isnan(fields[0x7F])


def test_e4m3_round_trip_all_finite_codes(orc):
    codes = np.arange(0x7F, dtype=np.uint8)
    assert np.array_equal(orc.e4m3_encode(orc.e4m3_decode(codes)), codes)


def test_e4m3_midpoints_match_brute_force(orc):
    pts = midpoints_with_neighbours(E4M3_POS)
    pts = np.concatenate([pts, np.float32([448.0, 460.0, 463.99, 464.0, 480.0, 1e9, 0.0,
                                           2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11])])
    assert np.array_equal(orc.e4m3_encode(pts), brute_e4m3(pts))


def test_e4m3_random_sweep_matches_brute_force_and_torch(orc):
    rng = np.random.default_rng(12)
    y = np.concatenate([
        rng.uniform(0, 500, 200_000),
        np.exp2(rng.uniform(-12, 9.5, 300_000)),
    ]).astype(np.float32)
    ours = orc.e4m3_encode(y)
    assert np.array_equal(ours, brute_e4m3(y))
    # PyTorch's float32 -> float8_e4m3fn cast rounds to nearest even; compare
    # where it does not overflow (it is not a saturating cast)
    inr = y <= 448.0
    lib = torch.from_numpy(y[inr]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours[inr], lib)
    assert np.all(ours[y > 448.0] == 0x7E)


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(13)
    x = (rng.standard_normal(1_000_000) * np.exp2(rng.integers(-30, 30, 1_000_000))).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16(x), lib)
