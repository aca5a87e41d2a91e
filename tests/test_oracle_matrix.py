"""Pins of the oracle's NVFP4 weight / activation quantizer with Four-Over-Six
(DeepRead page, Method > 训练基础设施: 1D row blocks for activations, 2D 16 x 16
blocks for weights), against what the definitions fix:

* every block of random matrices (with outliers) against the brute-force
  encoder of tests/brute.py (nearest-value search, bit-field decoding);
* 1D blocks against the KV path's V quantization of the same numbers;
* hand-made tiles whose encodings are known in closed form: exact at target 4
  (4 kept), exact at target 6 (6 kept), all zero, a lone nonzero element;
* the sign-flip and power-of-two invariants, the reconstruction bound, and the
  shapes each mode refuses."""
import numpy as np
import pytest

import synth
from brute import e2m1_value, e4m3_value, four_over_six_blocks, four_over_six_tiles, pack_codes


def bf16(a):
    return synth.to_bf16_bits(np.asarray(a, np.float64))


def f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _matrix(seed, M, N, outlier=30.0):
    z = synth.normal(synth.stream_key(seed, 0, 0, synth.T_EXTRA), M * N).reshape(M, N)
    u = synth.uniform(synth.stream_key(seed, 0, 1, synth.T_EXTRA), M * N).reshape(M, N)
    return bf16(np.where(u < 0.01, z * outlier, z))


@pytest.mark.parametrize("M,N", [(48, 256), (7, 64), (1, 16)])
def test_row_blocks_match_brute_force(orc, M, N):
    X = _matrix(11 + M, M, N)
    q = orc.quantize_matrix(X, orc.MATRIX_1D)
    codes, sb, keep4 = four_over_six_blocks(f32(X).reshape(-1, 16), np.float32(q["s"]))
    assert np.array_equal(q["scales"].reshape(-1), sb)
    assert np.array_equal(q["choice"].reshape(-1), keep4.astype(np.uint8))
    assert np.array_equal(q["codes"], pack_codes(codes.reshape(M, N)))


@pytest.mark.parametrize("M,N", [(64, 128), (16, 16), (48, 80)])
def test_tiles_match_brute_force(orc, M, N):
    X = _matrix(21 + M, M, N)
    q = orc.quantize_matrix(X, orc.MATRIX_2D)
    tiles = f32(X).reshape(M // 16, 16, N // 16, 16).transpose(0, 2, 1, 3).reshape(-1, 16, 16)
    codes, sb, keep4 = four_over_six_tiles(tiles, np.float32(q["s"]))
    assert np.array_equal(q["scales"].reshape(-1), sb)
    assert np.array_equal(q["choice"].reshape(-1), keep4.astype(np.uint8))
    full = codes.reshape(M // 16, N // 16, 16, 16).transpose(0, 2, 1, 3).reshape(M, N)
    assert np.array_equal(q["codes"], pack_codes(full))


def test_row_blocks_equal_the_kv_value_path(orc):
    """The same numbers as V of a chunk [T=M][H=N/128][128]: identical scales and
    codes (the cache stores them head-major)."""
    M, N = 40, 384
    X = _matrix(31, M, N)
    a = orc.quantize_matrix(X, orc.MATRIX_1D)
    v = orc.quantize_tensor(X.reshape(M, N // 128, 128), smooth=False)
    assert a["s"] == v["s"]
    assert np.array_equal(a["scales"], v["scales"].transpose(1, 0, 2).reshape(M, N // 16))
    assert np.array_equal(a["codes"], v["codes"].transpose(1, 0, 2).reshape(M, N // 2))


def _codes_of(vals):
    lut = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    return np.array([lut[abs(v)] | (8 if v < 0 else 0) for v in vals], np.uint8)


def test_hand_made_tiles(orc):
    """32 x 32, s = 1 (2688 in tile (0,0)).  Tile (0,1): every row on the grid
    at scale 1 with max 4 -> target 4 exact, kept.  Tile (1,0): max 6, on the
    grid at scale 1 -> target 6 exact, kept.  Tile (1,1): zeros -> scale 0."""
    b4 = [4, 3, 2, 1.5, 1, 0.5, 0, -4, -3, -2, -1.5, -1, -0.5, 0, 4, 1]
    b6 = [6, 4, 3, 2, 1, 0.5, 0, -6, -4, -3, -2, -1, -0.5, 0, 6, 1.5]
    W = np.zeros((32, 32))
    W[0, 0] = 2688.0
    W[0:16, 16:32] = b4
    W[16:32, 0:16] = b6
    q = orc.quantize_matrix(bf16(W), orc.MATRIX_2D)
    assert q["s"] == 1.0
    assert q["scales"][0, 0] == 0x7E and q["choice"][0, 0] == 0       # 2688/6 = 448: a tie, 6 kept
    assert q["scales"][0, 1] == 0x38 and q["choice"][0, 1] == 1       # 4/4 = 1.0
    assert q["scales"][1, 0] == 0x38 and q["choice"][1, 0] == 0       # 6/6 = 1.0
    assert q["scales"][1, 1] == 0 and q["choice"][1, 1] == 0
    for r in range(16):
        assert np.array_equal(q["codes"][r, 8:16], pack_codes(_codes_of(b4)))
        assert np.array_equal(q["codes"][16 + r, 0:8], pack_codes(_codes_of(b6)))
    assert not q["codes"][16:, 8:].any()


@pytest.mark.parametrize("mode", [1, 2])
def test_lone_nonzero_element(orc, mode):
    """One nonzero v: s = |v|/2688, its block's scale is 448 (0x7E) and its code
    6 with v's sign; every other block has scale 0 and +0 codes."""
    W = np.zeros((32, 48))
    W[19, 37] = -3.5
    q = orc.quantize_matrix(bf16(W), mode)
    assert q["s"] == np.float32(3.5) / np.float32(2688.0)
    br = 19 if mode == 1 else 1
    assert q["scales"][br, 2] == 0x7E
    assert q["scales"].sum() == 0x7E
    assert q["codes"][19, 18] == 0xF << 4          # element 37 = high nibble of byte 18: -6
    q["codes"][19, 18] = 0
    assert not q["codes"].any()


@pytest.mark.parametrize("mode", [1, 2])
def test_sign_flip_and_power_of_two_invariants(orc, mode):
    X = _matrix(41, 32, 64)
    q = orc.quantize_matrix(X, mode)
    neg = orc.quantize_matrix(X ^ np.uint16(0x8000), mode)
    assert np.array_equal(neg["scales"], q["scales"]) and neg["s"] == q["s"]
    assert np.array_equal(neg["codes"], q["codes"] ^ np.uint8(0x88))
    for k in (-3, 5):
        sc = orc.quantize_matrix(bf16(f32(X).astype(np.float64) * 2.0 ** k), mode)
        assert sc["s"] == np.float32(q["s"] * 2.0 ** k)
        assert np.array_equal(sc["scales"], q["scales"]) and np.array_equal(sc["codes"], q["codes"])


@pytest.mark.parametrize("mode", [1, 2])
def test_reconstruction_within_the_step(orc, mode):
    """|x - x_hat| <= D (the block step: at most half the widest E2M1 gap, 2D),
    unless x lies beyond 6 D, where the code saturates."""
    X = _matrix(51, 48, 96)
    q = orc.quantize_matrix(X, mode)
    xh = orc.dequantize_matrix(q, mode)
    rows = 1 if mode == 1 else 16
    D = (e4m3_value(q["scales"]) * np.float32(q["s"])).astype(np.float32)    # RN(decode(sb) s)
    Dfull = np.repeat(np.repeat(D, rows, axis=0), 16, axis=1)
    x = f32(X).astype(np.float64)
    err = np.abs(x - xh)
    bound = np.maximum(Dfull, np.abs(x) - 6 * Dfull.astype(np.float64)) * (1 + 1e-6)
    assert (err <= bound).all()
    codes = np.stack([q["codes"] & 15, q["codes"] >> 4], axis=-1).reshape(xh.shape)
    assert np.array_equal(xh, (e2m1_value(codes) * Dfull).astype(np.float32))


def test_shapes_the_modes_refuse(orc):
    with pytest.raises(ValueError):
        orc.quantize_matrix(np.zeros((4, 24), np.uint16), orc.MATRIX_1D)
    with pytest.raises(ValueError):
        orc.quantize_matrix(np.zeros((24, 32), np.uint16), orc.MATRIX_2D)
