"""Pins for the oracle of an FP4-operand S = Q K^T: attention with the queries
replaced by their NVFP4 reconstruction ("2605-LongLive2" DeepRead page, Method
> 推理基础设施: on Blackwell the generator runs W4A4, FP4 GEMMs in place of BF16
ones; Method > 训练基础设施: activations take 1D block scaling).  Q [T_q, H, d]
is quantized as the matrix [T_q * H, d], 16-element blocks along d (the
contraction), Four-Over-Six, one FP32 tensor scale.

Checked against what does not come from that code path:
* the blocks against the brute-force Four-Over-Six encoder (nearest-value
  search on the format definitions), along d, with s = max|Q| / 2688;
* the attention against torch's float64 SDPA over the definition's
  reconstruction RN(decode(q) * RN(decode(sb) * s));
* queries built to be exactly representable (grid values times E4M3 block
  scales, a tensor max of 2688 so that s = 1) come back unchanged, and the
  attention then equals the bf16-query attention bit for bit;
* scaling Q by a power of two moves exactly into the softmax scale."""
import numpy as np
import pytest
import torch

import synth
from brute import e2m1_value, e4m3_value, four_over_six_blocks, pack_codes
from test_oracle_attention import exact_dequant

GRID = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)


def f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _chunks(orc, seed, n=2, T=96, H=2):
    out = []
    for i in range(n):
        K = synth.k_with_offsets_bf16(seed + i, T, H, (T, H, 128))
        V = synth.gaussian_bf16(seed + i, T, H, synth.T_V, (T, H, 128))
        out.append(orc.quantize_chunk(K, V))
    return out


def _sdpa(Qf, chunks, scale=None):
    """softmax(scale Q K^T) V in float64 (torch), keys and values de-quantized
    exactly in the test."""
    Q = torch.from_numpy(np.asarray(Qf, np.float64))
    K = torch.from_numpy(np.concatenate([exact_dequant(c, "k") for c in chunks], axis=0))
    V = torch.from_numpy(np.concatenate([exact_dequant(c, "v") for c in chunks], axis=0))
    scale = scale if scale else 1.0 / np.sqrt(Q.shape[-1])
    out = torch.nn.functional.scaled_dot_product_attention(
        Q.permute(1, 0, 2)[None], K.permute(1, 0, 2)[None], V.permute(1, 0, 2)[None],
        scale=scale)
    return out[0].permute(1, 0, 2).numpy()


def test_fp32_queries_equal_the_bf16_path(orc):
    chunks = _chunks(orc, 700)
    Q = synth.gaussian_bf16(710, 0, 0, synth.T_Q, (40, 2, 128))
    a = orc.attention_f64(chunks, Q)
    b = orc.attention_f64_fq(chunks, f32(Q))
    assert np.array_equal(a, b)


@pytest.mark.parametrize("T_q,H", [(40, 2), (7, 3)])
def test_query_blocks_match_brute_force(orc, T_q, H):
    Q = synth.gaussian_bf16(720 + T_q, 0, 0, synth.T_Q, (T_q, H, 128))
    q, Qh = orc.quantize_queries(Q)
    x = f32(Q)
    s = np.float32(np.abs(x).max()) / np.float32(2688)
    assert np.float32(q["s"]) == s
    codes, sb, keep4 = four_over_six_blocks(x.reshape(-1, 16), s)
    assert np.array_equal(q["scales"].reshape(-1), sb)
    assert np.array_equal(q["choice"].reshape(-1), keep4.astype(np.uint8))
    assert np.array_equal(q["codes"], pack_codes(codes.reshape(T_q * H, 128)))
    # the reconstruction, one fp32 rounding per step
    D = (e4m3_value(sb).astype(np.float32) * s).astype(np.float32)
    want = (e2m1_value(codes).astype(np.float32) * D[:, None]).astype(np.float32)
    assert np.array_equal(Qh.reshape(-1, 16), want)


def test_fp4q_attention_matches_sdpa_over_the_reconstruction(orc):
    chunks = _chunks(orc, 730)
    Q = synth.gaussian_bf16(740, 0, 0, synth.T_Q, (24, 2, 128))
    q = orc.quantize_matrix(Q.reshape(-1, 128), orc.MATRIX_1D)
    codes, sb, _ = four_over_six_blocks(f32(Q).reshape(-1, 16), np.float32(q["s"]))
    D = (e4m3_value(sb).astype(np.float32) * np.float32(q["s"])).astype(np.float32)
    Qh = (e2m1_value(codes).astype(np.float32) * D[:, None]).astype(np.float32).reshape(Q.shape)
    out = orc.attention_f64_fp4q(chunks, Q)
    np.testing.assert_allclose(out, _sdpa(Qh, chunks), rtol=0, atol=1e-12)
    # and it differs from the bf16-query attention by the quantization of Q only
    assert np.abs(out - orc.attention_f64(chunks, Q)).max() > 1e-6


def _representable_queries(T_q, H, seed):
    """Blocks of 16 grid values (one of them +-6) times an E4M3 block scale; the
    first block's scale is 448, the rest smaller, so max|Q| = 2688 and s = 1:
    the 6-target reproduces every block exactly and the 4-target cannot do
    better than a zero error."""
    rng = np.random.default_rng(seed)
    scales = np.array([2.0 ** -4, 0.375, 1.0, 1.75, 5.0, 13.0, 96.0], np.float32)
    nblk = T_q * H * 8
    g = rng.choice(GRID, size=(nblk, 16)) * rng.choice([-1.0, 1.0], size=(nblk, 16))
    g = np.where(rng.random((nblk, 16)) < 0.1, 0.0, g).astype(np.float32)
    g[:, 0] = np.where(rng.random(nblk) < 0.5, -6.0, 6.0)
    m = rng.choice(scales, size=nblk).astype(np.float32)
    m[0] = 448.0
    x = (g * m[:, None]).astype(np.float32).reshape(T_q, H, 128)
    bits = synth.to_bf16_bits(x)
    assert np.array_equal(f32(bits), x)                   # exact in bf16
    return bits


def test_representable_queries_are_unchanged(orc):
    Q = _representable_queries(10, 2, 750)
    q, Qh = orc.quantize_queries(Q)
    assert np.float32(q["s"]) == np.float32(1.0)
    assert not q["choice"].any()                          # the 6-target everywhere
    assert np.array_equal(Qh, f32(Q))
    chunks = _chunks(orc, 760)
    assert np.array_equal(orc.attention_f64_fp4q(chunks, Q), orc.attention_f64(chunks, Q))


def test_power_of_two_query_scaling_moves_into_the_softmax_scale(orc):
    chunks = _chunks(orc, 770)
    Q = synth.gaussian_bf16(780, 0, 0, synth.T_Q, (16, 2, 128))
    Q8 = synth.to_bf16_bits(f32(Q) * np.float32(8.0))
    assert np.array_equal(f32(Q8), f32(Q) * np.float32(8.0))
    sigma = 0.03
    a = orc.attention_f64_fp4q(chunks, Q8, scale=sigma)
    b = orc.attention_f64_fp4q(chunks, Q, scale=sigma * 8.0)
    assert np.array_equal(a, b)
