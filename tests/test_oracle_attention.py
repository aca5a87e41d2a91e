"""Pins for the oracle's sink-window attention and key set.

Key set ("2605-LongLive2" DeepRead page, Method > 算法层设计, Multi-Shot
Attention Sink: K_eff(t) = A_g u A_s u KV[t-W, t), overlapping tokens counted
once, A_s re-bound on a prompt switch) against a brute-force set union.

Attention against PyTorch's scaled_dot_product_attention in float64 over keys
de-quantized in the test (exact products), and against closed forms: when the
window covers all history it is block-causal full attention; with W = 0 it is
sink-only attention; de-duplication is exact (and a duplicated list differs);
a single key returns its value row; identical keys return the mean of values;
key order does not matter; a vanishing scale gives the mean of values.
"""
import random

import numpy as np
import pytest
import torch

import synth
from brute import e2m1_value, e4m3_value, unpack_codes


def brute_keyset(n, S_g, S_s, W, s_begin):
    ids = set(range(min(S_g, n)))
    ids |= {c for c in range(s_begin, s_begin + S_s) if 0 <= c < n}
    ids |= set(range(max(0, n - W), n))
    return sorted(ids)


def test_keyset_matches_set_union(orc):
    rng = random.Random(7)
    for _ in range(3000):
        n = rng.randint(0, 40)
        S_g, S_s, W = rng.randint(0, 4), rng.randint(0, 4), rng.randint(0, 8)
        s_begin = rng.randint(0, max(0, n + 2))
        assert orc.keyset(n, S_g, S_s, W, s_begin) == brute_keyset(n, S_g, S_s, W, s_begin)


def test_keyset_of_the_configs(orc):
    # one-layer attention: global sink {0}, shot sink {4}, window {7, 8, 9}
    assert orc.keyset(10, 1, 1, 3, 4) == [0, 4, 7, 8, 9]
    # 30-layer rollout: 16 chunks, S_g = S_s = 1, W = 4, no switch
    assert sum(len(orc.keyset(n, 1, 1, 4, 0)) for n in range(1, 17)) == 70
    # multi-shot stream: switches at 12, 28, 45 re-bind the shot sink
    total, s_begin = 0, 0
    for n in range(1, 65):
        if n - 1 in (12, 28, 45):
            s_begin = n - 1
        total += len(orc.keyset(n, 1, 1, 4, s_begin))
    assert total == 350


# ------------------------------------------------------------------ attention

def exact_dequant(q, which):
    """float64 [T, H, d] of decode(q) * decode(sb) * s (+ mean for K), exact."""
    codes = unpack_codes(q[which + "_codes"]).astype(np.float64)           # [H, T, d]
    v = e2m1_value(unpack_codes(q[which + "_codes"])).astype(np.float64)
    sc = np.repeat(e4m3_value(q[which + "_scales"]).astype(np.float64), 16, axis=2)
    x = v * sc * float(q["s_" + which])
    if which == "k":
        x = x + q["k_mean"].astype(np.float64)[:, None, :]
    del codes
    return x.transpose(1, 0, 2)


def textbook(Q_bits, chunks, scale=None, mask=None):
    """softmax(scale Q K^T) V in float64 with torch's SDPA."""
    Q = torch.from_numpy(synth.bf16_bits_to_f32(Q_bits).astype(np.float64))
    K = torch.from_numpy(np.concatenate([exact_dequant(c, "k") for c in chunks], axis=0))
    V = torch.from_numpy(np.concatenate([exact_dequant(c, "v") for c in chunks], axis=0))
    d = Q.shape[-1]
    scale = scale if scale else 1.0 / np.sqrt(d)
    out = torch.nn.functional.scaled_dot_product_attention(
        Q.permute(1, 0, 2)[None], K.permute(1, 0, 2)[None], V.permute(1, 0, 2)[None],
        attn_mask=mask, scale=scale)
    return out[0].permute(1, 0, 2).numpy()


@pytest.fixture(scope="module")
def tiny(orc):
    data = [synth.tiny_chunk(c) for c in range(4)]
    qs = [orc.quantize_chunk(K, V) for (K, V, _) in data]
    return data, qs


def test_full_window_is_block_causal_full_attention(orc, tiny):
    data, qs = tiny
    T = data[0][0].shape[0]
    Qall = np.concatenate([d[2] for d in data], axis=0)
    # block-causal mask: query chunk i sees key chunks 0..i
    qi = np.arange(4 * T) // T
    mask = torch.from_numpy(qi[:, None] >= qi[None, :])
    ref = textbook(Qall, qs, mask=mask)
    for n in range(1, 5):
        ids = orc.keyset(n, 1, 1, 8, 0)                 # W = 8 >= n covers all history
        assert ids == list(range(n))
        out = orc.attention_f64([qs[i] for i in ids], data[n - 1][2])
        np.testing.assert_allclose(out, ref[(n - 1) * T:n * T], rtol=0, atol=1e-12)


def test_zero_window_is_sink_only(orc, tiny):
    data, qs = tiny
    ids = orc.keyset(4, 1, 1, 0, 2)
    assert ids == [0, 2]
    out = orc.attention_f64([qs[i] for i in ids], data[3][2])
    np.testing.assert_allclose(out, textbook(data[3][2], [qs[0], qs[2]]), rtol=0, atol=1e-12)


def test_overlapping_sinks_are_deduplicated(orc, tiny):
    data, qs = tiny
    # shot sink at chunk 0 overlaps the global sink; window {2, 3}
    ids = orc.keyset(4, 1, 1, 2, 0)
    assert ids == [0, 2, 3]
    out = orc.attention_f64([qs[i] for i in ids], data[3][2])
    np.testing.assert_allclose(out, textbook(data[3][2], [qs[0], qs[2], qs[3]]),
                               rtol=0, atol=1e-12)
    dup = orc.attention_f64([qs[0], qs[0], qs[2], qs[3]], data[3][2])
    assert np.abs(dup - out).max() > 1e-3           # counting chunk 0 twice changes O


def test_single_key_returns_its_value(orc):
    K, V, Q = (synth.gaussian_bf16(9, 0, 0, t, (1, 2, 128)) for t in (1, 2, 3))
    q = orc.quantize_chunk(K, V)
    out = orc.attention_f64([q], np.repeat(Q, 5, axis=0))
    want = exact_dequant(q, "v")
    np.testing.assert_allclose(out, np.repeat(want, 5, axis=0), rtol=0, atol=1e-15)


def test_identical_keys_give_mean_of_values(orc):
    T, H, d = 40, 2, 128
    Krow = synth.gaussian_bf16(10, 0, 0, 1, (1, H, d))
    K = np.repeat(Krow, T, axis=0)
    V = synth.gaussian_bf16(10, 0, 0, 2, (T, H, d))
    Q = synth.gaussian_bf16(10, 0, 0, 3, (7, H, d))
    q = orc.quantize_chunk(K, V)
    out = orc.attention_f64([q], Q)
    want = exact_dequant(q, "v").mean(axis=0)
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=1e-12)


def test_key_order_does_not_matter(orc, tiny):
    data, qs = tiny
    a = orc.attention_f64([qs[0], qs[1], qs[3]], data[3][2])
    b = orc.attention_f64([qs[3], qs[0], qs[1]], data[3][2])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_vanishing_scale_gives_mean_of_values(orc, tiny):
    data, qs = tiny
    out = orc.attention_f64([qs[1], qs[2]], data[2][2], scale=1e-12)
    V = np.concatenate([exact_dequant(qs[1], "v"), exact_dequant(qs[2], "v")], axis=0)
    np.testing.assert_allclose(out, np.broadcast_to(V.mean(axis=0), out.shape), atol=1e-9)


def test_sampled_rows_equal_full_rows(orc, tiny):
    data, qs = tiny
    full = orc.attention_f64(qs[:3], data[2][2])
    rows = [0, 5, 31, 17]
    part = orc.attention_f64(qs[:3], data[2][2], rows=rows)
    assert np.array_equal(part, full[rows])
