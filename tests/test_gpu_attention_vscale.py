"""Sink-window attention over chunks whose V tensor scales differ by many
binades.  Every chunk has its own FP32 tensor scale ("2605-LongLive2" DeepRead
page, Method > 推理基础设施: chunk-level NVFP4 with a per-tensor FP32 scale), so
one key set can hold a chunk whose s_V is 2^-40 (or 2^-100) of another's.  The
kernel's fp16 P' must keep the keys that carry O in normal range whichever
chunk they come from, and its softmax denominator must still count keys whose
P' underflows.

Three chunks A, B, C with s_V ratios 1 : r : sqrt(r) (A smallest), and the
attention mass steered by a constant channel 0 (Q[..., 0] = 8, K_c[..., 0] =
k_c, which K-smoothing moves exactly into the chunk's mean):
  small   all the mass on A (the chunk with the smallest s_V carries O),
  even    p_A / p_B = r (A's and B's contributions to O of the same size),
  large   all the mass on B.
Checked against the float64 oracle on every row: relative L2 per (row, head)
and over the tensor <= 1e-2."""
import math

import numpy as np
import pytest

import synth
from gpu_util import assert_attention_close, dev_bf16, host_to_f64

pytestmark = pytest.mark.gpu

Q0 = 8.0
SCALE = 1.0 / math.sqrt(128.0)


def _k0_for_gap(nats):
    """Channel-0 value of K that raises a chunk's logits by `nats` (Q0 * k * scale)."""
    return nats / (Q0 * SCALE)


def _chunk(seed, T, H, v_log2, k0):
    K = synth.k_with_offsets_bf16(seed, 0, 0, (T, H, 128), outlier_p=0.0)
    V = synth.gaussian_bf16(seed, 0, 0, synth.T_V, (T, H, 128))
    Kf = synth.bf16_bits_to_f32(K).astype(np.float64)
    Kf[..., 0] = k0
    Vf = synth.bf16_bits_to_f32(V).astype(np.float64) * 2.0 ** v_log2
    return synth.to_bf16_bits(Kf), synth.to_bf16_bits(Vf)


def _case(mass, log2r):
    """(V scale exponent, channel-0 K value) of chunks A, B, C."""
    v = (-log2r, 0.0, -log2r / 2)
    big = _k0_for_gap(50.0 + 0.7 * log2r)       # a logit gap far beyond r
    if mass == "small":
        k = (big, -big, 0.0)
    elif mass == "large":
        k = (-big, big, 0.0)
    else:                                        # p_A / p_B = r
        k = (_k0_for_gap(log2r * math.log(2.0)), 0.0, _k0_for_gap(log2r * math.log(2.0) / 2))
    return list(zip(v, k))


def _row_rel(out, ref):
    num = np.linalg.norm((out - ref).reshape(out.shape[0], out.shape[1], -1), axis=-1)
    den = np.linalg.norm(ref.reshape(ref.shape[0], ref.shape[1], -1), axis=-1)
    return num / den


def _run(lib, orc, mass, log2r, T_c, H, T_q, seed):
    import torch
    ws = lib.new_workspace(T_c, H)
    bufs, qs = [], []
    for i, (v_log2, k0) in enumerate(_case(mass, log2r)):
        K, V = _chunk(seed + i, T_c, H, v_log2, k0)
        b = lib.ChunkBuffer(T_c, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
        bufs.append(b)
        qs.append(orc.quantize_chunk(K, V))
    Qf = synth.bf16_bits_to_f32(synth.gaussian_bf16(seed + 9, 0, 0, synth.T_Q,
                                                    (T_q, H, 128))).astype(np.float64)
    Qf[..., 0] = Q0
    Q = synth.to_bf16_bits(Qf)
    ref = orc.attention_f64(qs, Q)
    for dt in (torch.float32, torch.bfloat16):
        O = torch.empty((T_q, H, 128), dtype=dt, device="cuda")
        lib.attention(bufs, dev_bf16(Q), O, ws)
        torch.cuda.synchronize()
        assert lib.workspace_status(ws) == lib.OK
        out = host_to_f64(O)
        what = f"{mass} mass, s_V ratio 2^{log2r}, {dt}"
        # the bar, relative to the output's own size (the tensor is tiny when
        # the small-scale chunk carries it)
        norm = float(np.abs(ref).max())
        assert_attention_close(out / norm, ref / norm, what, bf16_output=dt == torch.bfloat16)
        rr = _row_rel(out, ref)
        tol = 1e-2 if dt == torch.float32 else 1e-2 + 2.0 ** -8
        assert float(rr.max()) <= tol, f"{what}: worst row rel-L2 {rr.max():.3e}"


@pytest.mark.parametrize("log2r", [12, 20, 40, 64, 100])
@pytest.mark.parametrize("mass", ["small", "even", "large"])
def test_vscale_spread_split_blocks(lib, orc, mass, log2r):
    """4 query blocks, each split into key ranges merged by the second kernel."""
    _run(lib, orc, mass, log2r, T_c=200, H=2, T_q=300, seed=300 + log2r)


@pytest.mark.parametrize("log2r", [20, 64])
@pytest.mark.parametrize("mass", ["small", "even"])
def test_vscale_spread_whole_blocks(lib, orc, mass, log2r):
    """148 whole query blocks (one full wave, no split): the kernel normalizes
    its rows itself."""
    _run(lib, orc, mass, log2r, T_c=136, H=4, T_q=37 * 256, seed=500 + log2r)


@pytest.mark.parametrize("log2r", [20, 64])
@pytest.mark.parametrize("mass", ["small", "even", "large"])
def test_vscale_spread_fp4_queries(lib, orc, mass, log2r):
    """The FP4-query attention keeps the same per-chunk V-scale reference:
    checked against the oracle with NVFP4-reconstructed queries, every row."""
    import torch
    T_c, H, T_q, seed = 200, 2, 300, 900 + log2r
    ws = lib.new_workspace(T_c, H)
    bufs, qs = [], []
    for i, (v_log2, k0) in enumerate(_case(mass, log2r)):
        K, V = _chunk(seed + i, T_c, H, v_log2, k0)
        b = lib.ChunkBuffer(T_c, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
        bufs.append(b)
        qs.append(orc.quantize_chunk(K, V))
    Qf = synth.bf16_bits_to_f32(synth.gaussian_bf16(seed + 9, 0, 0, synth.T_Q,
                                                    (T_q, H, 128))).astype(np.float64)
    Qf[..., 0] = Q0
    Q = synth.to_bf16_bits(Qf)
    ref = orc.attention_f64_fp4q(qs, Q)
    qb = lib.Fp4QBuffer(T_q, H)
    O = torch.empty((T_q, H, 128), dtype=torch.float32, device="cuda")
    lib.attention_fp4q(bufs, dev_bf16(Q), O, qb, ws)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    out = host_to_f64(O)
    what = f"FP4 queries, {mass} mass, s_V ratio 2^{log2r}"
    norm = float(np.abs(ref).max())
    assert_attention_close(out / norm, ref / norm, what)
    rr = _row_rel(out, ref)
    assert float(rr.max()) <= 1e-2, f"{what}: worst row rel-L2 {rr.max():.3e}"


def test_vscale_spread_beyond_range_is_reported(lib, orc):
    """V scales 2^120 apart exceed what the fp32 softmax sums hold: the call is
    reported as ERR_UNSUPPORTED by the status check (not silently wrong), and
    the next in-range call on the same workspace is OK and correct."""
    import torch
    T_c, H, T_q = 136, 2, 200
    ws = lib.new_workspace(T_c, H)
    bufs, qs = [], []
    for i, (v_log2, k0) in enumerate([(-120.0, 0.0), (0.0, 0.0)]):
        K, V = _chunk(700 + i, T_c, H, v_log2, k0)
        b = lib.ChunkBuffer(T_c, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
        bufs.append(b)
        qs.append(orc.quantize_chunk(K, V))
    Q = synth.gaussian_bf16(709, 0, 0, synth.T_Q, (T_q, H, 128))
    O = torch.empty((T_q, H, 128), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    lib.attention(bufs, dev_bf16(Q), O, ws)
    assert lib.workspace_status(ws) == lib.ERR_UNSUPPORTED
    lib.attention(bufs[1:], dev_bf16(Q), O, ws)
    assert lib.workspace_status(ws) == lib.OK
    assert_attention_close(host_to_f64(O), orc.attention_f64(qs[1:], Q), "after the report")
