"""GPU quantizer and de-quantizer against the oracle, bit for bit: FP4 codes,
E4M3 scale bytes, the K-smoothing mean and both tensor scales, on the tiny
configuration, on full-size quantize-only chunks (7040 x 24 x 128) and on
ragged and degenerate shapes."""
import numpy as np
import pytest

import synth
from gpu_util import Guarded, GuardedChunk, dev_bf16

pytestmark = pytest.mark.gpu


def _gpu_quant(lib, K, V, ws=None, guard=False):
    """Quantize on the GPU; with guard, into a chunk carved from a sentinel
    buffer whose bytes outside the chunk's parts are checked afterwards."""
    import torch
    T, H, d = K.shape
    ws = lib.new_workspace(T, H, d) if ws is None else ws
    g = GuardedChunk(lib, T, H) if guard else None
    out = g.chunk if guard else lib.ChunkBuffer(T, H, d)
    lib.quantize_chunk(dev_bf16(K), dev_bf16(V), out, ws)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    if guard:
        g.assert_intact(f"quantize T={T} H={H}")
    return out, ws


def _assert_same(gpu: dict, ref: dict, what=""):
    for k in ("k_codes", "k_scales", "v_codes", "v_scales"):
        a, b = gpu[k], ref[k]
        if not np.array_equal(a, b):
            idx = np.argwhere(a != b)
            raise AssertionError(f"{what} {k}: {len(idx)} bytes differ, first at {idx[:4].tolist()}")
    assert np.array_equal(gpu["k_mean"].view(np.uint32), ref["k_mean"].view(np.uint32)), \
        f"{what} k_mean differs"
    assert np.float32(gpu["s_k"]) == np.float32(ref["s_k"]), f"{what} s_K"
    assert np.float32(gpu["s_v"]) == np.float32(ref["s_v"]), f"{what} s_V"


def test_tiny_config_bit_exact(lib, orc):
    ws = None
    for c in range(synth.TINY["chunks"]):
        K, V, _ = synth.tiny_chunk(c)
        out, ws = _gpu_quant(lib, K, V, ws)
        _assert_same(out.to_host(), orc.quantize_chunk(K, V), f"tiny chunk {c}")


@pytest.mark.parametrize("index", [0, 1, 9, 19, 33, 47, 58, 71, 86, 99])
def test_quantize_only_full_size_bit_exact(lib, orc, index):
    """Ten of the quantize-only workload's 100 chunks (seeds 1..100), spread
    over the range, bit-exact at full size."""
    K, V = synth.quant_chunk(index)
    out, _ = _gpu_quant(lib, K, V)
    _assert_same(out.to_host(), orc.quantize_chunk(K, V), f"quantize-only chunk {index}")


@pytest.mark.parametrize("T,H", [(1, 2), (48, 2), (63, 3), (65, 1), (136, 4), (200, 5), (1000, 6)])
def test_ragged_shapes_bit_exact(lib, orc, T, H):
    K = synth.k_with_offsets_bf16(31, T, H, (T, H, 128), outlier_mult=50.0)
    V = synth.gaussian_bf16(31, T, H, synth.T_V, (T, H, 128))
    out, _ = _gpu_quant(lib, K, V, guard=True)
    _assert_same(out.to_host(), orc.quantize_chunk(K, V), f"T={T} H={H}")


def test_degenerate_inputs_bit_exact(lib, orc):
    T, H = 100, 2
    zeros = np.zeros((T, H, 128), np.uint16)
    rng = np.random.default_rng(3)
    const = np.repeat(synth.to_bf16_bits(rng.standard_normal((1, H, 128)) * 3), T, axis=0)
    for K, V, what in ((zeros, zeros, "zeros"), (const, const, "constant channels"),
                       (const, zeros, "constant K, zero V")):
        out, _ = _gpu_quant(lib, K, V)
        _assert_same(out.to_host(), orc.quantize_chunk(K, V), what)


def _bf16_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_signed_zeros_subnormals_and_extreme_magnitudes_bit_exact(lib, orc):
    """Cases the fast division path must reproduce exactly: -0 inside blocks
    with a nonzero scale (the code keeps the sign), bf16 subnormals, whole
    tensors scaled to 2^-110 and 2^100, and single blocks scaled to 2^-110
    inside an ordinary tensor (their block max is below the fast-path bound)."""
    T, H = 200, 3
    rng = np.random.default_rng(11)
    K = synth.k_with_offsets_bf16(61, T, H, (T, H, 128))
    V = synth.gaussian_bf16(61, T, H, synth.T_V, (T, H, 128))
    cases = []
    # exact -0 in V, and a K channel of signed zeros: its mean is +0, so
    # RN(-0 - mean) = -0 reaches the encoder
    Vz = V.copy()
    Vz[rng.random(V.shape) < 0.05] = 0x8000
    Kz = K.copy()
    Kz[:, :, 5] = np.where(rng.random((T, H)) < 0.5, 0x8000, 0x0000).astype(np.uint16)
    cases.append((Kz, Vz, "signed zeros"))
    Vs = V.copy()
    m = rng.random(V.shape) < 0.03
    Vs[m] = (rng.integers(1, 0x80, m.sum()) | (rng.integers(0, 2, m.sum()) << 15)).astype(np.uint16)
    cases.append((K, Vs, "bf16 subnormals"))
    for e in (-110, 100):
        cases.append((synth.to_bf16_bits(_bf16_to_f64(K) * 2.0 ** e),
                      synth.to_bf16_bits(_bf16_to_f64(V) * 2.0 ** e), f"scaled by 2^{e}"))
    blocks = rng.random((T, H, 8)) < 0.02
    scale = np.where(np.repeat(blocks, 16, axis=2), 2.0 ** -110, 1.0)
    cases.append((synth.to_bf16_bits(_bf16_to_f64(K) * scale),
                  synth.to_bf16_bits(_bf16_to_f64(V) * scale), "tiny blocks"))
    for K_, V_, what in cases:
        out, _ = _gpu_quant(lib, K_, V_)
        _assert_same(out.to_host(), orc.quantize_chunk(K_, V_), what)


def test_repeated_calls_share_one_workspace(lib, orc):
    ws = None
    for i in range(3):
        K = synth.k_with_offsets_bf16(40 + i, 0, 0, (300, 4, 128))
        V = synth.gaussian_bf16(40 + i, 0, 0, synth.T_V, (300, 4, 128))
        out, ws = _gpu_quant(lib, K, V, ws)
        _assert_same(out.to_host(), orc.quantize_chunk(K, V), f"call {i}")


@pytest.mark.parametrize("bf16_out", [False, True])
def test_dequantize_bit_exact(lib, orc, bf16_out):
    import torch
    K, V, _ = synth.tiny_chunk(1)
    T, H, d = K.shape
    out, _ = _gpu_quant(lib, K, V)
    dt = torch.bfloat16 if bf16_out else torch.float32
    Kd = torch.empty((T, H, d), dtype=dt, device="cuda")
    Vd = torch.empty((T, H, d), dtype=dt, device="cuda")
    lib.dequantize(out, Kd, Vd)
    torch.cuda.synchronize()
    q = orc.quantize_chunk(K, V)
    Kr, Vr = orc.dequantize_chunk(q)
    if bf16_out:
        Kr, Vr = orc.f32_to_bf16(Kr), orc.f32_to_bf16(Vr)
        Kg = Kd.view(torch.int16).cpu().numpy().view(np.uint16)
        Vg = Vd.view(torch.int16).cpu().numpy().view(np.uint16)
    else:
        Kr, Vr = Kr.view(np.uint32), Vr.view(np.uint32)
        Kg = Kd.cpu().numpy().view(np.uint32)
        Vg = Vd.cpu().numpy().view(np.uint32)
    assert np.array_equal(Kg, Kr) and np.array_equal(Vg, Vr)


@pytest.mark.parametrize("T,H", [(1, 1), (13, 3), (200, 5), (37, 33), (64, 40), (9, 70)])
@pytest.mark.parametrize("bf16_out", [False, True])
def test_dequantize_ragged_tiles_bit_exact(lib, orc, T, H, bf16_out):
    """Token counts that leave a partial tile, head counts below a tile's
    width, across two and three head blocks."""
    import torch
    K = synth.k_with_offsets_bf16(57, T, H, (T, H, 128), outlier_mult=20.0)
    V = synth.gaussian_bf16(57, T, H, synth.T_V, (T, H, 128))
    out, _ = _gpu_quant(lib, K, V, guard=True)
    q = orc.quantize_chunk(K, V)
    _assert_same(out.to_host(), q, f"T={T} H={H}")
    dt = torch.bfloat16 if bf16_out else torch.float32
    gK, gV = Guarded((T, H, 128), dt), Guarded((T, H, 128), dt)
    Kd, Vd = gK.t, gV.t
    lib.dequantize(out, Kd, Vd)
    torch.cuda.synchronize()
    gK.assert_intact(f"de-quantized K T={T} H={H}")
    gV.assert_intact(f"de-quantized V T={T} H={H}")
    Kr = orc.dequantize_tensor(q["k_codes"], q["k_scales"], q["k_mean"], q["s_k"], T, H, 128)
    Vr = orc.dequantize_tensor(q["v_codes"], q["v_scales"], None, q["s_v"], T, H, 128)
    for name, got, want in (("K", Kd, Kr), ("V", Vd, Vr)):
        if bf16_out:
            g = got.view(torch.int16).cpu().numpy().view(np.uint16)
            w = orc.f32_to_bf16(want)
        else:
            g, w = got.cpu().numpy().view(np.uint32), want.view(np.uint32)
        assert np.array_equal(g, w), f"{name} T={T} H={H}"


def test_dequantize_rejects_mixed_or_short_outputs(lib):
    import torch
    K, V, _ = synth.tiny_chunk(1)
    T, H, d = K.shape
    out, _ = _gpu_quant(lib, K, V)
    Kd = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
    with pytest.raises(TypeError):
        lib.dequantize(out, Kd, torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        lib.dequantize(out, Kd, torch.empty((T - 1, H, d), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("which", ["K", "V"])
def test_dequantize_full_size_bit_exact(lib, orc, which):
    """One tensor at a time (the other output pointer NULL), full chunk size;
    K to fp32, V to bf16."""
    import torch
    K, V = synth.quant_chunk(2)
    T, H, d = K.shape
    out, _ = _gpu_quant(lib, K, V)
    q = orc.quantize_chunk(K, V)
    if which == "K":
        Kd = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
        lib.dequantize(out, K_out=Kd)
        torch.cuda.synchronize()
        Kr = orc.dequantize_tensor(q["k_codes"], q["k_scales"], q["k_mean"], q["s_k"], T, H, d)
        assert np.array_equal(Kd.cpu().numpy().view(np.uint32), Kr.view(np.uint32))
    else:
        Vd = torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda")
        lib.dequantize(out, V_out=Vd)
        torch.cuda.synchronize()
        Vr = orc.dequantize_tensor(q["v_codes"], q["v_scales"], None, q["s_v"], T, H, d)
        Vg = Vd.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(Vg, orc.f32_to_bf16(Vr))
