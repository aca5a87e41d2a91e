"""GPU parity of the 3D rotary position embedding with the multi-shot frame
offset (the txtmix page "LongLive 2.0：给长视频生成补上 NVFP4 并行基础设施" names a
fused RoPE kernel, section NVFP4, and multi_shot_rope_offset, section 多 shot
一致性; the rotary form is the reading stated at oracle.c's oracle_rope, pinned
to rotation properties in test_oracle_rope.py, unpinned against the pages).

* The cos/sin table, every entry bit-exact against the oracle's fp32 values.
* The rotation of queries, bit-exact, at the layer shape, ragged shapes and in
  place, with guard bytes around the output.
* The chunk quantizer with the rotation fused into its reads of K, bit-exact
  against the oracle's quantization of the oracle's rotated K, and equal to the
  unfused composition (rotate, then quantize) on the GPU.
* A multi-shot stream through the cache (kvcache_append_rope), frame positions
  from the shot offset: quantized chunks bit-exact, attention of the rotated
  queries over the rotated keys within the parity bar."""
import numpy as np
import pytest

import synth
from gpu_util import Guarded, assert_attention_close, dev_bf16

pytestmark = pytest.mark.gpu

ROWS, COLS = 22, 40                     # 880 latent tokens per frame, 8 frames per chunk


def expected_table(orc, p0, frames, rows, cols):
    ent = [(p0 + f, i, 44) for f in range(frames) for i in range(22)]
    ent += [(r, i, 42) for r in range(rows) for i in range(21)]
    ent += [(c, i, 42) for c in range(cols) for i in range(21)]
    return np.array([orc.rope_cos_sin(p, i, w) for p, i, w in ent], np.float32)


@pytest.mark.parametrize("p0,frames,rows,cols", [
    (0, 8, ROWS, COLS), (72, 8, ROWS, COLS), (2040, 8, ROWS, COLS), (1_000_003, 3, 3, 5),
    (5, 1, 1, 1)])
def test_table_bit_exact(lib, orc, p0, frames, rows, cols):
    import torch
    tab = lib.RopeTable(frames, rows, cols).fill(p0)
    torch.cuda.synchronize()
    got = tab.table.cpu().numpy().reshape(-1, 2)
    want = expected_table(orc, p0, frames, rows, cols)
    assert got.shape == want.shape
    bad = np.nonzero((got.view(np.uint32) != want.view(np.uint32)).any(axis=1))[0]
    assert bad.size == 0, f"entries {bad[:8]} differ: {got[bad[:4]]} vs {want[bad[:4]]}"


def _x(seed, T, H):
    return synth.gaussian_bf16(seed, 0, 0, 2, (T, H, 128))


@pytest.mark.parametrize("T,H,p0,frames", [(7040, 24, 72, 8), (1000, 3, 5, 2), (100, 2, 0, 1),
                                           (881, 1, 2040, 2)])
def test_rope_bit_exact(lib, orc, T, H, p0, frames):
    import torch
    X = _x(T, T, H)
    tab = lib.RopeTable(frames, ROWS, COLS).fill(p0)
    want = orc.rope(X, p0, ROWS, COLS)
    out = Guarded((T, H, 128), torch.bfloat16)
    Xd = dev_bf16(X)
    lib.rope(Xd, tab, Y=out.t)
    torch.cuda.synchronize()
    got = out.t.cpu().view(torch.int16).numpy().view(np.uint16)
    _assert_bits_equal(got, want, f"rope T={T} H={H}")
    out.assert_intact("rope output")
    lib.rope(Xd, tab, Y=Xd)                        # in place
    torch.cuda.synchronize()
    _assert_bits_equal(Xd.cpu().view(torch.int16).numpy().view(np.uint16), want,
                       f"rope in place T={T} H={H}")


def _assert_bits_equal(got, want, what):
    bad = np.argwhere(got != want)
    if bad.size:
        t, h, c = bad[0]
        raise AssertionError(
            f"{what}: {len(bad)} of {got.size} elements differ; first at token {t}, head {h}, "
            f"channel {c}: got {got[t, h, c]:#06x}, want {want[t, h, c]:#06x}; "
            f"tokens {np.unique(bad[:, 0])[:8]}, channels {np.unique(bad[:, 2])[:16]}")


def _assert_chunk_equal(got, ref, what):
    for k in ("k_codes", "k_scales", "v_codes", "v_scales"):
        assert np.array_equal(got[k], ref[k]), f"{what}: {k}"
    assert np.array_equal(np.asarray(got["k_mean"]).view(np.uint32),
                          np.asarray(ref["k_mean"]).view(np.uint32)), f"{what}: k_mean"
    assert np.float32(got["s_k"]).view(np.uint32) == np.float32(ref["s_k"]).view(np.uint32)
    assert np.float32(got["s_v"]).view(np.uint32) == np.float32(ref["s_v"]).view(np.uint32)


@pytest.mark.parametrize("T,H,p0,frames", [(7040, 24, 72, 8), (1000, 3, 5, 2), (100, 2, 0, 1)])
def test_quantize_chunk_rope_bit_exact(lib, orc, T, H, p0, frames):
    import torch
    K, V = synth.quant_chunk(T % 97, T_c=T, H=H)
    tab = lib.RopeTable(frames, ROWS, COLS).fill(p0)
    ref = orc.quantize_chunk(orc.rope(K, p0, ROWS, COLS), V)
    ws = lib.new_workspace(T, H)
    out = lib.ChunkBuffer(T, H)
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    lib.quantize_chunk_rope(Kd, Vd, tab, out, ws)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    _assert_chunk_equal(out.to_host(), ref, f"fused T={T} H={H}")
    # the unfused composition on the GPU gives the same bytes
    out2 = lib.ChunkBuffer(T, H)
    lib.quantize_chunk(lib.rope(Kd, tab), Vd, out2, ws)
    torch.cuda.synchronize()
    _assert_chunk_equal(out2.to_host(), ref, f"unfused T={T} H={H}")


def test_multishot_stream_through_the_cache(lib, orc):
    """Chunks of 2 frames of 4 x 8 tokens, two heads; shots switch at chunks 5
    and 9 with multi_shot_rope_offset 100, so a chunk of shot s starts at frame
    2 n + 100 s.  Every chunk: the rotated keys' quantization bit-exact, the
    rotated queries bit-exact, and the attention over K_eff within the bar."""
    import torch
    cfg = dict(synth.MULTISHOT, S_g=1, S_s=1, W=3)
    rows, cols, F, H, offset = 4, 8, 2, 2, 100
    T_c = F * rows * cols
    switches = {5, 9}
    cache = lib.KVCache(1, H, T_c, cfg["S_g"], cfg["S_s"], cfg["W"])
    tab = lib.RopeTable(F, rows, cols)
    shot, s_begin = 0, 0
    stored = {}
    for n in range(13):
        if n in switches:
            cache.rebind_shot_sink(n)
            shot += 1
            s_begin = n
        p0 = lib.rope_frame_position(n, F, shot, offset)
        assert p0 == orc.rope_frame_position(n, F, shot, offset)
        tab.fill(p0)
        K, V, Q = synth.layer_chunk(cfg, 0, n, T_c=T_c, H=H)
        cache.append_rope(0, dev_bf16(K), dev_bf16(V), tab)
        Qr = lib.rope(dev_bf16(Q), tab)
        Qr_ref = orc.rope(Q, p0, rows, cols)
        stored[n] = orc.quantize_chunk(orc.rope(K, p0, rows, cols), V)
        torch.cuda.synchronize()
        _assert_bits_equal(Qr.cpu().view(torch.int16).numpy().view(np.uint16), Qr_ref,
                           f"queries of chunk {n}")
        got = cache.chunk(0, n).to_host()
        for k in ("k_codes", "k_scales", "v_codes", "v_scales"):
            assert np.array_equal(got[k], stored[n][k]), f"chunk {n} {k}"
        ids = cache.keyset(0)
        assert ids == orc.keyset(n + 1, cfg["S_g"], cfg["S_s"], cfg["W"], s_begin)
        O = torch.empty((T_c, H, 128), dtype=torch.float32, device="cuda")
        cache.attention(0, Qr, O)
        torch.cuda.synchronize()
        assert cache.check_status() == lib.OK
        want = orc.attention_f64([stored[i] for i in ids], Qr_ref)
        assert_attention_close(O.cpu().numpy().astype(np.float64), want, f"chunk {n}")
