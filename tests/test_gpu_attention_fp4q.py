"""GPU attention with an FP4-operand Q K^T (nvfp4kv_attention_fp4q) against the
float64 oracle with the queries replaced by their NVFP4 reconstruction
(attention_f64_fp4q; "2605-LongLive2" DeepRead page, Method > 推理基础设施:
W4A4, FP4 GEMMs in place of BF16 ones).  The bar is the attention parity bar
(relative L2 <= 1e-2, max-abs <= 2e-2; bf16 outputs half a bf16 ulp more).

* the quantized queries the call leaves in its buffer: bit-exact with the
  oracle's activation quantizer;
* the tiny rollout through the cache, every chunk, every row;
* ragged shapes (one key, tails of the 96-key tile, a split last wave) with
  canaries around the output and the workspace;
* the rollout schedules at reduced shapes, every chunk, every row;
* one layer at full size (35,200 keys) and the 30-layer rollout's key sets at
  full size, sampled rows."""
import numpy as np
import pytest

import synth
from gpu_util import Guarded, assert_attention_close, dev_bf16, host_to_f64, sample_rows

pytestmark = pytest.mark.gpu


def _fp4q(lib, chunks, Q, ws, dtypes=None):
    """Run attention_fp4q for each output dtype: [(dtype, float64 output)]."""
    import torch
    dtypes = dtypes or (torch.float32, torch.bfloat16)
    T_q, H, _ = Q.shape
    qb = lib.Fp4QBuffer(T_q, H)
    outs = []
    for dt in dtypes:
        O = torch.empty((T_q, H, 128), dtype=dt, device="cuda")
        lib.attention_fp4q(chunks, dev_bf16(Q), O, qb, ws)
        torch.cuda.synchronize()
        assert lib.workspace_status(ws) == lib.OK
        outs.append((dt, host_to_f64(O)))
    return outs, qb


def _close(outs, ref, what, rows=None):
    import torch
    for dt, o in outs:
        if rows is not None:
            o = o[rows]
        assert_attention_close(o, ref, f"{what} ({dt})", bf16_output=dt == torch.bfloat16)


@pytest.mark.parametrize("T_q,H,zero", [(300, 2, False), (1, 1, False), (40, 3, True)])
def test_queries_quantized_bit_exact(lib, orc, T_q, H, zero):
    """The call's query buffer holds exactly the oracle's NVFP4 of Q (codes,
    block scales, tensor scale; all-zero queries: zero codes, scale 1)."""
    T_c = 48
    ws = lib.new_workspace(T_c, H)
    K = synth.k_with_offsets_bf16(70, 0, 0, (T_c, H, 128))
    V = synth.gaussian_bf16(70, 0, 0, synth.T_V, (T_c, H, 128))
    b = lib.ChunkBuffer(T_c, H)
    lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
    Q = synth.gaussian_bf16(71, 0, 0, synth.T_Q, (T_q, H, 128))
    if zero:
        Q = np.zeros_like(Q)
    _, qb = _fp4q(lib, [b], Q, ws)
    got = qb.to_host()
    want, _ = orc.quantize_queries(Q)
    assert np.array_equal(got["codes"], want["codes"])
    assert np.array_equal(got["scales"], want["scales"])
    assert np.float32(got["s"]).view(np.uint32) == np.float32(want["s"]).view(np.uint32)


def test_tiny_config_rollout(lib, orc):
    c = synth.TINY
    cache = lib.KVCache(1, c["H"], c["T_c"], c["S_g"], c["S_s"], c["W"])
    qs = []
    for n in range(c["chunks"]):
        K, V, Q = synth.tiny_chunk(n)
        cache.append(0, dev_bf16(K), dev_bf16(V))
        qs.append(orc.quantize_chunk(K, V))
        ids = cache.keyset(0)
        outs, _ = _fp4q(lib, [cache.chunk(0, i) for i in ids], Q, cache.ws)
        _close(outs, orc.attention_f64_fp4q([qs[i] for i in ids], Q), f"tiny chunk {n}")


@pytest.mark.parametrize("T_c,T_q,H", [(48, 100, 2), (96, 136, 3), (97, 257, 1), (200, 7, 2),
                                       (1, 5, 2), (191, 300, 2)])
def test_ragged_shapes(lib, orc, T_c, T_q, H):
    import torch
    chunks, qs = [], []
    gws = Guarded((lib.workspace_bytes(T_c, H),), torch.uint8)
    ws = gws.t
    lib.workspace_init(ws)
    for i in range(3):
        K = synth.k_with_offsets_bf16(80 + i, T_c, H, (T_c, H, 128))
        V = synth.gaussian_bf16(80 + i, T_c, H, synth.T_V, (T_c, H, 128))
        buf = lib.ChunkBuffer(T_c, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), buf, ws)
        chunks.append(buf)
        qs.append(orc.quantize_chunk(K, V))
    Q = synth.gaussian_bf16(88, T_c, H, synth.T_Q, (T_q, H, 128))
    ref = orc.attention_f64_fp4q(qs, Q)
    qb = lib.Fp4QBuffer(T_q, H)
    for dt in (torch.float32, torch.bfloat16):
        gO = Guarded((T_q, H, 128), dt)
        lib.attention_fp4q(chunks, dev_bf16(Q), gO.t, qb, ws)
        torch.cuda.synchronize()
        assert lib.workspace_status(ws) == lib.OK
        gO.assert_intact(f"O T_c={T_c} T_q={T_q} {dt}")
        gws.assert_intact(f"workspace T_c={T_c} T_q={T_q} {dt}")
        assert_attention_close(host_to_f64(gO.t), ref, f"T_c={T_c} T_q={T_q} {dt}",
                               bf16_output=dt == torch.bfloat16)


def test_split_last_wave(lib, orc):
    """Query rows for a few whole waves of query blocks plus a last wave of a
    few blocks, which are split over key ranges (three kernels: query
    quantizer, attention, merge)."""
    T_c, H, T_q = 200, 1, 149 * 256 - 100
    assert lib.attention_fp4q_launches(2, T_c, H, T_q) == 3
    ws = lib.new_workspace(T_c, H)
    bufs, qs = [], []
    for i in range(2):
        K = synth.k_with_offsets_bf16(92 + i, T_c, H, (T_c, H, 128))
        V = synth.gaussian_bf16(92 + i, T_c, H, synth.T_V, (T_c, H, 128))
        b = lib.ChunkBuffer(T_c, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
        bufs.append(b)
        qs.append(orc.quantize_chunk(K, V))
    Q = synth.gaussian_bf16(97, T_c, H, synth.T_Q, (T_q, H, 128))
    outs, _ = _fp4q(lib, bufs, Q, ws)
    rows = sorted(set(sample_rows(T_q, n_random=64, seed=5)) | set(range(148 * 256, T_q, 7)))
    _close(outs, orc.attention_f64_fp4q(qs, Q, rows=rows), "split last wave", rows=rows)


@pytest.mark.parametrize("cfg", [synth.ROLLOUT, synth.MULTISHOT], ids=["rollout", "multishot"])
def test_schedule_reduced_shapes(lib, orc, cfg):
    import torch
    layers, H, T_c = 2, 2, 200
    cache = lib.KVCache(layers, H, T_c, cfg["S_g"], cfg["S_s"], cfg["W"])
    switches = set(cfg["switches"])
    s_begin = 0
    quantized = [dict() for _ in range(layers)]
    for n in range(cfg["chunks"]):
        if n in switches:
            cache.rebind_shot_sink(n)
            s_begin = n
        for layer in range(layers):
            K, V, Q = synth.layer_chunk(cfg, layer, n, T_c=T_c, H=H)
            cache.append(layer, dev_bf16(K), dev_bf16(V))
            quantized[layer][n] = orc.quantize_chunk(K, V)
            ids = cache.keyset(layer)
            outs, _ = _fp4q(lib, [cache.chunk(layer, i) for i in ids], Q, cache.ws,
                            dtypes=None if n % 5 == 0 else (torch.float32,))
            want = orc.attention_f64_fp4q([quantized[layer][i] for i in ids], Q)
            _close(outs, want, f"{cfg['name']} layer {layer} chunk {n}")
            keep = set(ids) | {s_begin} | set(range(cfg["S_g"]))
            quantized[layer] = {i: q for i, q in quantized[layer].items() if i in keep}


def test_one_layer_attention_full_size(lib, orc):
    """Q [7040, 24, 128] over the global sink {0}, the shot sink {4} and the
    window {7, 8, 9}: 35,200 keys."""
    c = synth.ATTN
    cache = lib.KVCache(1, c["H"], c["T_c"], c["S_g"], c["S_s"], c["W"])
    want_ids = [0, 4, 7, 8, 9]
    qs = {}
    for n in range(c["appended"]):
        if n == c["shot_start"]:
            cache.rebind_shot_sink(n)
        K, V, Q = synth.layer_chunk(c, 0, n)
        cache.append(0, dev_bf16(K), dev_bf16(V))
        if n in want_ids:
            qs[n] = orc.quantize_chunk(K, V)
    assert cache.keyset(0) == want_ids
    outs, qb = _fp4q(lib, [cache.chunk(0, i) for i in want_ids], Q, cache.ws)
    want, _ = orc.quantize_queries(Q)
    got = qb.to_host()
    assert np.array_equal(got["codes"], want["codes"]) and np.array_equal(got["scales"],
                                                                         want["scales"])
    rows = sample_rows(c["T_c"], n_random=24, seed=2)
    ref = orc.attention_f64_fp4q([qs[i] for i in want_ids], Q, rows=rows)
    _close(outs, ref, "one-layer attention", rows=rows)


def test_rollout_key_sets_full_size(lib, orc):
    """Layer 0 of the 30-layer rollout (W = 4, the shot sink on chunk 0) at
    full size: the key sets of chunks 0, 1 and 5 (1, 2 and 5 chunks)."""
    import torch
    cfg = synth.ROLLOUT
    T_c, H = cfg["T_c"], cfg["H"]
    cache = lib.KVCache(1, H, T_c, cfg["S_g"], cfg["S_s"], cfg["W"])
    quantized = {}
    for n in range(6):
        K, V, Q = synth.layer_chunk(cfg, 0, n)
        cache.append(0, dev_bf16(K), dev_bf16(V))
        quantized[n] = orc.quantize_chunk(K, V)
        ids = cache.keyset(0)
        if n in (0, 1, 5):
            outs, _ = _fp4q(lib, [cache.chunk(0, i) for i in ids], Q, cache.ws,
                            dtypes=(torch.float32,))
            rows = sample_rows(T_c, n_random=8, seed=n)
            want = orc.attention_f64_fp4q([quantized[i] for i in ids], Q, rows=rows)
            _close(outs, want, f"rollout chunk {n}, key set {ids}", rows=rows)
