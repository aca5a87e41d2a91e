"""Rollout parity: the whole streaming schedule of the 30-layer rollout and of
the multi-shot long stream (sinks, window, shot switches re-binding A_s,
de-duplication when A_s overlaps the window) run through the cache on the GPU
and compared with the oracle.

* Reduced shapes (2 layers, 2 heads, 200-token chunks: one full 128-key tile
  and a ragged tail), every chunk of the schedule: key sets equal, codes and
  scales bit-exact on every (layer, chunk), attention on every query row
  within the parity bar.
* Full size (7040 x 24 x 128), one layer of the multi-shot stream through its
  first two shot switches: key sets at every chunk, quantization bit-exact and
  attention on sampled rows at checkpoints around the switches."""
import numpy as np
import pytest

import synth
from gpu_util import assert_attention_close, dev_bf16, sample_rows

pytestmark = pytest.mark.gpu


def _expected_keyset(orc, n, cfg, s_begin):
    return orc.keyset(n, cfg["S_g"], cfg["S_s"], cfg["W"], s_begin)


def _attend(lib, cache, layer, Q):
    import torch
    O = torch.empty(Q.shape, dtype=torch.float32, device="cuda")
    cache.attention(layer, dev_bf16(Q), O)
    torch.cuda.synchronize()
    assert cache.check_status() == lib.OK
    return O.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("cfg", [synth.ROLLOUT, synth.MULTISHOT], ids=["rollout", "multishot"])
def test_schedule_reduced_shapes(lib, orc, cfg):
    layers, H, T_c = 2, 2, 200
    cache = lib.KVCache(layers, H, T_c, cfg["S_g"], cfg["S_s"], cfg["W"])
    switches = set(cfg["switches"])
    s_begin = 0
    quantized = [dict() for _ in range(layers)]
    dedup_seen = False
    for n in range(cfg["chunks"]):
        if n in switches:
            cache.rebind_shot_sink(n)
            s_begin = n
        for layer in range(layers):
            K, V, Q = synth.layer_chunk(cfg, layer, n, T_c=T_c, H=H)
            cache.append(layer, dev_bf16(K), dev_bf16(V))
            ref = orc.quantize_chunk(K, V)
            quantized[layer][n] = ref
            got = cache.chunk(layer, n).to_host()
            for k in ("k_codes", "k_scales", "v_codes", "v_scales"):
                assert np.array_equal(got[k], ref[k]), f"{cfg['name']} layer {layer} chunk {n} {k}"
            assert np.array_equal(got["k_mean"].view(np.uint32), ref["k_mean"].view(np.uint32))
            ids = cache.keyset(layer)
            assert ids == _expected_keyset(orc, n + 1, cfg, s_begin), f"chunk {n}"
            union = cfg["S_g"] + cfg["S_s"] + min(cfg["W"], n + 1)
            dedup_seen |= len(ids) < min(union, n + 1)
            out = _attend(lib, cache, layer, Q)
            want = orc.attention_f64([quantized[layer][i] for i in ids], Q)
            assert_attention_close(out, want, f"{cfg['name']} layer {layer} chunk {n}")
            # chunks no key set can reach again are dropped from the host copy
            keep = set(ids) | {s_begin} | set(range(cfg["S_g"]))
            quantized[layer] = {i: q for i, q in quantized[layer].items() if i in keep}
    assert dedup_seen, "the schedule never de-duplicated a sink against the window"


def test_multishot_full_size_through_two_switches(lib, orc):
    cfg = synth.MULTISHOT
    T_c, H = cfg["T_c"], cfg["H"]
    last = 30                                   # chunks 0..30: switches at 12 and 28
    checkpoints = {0, 12, 13, 16, 28, 30}
    switches = {s for s in cfg["switches"] if s <= last}
    # chunks that some checkpoint's key set reads: sinks and the W before each
    needed = set(range(cfg["S_g"])) | switches
    for c in checkpoints:
        needed |= set(range(max(0, c - cfg["W"] + 1), c + 1))
    cache = lib.KVCache(1, H, T_c, cfg["S_g"], cfg["S_s"], cfg["W"])
    s_begin = 0
    quantized = {}
    for n in range(last + 1):
        if n in switches:
            cache.rebind_shot_sink(n)
            s_begin = n
        K, V, Q = synth.layer_chunk(cfg, 0, n)
        cache.append(0, dev_bf16(K), dev_bf16(V))
        ids = cache.keyset(0)
        assert ids == _expected_keyset(orc, n + 1, cfg, s_begin), f"chunk {n}"
        if n in needed:
            quantized[n] = orc.quantize_chunk(K, V)
        if n in checkpoints:
            got = cache.chunk(0, n).to_host()
            for k in ("k_codes", "k_scales", "v_codes", "v_scales"):
                assert np.array_equal(got[k], quantized[n][k]), f"chunk {n} {k}"
            out = _attend(lib, cache, 0, Q)
            rows = sample_rows(T_c, n_random=8, seed=n)
            want = orc.attention_f64([quantized[i] for i in ids], Q, rows=rows)
            assert_attention_close(out[rows], want, f"full-size chunk {n}, key set {ids}")
