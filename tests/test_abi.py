"""The C-ABI library on the host (no GPU work): it loads, exports every
symbol include/nvfp4kv.h declares, lays chunks out in (9/8)*T*H*d payload
bytes, rejects bad arguments before touching a device, and its cache
bookkeeping (slot pool, eviction, shot-sink rebinding) keeps exactly the key
set of the oracle.  Pointers passed here are never dereferenced: every call
either does host bookkeeping only or fails validation first."""
import ctypes
import os
import random
import re
import subprocess
import sys

import pytest

import sink_window_video_b200 as swv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4kv.h")
FAKE = 0x7F0000000000      # 256-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(swv.LIB_PATH):
        from sink_window_video_b200 import build
        build.build()
    return swv.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted({n for n in names if n not in ("if", "defined")})


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", swv.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing


def test_chunk_layout_holds_the_payload(L):
    for T, H in [(7040, 24), (32, 2), (48, 3)]:
        n = T * H * 128
        cb = swv.chunk_bytes(T, H)
        assert cb % 256 == 0 and cb >= n * 9 // 8 + H * 128 * 4 + 8
        assert cb - (n * 9 // 8 + H * 128 * 4 + 8) < 6 * 256
        v = swv.chunk_view_init(FAKE, T, H)
        parts = sorted([(v.k_codes, n // 2), (v.v_codes, n // 2), (v.k_scales, n // 16),
                        (v.v_scales, n // 16), (v.k_mean, H * 128 * 4), (v.tensor_scales, 8)])
        for (a, na), (b, _) in zip(parts, parts[1:]):
            assert a + na <= b                       # no overlap
        assert parts[-1][0] + parts[-1][1] <= FAKE + cb
        assert all(p % 16 == 0 for p, _ in parts)
    assert swv.chunk_bytes(0, 2) == 0 and swv.chunk_bytes(32, 2, 100) == 0


def test_rejects_bad_arguments_without_device_work(L):
    cv = swv.ChunkView(FAKE, FAKE + 4096, FAKE + 8192, FAKE + 12288, FAKE + 16384, FAKE + 20480)
    q = L.nvfp4kv_quantize_chunk
    assert q(None, FAKE, 32, 2, 128, ctypes.byref(cv), FAKE, None) == swv.ERR_INVALID_ARG
    assert q(FAKE, FAKE, 0, 2, 128, ctypes.byref(cv), FAKE, None) == swv.ERR_INVALID_ARG
    assert q(FAKE, FAKE, 32, 2, 64, ctypes.byref(cv), FAKE, None) == swv.ERR_UNSUPPORTED
    assert q(FAKE + 8, FAKE, 32, 2, 128, ctypes.byref(cv), FAKE, None) == swv.ERR_ALIGNMENT
    assert q(FAKE, FAKE, 32, 2, 128, ctypes.byref(cv), FAKE + 16, None) == swv.ERR_ALIGNMENT
    a = L.nvfp4kv_attention
    arr = (swv.ChunkView * 1)(cv)
    assert a(arr, 0, 32, 2, 128, FAKE, 32, FAKE, 1, 0.0, FAKE, None) == swv.ERR_EMPTY_KEYSET
    assert a(arr, 33, 32, 2, 128, FAKE, 32, FAKE, 1, 0.0, FAKE, None) == swv.ERR_CAPACITY
    assert a(arr, 1, 32, 2, 128, FAKE + 4, 32, FAKE, 1, 0.0, FAKE, None) == swv.ERR_ALIGNMENT
    assert a(arr, 1, 32, 2, 96, FAKE, 32, FAKE, 1, 0.0, FAKE, None) == swv.ERR_UNSUPPORTED
    assert a(arr, 1, 32, 2, 128, FAKE, 32, FAKE, 7, 0.0, FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_check_formats(9, FAKE, FAKE, 1, None) == swv.ERR_INVALID_ARG
    m = L.nvfp4kv_quantize_matrix
    assert m(None, 16, 32, 1, FAKE, FAKE, FAKE, FAKE, None) == swv.ERR_INVALID_ARG
    assert m(FAKE, 16, 32, 3, FAKE, FAKE, FAKE, FAKE, None) == swv.ERR_INVALID_ARG
    assert m(FAKE, 16, 40, 1, FAKE, FAKE, FAKE, FAKE, None) == swv.ERR_UNSUPPORTED
    assert m(FAKE, 24, 32, 2, FAKE, FAKE, FAKE, FAKE, None) == swv.ERR_UNSUPPORTED
    assert m(FAKE + 8, 16, 32, 2, FAKE, FAKE, FAKE, FAKE, None) == swv.ERR_ALIGNMENT
    assert L.nvfp4kv_matrix_workspace_bytes() >= 256
    assert L.nvfp4kv_chunk_stats(None, FAKE, 64, 2, 128, FAKE, FAKE, FAKE, FAKE, FAKE, None) \
        == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_chunk_stats(FAKE, FAKE, 64, 2, 96, FAKE, FAKE, FAKE, FAKE, FAKE, None) \
        == swv.ERR_UNSUPPORTED
    assert L.nvfp4kv_chunk_finalize(FAKE, FAKE, FAKE, 3, 200, 2, 128, FAKE, FAKE, FAKE, FAKE,
                                    None) == swv.ERR_INVALID_ARG           # 200 tokens: 4 segments
    assert L.nvfp4kv_chunk_encode(FAKE, FAKE, 64, 2, 128, FAKE, FAKE, None, None) \
        == swv.ERR_INVALID_ARG
    a = L.nvfp4kv_chunk_amax
    assert a(FAKE, FAKE, FAKE, 3, 200, 2, 128, FAKE, FAKE, FAKE, FAKE, None) \
        == swv.ERR_INVALID_ARG                                            # 200 tokens: 4 segments
    assert a(FAKE, FAKE, FAKE, 4, 200, 2, 128, FAKE, FAKE, None, FAKE, None) \
        == swv.ERR_INVALID_ARG                                            # no amax output
    assert a(FAKE, FAKE, FAKE, 4, 200, 2, 96, FAKE, FAKE, FAKE, FAKE, None) == swv.ERR_UNSUPPORTED
    assert a(FAKE, FAKE, FAKE, 4, 200, 2, 128, FAKE, FAKE, FAKE, FAKE + 16, None) \
        == swv.ERR_ALIGNMENT                                              # workspace not 256-aligned
    assert L.nvfp4kv_tensor_scales_from_amax(None, FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_tensor_scales_from_amax(FAKE, None, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_workspace_init(None, 256, None) == swv.ERR_INVALID_ARG


def test_fp4q_entry_checks_and_layout(L):
    """nvfp4kv_attention_fp4q rejects what nvfp4kv_attention rejects, plus a
    missing or misaligned query buffer; the buffer size follows the stated
    layout (codes, scales, each rounded up to 256 bytes, then the scale)."""
    cv = swv.ChunkView(FAKE, FAKE + 4096, FAKE + 8192, FAKE + 12288, FAKE + 16384, FAKE + 20480)
    arr = (swv.ChunkView * 1)(cv)
    f = L.nvfp4kv_attention_fp4q
    ok = (arr, 1, 32, 2, 128, FAKE, 32, FAKE, 1, 0.0, FAKE, FAKE, None)

    def call(**kw):
        args = list(ok)
        for i, v in kw.items():
            args[int(i[1:])] = v
        return f(*args)
    assert call(a1=0) == swv.ERR_EMPTY_KEYSET
    assert call(a1=33) == swv.ERR_CAPACITY
    assert call(a10=None) == swv.ERR_INVALID_ARG          # no query buffer
    assert call(a11=None) == swv.ERR_INVALID_ARG          # no workspace
    assert call(a8=7) == swv.ERR_INVALID_ARG              # output dtype
    assert call(a6=0) == swv.ERR_INVALID_ARG              # T_q = 0
    assert call(a4=96) == swv.ERR_UNSUPPORTED
    assert call(a10=FAKE + 16) == swv.ERR_ALIGNMENT
    assert call(a5=FAKE + 4) == swv.ERR_ALIGNMENT
    up = lambda x: (x + 255) // 256 * 256
    for T_q, H in [(1, 1), (300, 2), (7040, 24)]:
        R = T_q * H
        assert swv.fp4q_bytes(T_q, H) == up(R * 64) + up(R * 8) + 256
    assert swv.fp4q_bytes(0, 2) == 0 and swv.fp4q_bytes(32, 2, 64) == 0
    assert L.nvfp4kv_attention_fp4q_launches(0, 32, 2, 128, 32) == 0
    assert L.nvfp4kv_attention_fp4q_launches(1, 32, 2, 96, 32) == 0


def _cache(L, layers, S_g, S_s, W, T=32, H=2):
    cfg = swv.KVCacheConfig(layers, H, 128, T, S_g, S_s, W)
    h = ctypes.c_void_p()
    assert L.kvcache_create(ctypes.byref(cfg), FAKE, FAKE, ctypes.byref(h)) == swv.OK
    return h, cfg


def _keyset(L, h, layer):
    ids = (ctypes.c_int64 * 64)()
    n = ctypes.c_int()
    assert L.kvcache_keyset(h, layer, ids, ctypes.byref(n)) == swv.OK
    return [ids[i] for i in range(n.value)]


def test_cache_bookkeeping_matches_oracle_keyset(L, orc):
    rng = random.Random(3)
    for trial in range(60):
        S_g, S_s, W = rng.randint(0, 3), rng.randint(0, 3), rng.randint(0, 5)
        if S_g + S_s + W == 0:
            W = 1
        layers = rng.randint(1, 3)
        h, cfg = _cache(L, layers, S_g, S_s, W)
        slots = S_g + S_s + W
        cb = swv.chunk_bytes(32, 2)
        pool_end = FAKE + swv.load().kvcache_pool_bytes(ctypes.byref(cfg))
        s_begin = 0
        n = [0] * layers
        for step in range(rng.randint(5, 40)):
            if rng.random() < 0.15:
                # the next shot starts at or after the newest chunk of every layer
                s_begin = max(n) + rng.randint(0, 2)
                assert L.kvcache_rebind_shot_sink(h, s_begin) == swv.OK
            if rng.random() < 0.1 and S_s > 0:
                # a shot sink on past chunks is accepted only if every layer that
                # appended them still stores them; otherwise refused, state kept
                stale = rng.randint(0, max(n))
                cv = swv.ChunkView()
                ok = all(L.kvcache_chunk_view(h, ly, c, ctypes.byref(cv)) == swv.OK
                         for ly in range(layers)
                         for c in range(stale, min(stale + S_s, n[ly])))
                st = L.kvcache_rebind_shot_sink(h, stale)
                assert st == (swv.OK if ok else swv.ERR_INVALID_ARG)
                if ok:
                    s_begin = stale
            layer = rng.randrange(layers)
            v = swv.ChunkView()
            assert L.kvcache_advance(h, layer, ctypes.byref(v)) == swv.OK
            n[layer] += 1
            ids = _keyset(L, h, layer)
            assert ids == orc.keyset(n[layer], S_g, S_s, W, s_begin)
            stored = []
            for c in range(n[layer]):
                cv = swv.ChunkView()
                st = L.kvcache_chunk_view(h, layer, c, ctypes.byref(cv))
                if st == swv.OK:
                    stored.append((c, cv.k_codes))
            # every attended chunk is stored; nothing else is kept past its use
            live_next = set(orc.keyset(n[layer] + 1, S_g, S_s, W, s_begin)) | set(ids)
            assert set(ids) <= {c for c, _ in stored}
            assert {c for c, _ in stored} <= live_next
            assert len(stored) <= slots
            addrs = [a for _, a in stored]
            assert len(set(addrs)) == len(addrs)
            assert all(FAKE <= a < pool_end for a in addrs)
            assert all((a - FAKE) % cb == 0 for a in addrs)
            cnt = ctypes.c_int64()
            assert L.kvcache_num_chunks(h, layer, ctypes.byref(cnt)) == swv.OK
            assert cnt.value == n[layer]
        L.kvcache_destroy(h)


def test_cache_rejects_bad_layers_and_sizes(L):
    h, _ = _cache(L, 2, 1, 1, 2)
    v = swv.ChunkView()
    assert L.kvcache_advance(h, 2, ctypes.byref(v)) == swv.ERR_CAPACITY
    assert L.kvcache_advance(h, -1, ctypes.byref(v)) == swv.ERR_CAPACITY
    assert L.kvcache_rebind_shot_sink(h, -3) == swv.ERR_INVALID_ARG
    # no chunk yet: nothing to attend, reported before any launch
    assert L.sink_window_attention(h, 0, FAKE, 32, FAKE, 1, 0.0, None) == swv.ERR_EMPTY_KEYSET
    L.kvcache_destroy(h)
    cfg = swv.KVCacheConfig(1, 2, 128, 32, 20, 10, 10)
    hh = ctypes.c_void_p()
    assert L.kvcache_create(ctypes.byref(cfg), FAKE, FAKE, ctypes.byref(hh)) == swv.ERR_CAPACITY


def test_binding_fails_loudly_without_library(tmp_path):
    code = ("import sink_window_video_b200 as s; s.LIB_PATH = '/nonexistent/libnvfp4kv.so'\n"
            "try:\n    s.load()\nexcept ImportError as e:\n    print('LOUD', e)\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert "LOUD" in r.stdout


def test_noalloc_refuses_every_bad_argument_as_the_workspace_entry_point(L):
    """nvfp4kv_quantize_chunk_noalloc runs nvfp4kv_quantize_chunk's argument
    checks in its order: each bad argument gets the same status from both
    (nothing reaches the device)."""
    good = swv.chunk_view_init(FAKE, 64, 2)

    def view(**kw):
        v = swv.ChunkView(good.k_codes, good.k_scales, good.v_codes, good.v_scales,
                          good.k_mean, good.tensor_scales)
        for k, x in kw.items():
            setattr(v, k, x)
        return v

    K = V = FAKE + (1 << 24)
    cases = [
        dict(K=0), dict(V=0), dict(out=None),
        dict(T=0), dict(H=0), dict(d=0), dict(d=24), dict(d=64), dict(T=(1 << 24) + 1),
        dict(H=4097), dict(K=K + 8), dict(V=V + 2),
        dict(out=view(k_codes=good.k_codes + 8)), dict(out=view(v_scales=good.v_scales + 4)),
        dict(out=view(k_mean=0)), dict(out=view(tensor_scales=good.tensor_scales + 4)),
        dict(d=64, K=K + 8), dict(d=24, K=0),
    ]
    for c in cases:
        a = dict(K=K, V=V, T=64, H=2, d=128, out=good)
        a.update(c)
        out = ctypes.byref(a["out"]) if a["out"] is not None else None
        ws_status = L.nvfp4kv_quantize_chunk(a["K"], a["V"], a["T"], a["H"], a["d"], out,
                                             FAKE, None)
        na_status = L.nvfp4kv_quantize_chunk_noalloc(a["K"], a["V"], a["T"], a["H"], a["d"],
                                                     out, None)
        assert ws_status != swv.OK and na_status == ws_status, (c, ws_status, na_status)


def _views(L, h, layers):
    out = []
    for layer in range(layers):
        ids = _keyset(L, h, layer)
        n = ctypes.c_int64()
        assert L.kvcache_num_chunks(h, layer, ctypes.byref(n)) == swv.OK
        vs = []
        for c in ids:
            v = swv.ChunkView()
            assert L.kvcache_chunk_view(h, layer, c, ctypes.byref(v)) == swv.OK
            vs.append((c, v.k_codes, v.v_codes, v.k_scales, v.v_scales, v.k_mean, v.tensor_scales))
        out.append((n.value, ids, vs))
    return out


def _state(L, h):
    n = L.kvcache_state_bytes(h)
    buf = ctypes.create_string_buffer(n)
    assert L.kvcache_get_state(h, buf, n) == swv.OK
    return bytearray(buf.raw)


def _set(L, h, state):
    buf = ctypes.create_string_buffer(bytes(state), len(state))
    return L.kvcache_set_state(h, buf, len(state))


def test_cache_state_round_trip(L):
    """kvcache_get_state / kvcache_set_state: a second cache over the same pool,
    given the first one's state at random points of a schedule with shot
    switches, holds the same chunks in the same slots, and both evolve alike
    afterwards."""
    rng = random.Random(11)
    for trial in range(20):
        layers = rng.randint(1, 3)
        S_g, S_s, W = rng.randint(0, 2), rng.randint(0, 2), rng.randint(1, 4)
        h1, cfg = _cache(L, layers, S_g, S_s, W)
        h2, _ = _cache(L, layers, S_g, S_s, W)
        assert L.kvcache_state_bytes(h1) == 44 + 8 * layers * (1 + max(1, S_g + S_s + W))
        n = [0] * layers
        for step in range(rng.randint(3, 25)):
            if rng.random() < 0.2 and step > 0:
                first = max(n)
                assert L.kvcache_rebind_shot_sink(h1, first) == swv.OK
                assert L.kvcache_rebind_shot_sink(h2, first) == swv.OK
            layer = rng.randrange(layers)
            v1, v2 = swv.ChunkView(), swv.ChunkView()
            assert L.kvcache_advance(h1, layer, ctypes.byref(v1)) == swv.OK
            assert L.kvcache_advance(h2, layer, ctypes.byref(v2)) == swv.OK
            n[layer] += 1
            if rng.random() < 0.3:
                assert _set(L, h2, _state(L, h1)) == swv.OK
                assert _views(L, h2, layers) == _views(L, h1, layers)
                assert _state(L, h2) == _state(L, h1)
        assert _views(L, h2, layers) == _views(L, h1, layers)
        L.kvcache_destroy(h1)
        L.kvcache_destroy(h2)


def test_cache_state_refusals_change_nothing(L):
    h, cfg = _cache(L, 2, 1, 1, 3)
    for layer in (0, 1, 0, 0):
        v = swv.ChunkView()
        assert L.kvcache_advance(h, layer, ctypes.byref(v)) == swv.OK
    good = _state(L, h)
    other, _ = _cache(L, 2, 1, 1, 4)
    slots = 5
    n_off, s_off = 44, 44 + 16                 # counts of 2 layers, then the slot map

    def put64(st, off, v):
        st[off:off + 8] = int(v).to_bytes(8, "little", signed=True)

    bad = []
    bad.append(good[:-1])                                       # short
    b = bytearray(good); b[0:4] = b"NVKX"; bad.append(b)        # not this format
    b = bytearray(good); b[4] = 2; bad.append(b)                # another version
    b = bytearray(good); b[8 + 6 * 4] = 9; bad.append(b)        # another window
    b = bytearray(good); put64(b, n_off, -1); bad.append(b)     # negative count
    b = bytearray(good); put64(b, 36, -3); bad.append(b)        # negative shot sink
    b = bytearray(good); put64(b, s_off, 7); bad.append(b)      # a chunk never appended
    b = bytearray(good)
    put64(b, s_off, 1); put64(b, s_off + 8, 1); bad.append(b)   # one chunk in two slots
    before = _views(L, h, 2)
    for st in bad:
        assert _set(L, h, st) == swv.ERR_INVALID_ARG
        assert _state(L, h) == good and _views(L, h, 2) == before
    assert _set(L, other, good) == swv.ERR_INVALID_ARG          # another configuration
    assert _set(L, h, good) == swv.OK
    L.kvcache_destroy(h)
    L.kvcache_destroy(other)


def test_rope_entry_points_refuse_bad_arguments(L):
    """The rotary embedding's host checks, before any device work."""
    assert L.nvfp4kv_rope_frame_position(5, 8, 2, 1000) == 40 + 2000
    assert L.nvfp4kv_rope_frame_position(3, 8, 0, 0) == 24
    for bad in [(-1, 8, 0, 0), (1, 0, 0, 0), (1, 8, -1, 0), (1, 8, 0, -5)]:
        assert L.nvfp4kv_rope_frame_position(*bad) == -1
    assert L.nvfp4kv_rope_table_bytes(8, 22, 40) == 8 * (8 * 22 + (22 + 40) * 21)
    for bad in [(0, 22, 40), (8, 0, 40), (8, 22, 0), (1, 256, 256), (1 << 21, 1, 1)]:
        assert L.nvfp4kv_rope_table_bytes(*bad) == 0
    # table
    assert L.nvfp4kv_rope_table(0, 8, 22, 40, None, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_rope_table(-1, 8, 22, 40, FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_rope_table((1 << 40) + 1, 8, 22, 40, FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_rope_table(0, 0, 22, 40, FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_rope_table(0, 8, 22, 40, FAKE + 8, None) == swv.ERR_ALIGNMENT
    # rotation
    view = swv.RopeView(FAKE, 8, 22, 40)
    r = ctypes.byref(view)
    assert L.nvfp4kv_rope(None, FAKE, 7040, 24, 128, r, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_rope(FAKE, FAKE, 7040, 24, 128, None, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_rope(FAKE, FAKE, 7041, 24, 128, r, None) == swv.ERR_INVALID_ARG  # > 8 frames
    assert L.nvfp4kv_rope(FAKE, FAKE, 0, 24, 128, r, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_rope(FAKE, FAKE, 7040, 24, 96, r, None) == swv.ERR_UNSUPPORTED
    n = 7040 * 24 * 128 * 2
    for y in (FAKE + 16, FAKE + n - 16, FAKE - n + 16):                 # partial overlaps
        assert L.nvfp4kv_rope(FAKE, y, 7040, 24, 128, r, None) == swv.ERR_INVALID_ARG
    for y in (FAKE, FAKE + n, FAKE - n):                                 # in place, disjoint
        assert L.nvfp4kv_rope(FAKE, y, 7040, 24, 128, r, None) == swv.ERR_UNSUPPORTED
    far = FAKE + (1 << 32)                                      # disjoint from X
    assert L.nvfp4kv_rope(FAKE + 8, far, 7040, 24, 128, r, None) == swv.ERR_ALIGNMENT
    assert L.nvfp4kv_rope(FAKE, FAKE, 100, 1 << 13, 128, r, None) == swv.ERR_INVALID_ARG
    big = swv.RopeView(FAKE, 2, 300, 300)                       # rows * cols > 65535
    assert L.nvfp4kv_rope(FAKE, FAKE, 100, 2, 128, ctypes.byref(big), None) == \
        swv.ERR_INVALID_ARG
    wide = swv.RopeView(FAKE, 1, 100, 200)                      # too large to stage
    assert L.nvfp4kv_rope(FAKE, FAKE, 100, 2, 128, ctypes.byref(wide), None) == \
        swv.ERR_INVALID_ARG
    huge = swv.RopeView(FAKE, 100, 22, 40)                      # T > 65535
    assert L.nvfp4kv_rope(FAKE, FAKE, 70000, 1, 128, ctypes.byref(huge), None) == \
        swv.ERR_INVALID_ARG
    for bad_view in [swv.RopeView(None, 8, 22, 40), swv.RopeView(FAKE, 0, 22, 40)]:
        assert L.nvfp4kv_rope(FAKE, FAKE, 7040, 24, 128, ctypes.byref(bad_view), None) == \
            swv.ERR_INVALID_ARG
    unaligned = swv.RopeView(FAKE + 4, 8, 22, 40)
    assert L.nvfp4kv_rope(FAKE, FAKE, 7040, 24, 128, ctypes.byref(unaligned), None) == \
        swv.ERR_ALIGNMENT
    # fused quantizer and cache append
    v = swv.chunk_view_init(FAKE, 7040, 24)
    assert L.nvfp4kv_quantize_chunk_rope(FAKE, FAKE, 7040, 24, 128, None, ctypes.byref(v),
                                         FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_quantize_chunk_rope(FAKE, FAKE, 7041, 24, 128, r, ctypes.byref(v),
                                         FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_quantize_chunk_rope(None, FAKE, 7040, 24, 128, r, ctypes.byref(v),
                                         FAKE, None) == swv.ERR_INVALID_ARG
    assert L.nvfp4kv_quantize_chunk_rope(FAKE, FAKE, 7040, 24, 128, r, ctypes.byref(v),
                                         None, None) == swv.ERR_INVALID_ARG
    h, _ = _cache(L, 1, 1, 1, 2, T=32, H=2)
    small = swv.RopeView(FAKE, 1, 4, 4)                         # 16 tokens < T_c = 32
    assert L.kvcache_append_rope(h, 0, FAKE, FAKE, None, None) == swv.ERR_INVALID_ARG
    assert L.kvcache_append_rope(h, 0, FAKE, FAKE, ctypes.byref(small), None) == \
        swv.ERR_INVALID_ARG
    n = ctypes.c_int64()
    assert L.kvcache_num_chunks(h, 0, ctypes.byref(n)) == swv.OK and n.value == 0
    L.kvcache_destroy(h)
