"""nvfp4kv_quantize_chunk_noalloc -- the quantizer for callers that may not
allocate device memory (engines that own all GPU memory and give plugins no
scratch, real-time loops that must not risk cudaMalloc's synchronization).  It
keeps its scratch in an array compiled into the library instead of a caller
workspace.  Checked through the C ABI against nvfp4kv_quantize_chunk (the
workspace entry point), bit for bit, on two calls in a row (through the
Python binding), and its refusals through the raw C ABI; this file is
collected last so that a failure here comes after every other test ran."""
import ctypes

import numpy as np
import pytest

import synth
from gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def _entry(lib):
    L = lib.load()
    fn = L.nvfp4kv_quantize_chunk_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                   ctypes.POINTER(lib.ChunkView), ctypes.c_void_p]
    return fn


def _parts(buf):
    return {k: getattr(buf, k).cpu().numpy()
            for k in ("k_codes", "k_scales", "v_codes", "v_scales", "k_mean", "tensor_scales")}


def test_noalloc_matches_workspace_entry_point_twice(lib):
    import torch
    inputs = [synth.quant_chunk(0), synth.layer_chunk(synth.MULTISHOT, 0, 3)[:2]]
    for call, (K, V) in enumerate(inputs):
        T, H, d = K.shape
        Kd, Vd = dev_bf16(K), dev_bf16(V)
        ref = lib.ChunkBuffer(T, H, d)
        ws = lib.new_workspace(T, H, d)
        lib.quantize_chunk(Kd, Vd, ref, ws)
        got = lib.ChunkBuffer(T, H, d)
        lib.quantize_chunk_noalloc(Kd, Vd, got)          # raises on a status other than OK
        torch.cuda.synchronize()
        assert lib.workspace_status(ws) == lib.OK
        a, b = _parts(got), _parts(ref)
        for k in a:
            assert np.array_equal(a[k].view(np.uint8), b[k].view(np.uint8)), f"call {call}: {k}"


def test_noalloc_at_its_largest_chunk(lib):
    """T_c = 10,816 at H = 24 fills the compiled-in scratch to within 8 KB of its
    end: the same bytes as the workspace entry point, twice in a row."""
    import torch
    T, H, d = 10816, 24, 128
    K = synth.k_with_offsets_bf16(91, 0, 0, (T, H, d))
    V = synth.gaussian_bf16(91, 0, 0, synth.T_V, (T, H, d))
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    ref = lib.ChunkBuffer(T, H, d)
    ws = lib.new_workspace(T, H, d)
    lib.quantize_chunk(Kd, Vd, ref, ws)
    b = _parts(ref)
    for call in range(2):
        got = lib.ChunkBuffer(T, H, d)
        lib.quantize_chunk_noalloc(Kd, Vd, got)
        torch.cuda.synchronize()
        a = _parts(got)
        for k in a:
            assert np.array_equal(a[k].view(np.uint8), b[k].view(np.uint8)), f"call {call}: {k}"
    assert lib.workspace_status(ws) == lib.OK


def test_noalloc_refuses_chunks_beyond_its_scratch(lib):
    import torch
    fn = _entry(lib)
    K = torch.zeros((16, 2, 128), dtype=torch.bfloat16, device="cuda")
    buf = lib.ChunkBuffer(16, 2)
    # one token past the largest chunk (10,817 x 24 needs a 170th 64-token
    # segment: more than the 4 MiB compiled-in scratch); refused from the sizes
    # alone, before anything reads K
    for T in (10817, 10880):
        st = fn(K.data_ptr(), K.data_ptr(), T, 24, 128, ctypes.byref(buf.view),
                torch.cuda.current_stream().cuda_stream)
        assert st == lib.ERR_CAPACITY
    assert fn(K.data_ptr(), K.data_ptr(), 16, 2, 64, ctypes.byref(buf.view), None) \
        == lib.ERR_UNSUPPORTED
