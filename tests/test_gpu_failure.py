"""Failure detection on the GPU without a fault: every wait in the kernels is
bounded in time (200 ms) and reports through the workspace's status word.  A
planted count in the quantizer's "CTAs counted into max |V|" word means that
the count never reaches the grid size; every CTA's V-table builder waits for
it, and the kernel must give up, record ERR_DEVICE_TIMEOUT with that wait's
site, and leave the context usable: after nvfp4kv_workspace_init the same
workspace quantizes the chunk bit-exactly again."""
import numpy as np
import pytest

import synth
from gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def test_quantizer_barrier_timeout_is_reported_and_recoverable(lib, orc):
    import torch
    T, H = 256, 4
    K = synth.k_with_offsets_bf16(71, 0, 0, (T, H, 128))
    V = synth.gaussian_bf16(71, 0, 0, synth.T_V, (T, H, 128))
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    ws = lib.new_workspace(T, H)
    torch.cuda.synchronize()
    ws.view(torch.int32)[26] = 1 << 30     # q_vdone: the count can never reach the grid size
    out = lib.ChunkBuffer(T, H)
    lib.quantize_chunk(Kd, Vd, out, ws)
    diag = ws.view(torch.int32)[3:7].cpu().numpy()        # site, block, step, phase
    assert lib.workspace_status(ws) == lib.ERR_DEVICE_TIMEOUT
    assert diag[0] == 101                  # the wait for every CTA's max |V| gave up
    assert lib.workspace_status(ws) == lib.OK              # reading cleared the status
    lib.workspace_init(ws)
    out = lib.ChunkBuffer(T, H)
    lib.quantize_chunk(Kd, Vd, out, ws)
    assert lib.workspace_status(ws) == lib.OK
    got, ref = out.to_host(), orc.quantize_chunk(K, V)
    for k in ("k_codes", "k_scales", "v_codes", "v_scales"):
        assert np.array_equal(got[k], ref[k]), k


def test_attention_wait_timeout_is_reported_and_recoverable(lib, orc):
    """The attention kernel's bounded waits: a test word in the workspace makes
    one de-quantization thread of CTA 0 withhold its first tile's arrival, so
    the MMA issuer (waiting for that tile) and everything queued behind it give
    up after the 200 ms bound.  The kernel must report ERR_DEVICE_TIMEOUT with
    the site of one of those waits and CTA 0, leave the context usable (its
    abort path drains the MMAs and frees tensor memory), and, with the word
    cleared by nvfp4kv_workspace_init, the same workspace must then give the
    oracle's attention."""
    import time

    import torch
    from gpu_util import assert_attention_close, host_to_f64
    T_c, H, T_q = 256, 2, 300
    ws = lib.new_workspace(T_c, H)
    bufs, qs = [], []
    for i in range(3):
        K = synth.k_with_offsets_bf16(80 + i, 0, 0, (T_c, H, 128))
        V = synth.gaussian_bf16(80 + i, 0, 0, synth.T_V, (T_c, H, 128))
        b = lib.ChunkBuffer(T_c, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
        bufs.append(b)
        qs.append(orc.quantize_chunk(K, V))
    Q = synth.gaussian_bf16(89, 0, 0, synth.T_Q, (T_q, H, 128))
    Qd = dev_bf16(Q)
    O = torch.empty((T_q, H, 128), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    ws.view(torch.int32)[7] = 1            # test word: withhold one arrival in CTA 0
    t0 = time.perf_counter()
    lib.attention(bufs, Qd, O, ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    diag = ws.view(torch.int32)[3:7].cpu().numpy()        # site, block, step, phase
    assert lib.workspace_status(ws) == lib.ERR_DEVICE_TIMEOUT
    assert int(diag[0]) in (10, 11, 30, 42), diag     # S waits, ring refill, MMA issue
    assert int(diag[1]) & 0xFFFF == 0                 # CTA 0
    assert 0.15 < elapsed < 5.0
    lib.workspace_init(ws)
    lib.attention(bufs, Qd, O, ws)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    assert_attention_close(host_to_f64(O), orc.attention_f64(qs, Q), "after the timeout")


def test_fp4q_attention_wait_timeout_is_reported_and_recoverable(lib, orc):
    """The same for the FP4-operand attention kernel: its first producer thread
    of CTA 0 withholds the first tile's arrival; the call reports
    ERR_DEVICE_TIMEOUT at one of the waits behind it, in CTA 0, and the next
    call on the re-initialized workspace matches the oracle."""
    import time

    import torch
    from gpu_util import assert_attention_close, host_to_f64
    T_c, H, T_q = 256, 2, 300
    ws = lib.new_workspace(T_c, H)
    bufs, qs = [], []
    for i in range(3):
        K = synth.k_with_offsets_bf16(180 + i, 0, 0, (T_c, H, 128))
        V = synth.gaussian_bf16(180 + i, 0, 0, synth.T_V, (T_c, H, 128))
        b = lib.ChunkBuffer(T_c, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
        bufs.append(b)
        qs.append(orc.quantize_chunk(K, V))
    Q = synth.gaussian_bf16(189, 0, 0, synth.T_Q, (T_q, H, 128))
    Qd = dev_bf16(Q)
    qb = lib.Fp4QBuffer(T_q, H)
    O = torch.empty((T_q, H, 128), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    ws.view(torch.int32)[7] = 1
    t0 = time.perf_counter()
    lib.attention_fp4q(bufs, Qd, O, qb, ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    diag = ws.view(torch.int32)[3:7].cpu().numpy()
    assert lib.workspace_status(ws) == lib.ERR_DEVICE_TIMEOUT
    assert int(diag[0]) in (10, 11, 30, 42), diag
    assert int(diag[1]) & 0xFFFF == 0
    assert 0.15 < elapsed < 5.0
    lib.workspace_init(ws)
    lib.attention_fp4q(bufs, Qd, O, qb, ws)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    assert_attention_close(host_to_f64(O), orc.attention_f64_fp4q(qs, Q), "after the timeout")
