"""Failure detection on the GPU without a fault: every wait in the kernels is
bounded in time (200 ms) and reports through the workspace's status word.  A
planted arrival count in the quantizer's grid-barrier counter means that no
arrival completes the first barrier; every CTA waits for a generation that never
comes, and the kernel must give up,
record ERR_DEVICE_TIMEOUT with the barrier's site, and leave the context
usable: after nvfp4kv_workspace_init the same workspace quantizes the chunk
bit-exactly again."""
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
    ws.view(torch.int32)[1] = 1 << 30      # bar_count: no arrival can complete the barrier
    out = lib.ChunkBuffer(T, H)
    lib.quantize_chunk(Kd, Vd, out, ws)
    diag = ws.view(torch.int32)[3:7].cpu().numpy()        # site, block, step, phase
    assert lib.workspace_status(ws) == lib.ERR_DEVICE_TIMEOUT
    assert diag[0] == 100                  # the grid barrier gave up
    assert lib.workspace_status(ws) == lib.OK              # reading cleared the status
    lib.workspace_init(ws)
    out = lib.ChunkBuffer(T, H)
    lib.quantize_chunk(Kd, Vd, out, ws)
    assert lib.workspace_status(ws) == lib.OK
    got, ref = out.to_host(), orc.quantize_chunk(K, V)
    for k in ("k_codes", "k_scales", "v_codes", "v_scales"):
        assert np.array_equal(got[k], ref[k]), k
