"""Sequence-parallel quantization and head-shard attention on one GPU.

* The ranks emulated one after the other (no collectives): per token shard
  nvfp4kv_chunk_stats, the statistics concatenated in token order,
  nvfp4kv_chunk_finalize, per shard nvfp4kv_chunk_encode; the mean, tensor
  scales and every head shard's codes and scales must equal
  nvfp4kv_quantize_chunk on the whole chunk bit for bit (2, 4 and 8 shards of
  the 7040 x 24 chunk; 3 shards of a ragged one).
* Attention over head shards of the cache against the oracle.
* Head parallelism, ranks emulated: each rank's heads quantized on their own,
  the amaxes' maximum over ranks setting the tensor scales; bit-equal to those
  heads of the one-GPU quantization.
* quantize_chunk_sp / attention_sp / quantize_chunk_heads end to end through a
  one-rank NCCL group (the collectives degenerate to copies), against the
  one-GPU path."""
import numpy as np
import pytest

import synth
from gpu_util import assert_attention_close, dev_bf16, host_bf16_to_f64, sample_rows

pytestmark = pytest.mark.gpu


def _chunk(seed, T, H):
    K = synth.k_with_offsets_bf16(seed, 0, 0, (T, H, 128))
    V = synth.gaussian_bf16(seed, 0, 0, synth.T_V, (T, H, 128))
    return K, V


@pytest.mark.parametrize("P,T,H", [(2, 7040, 24), (4, 7040, 24), (8, 7040, 24), (3, 200, 6)])
def test_sharded_quantization_equals_one_gpu(lib, P, T, H):
    import torch
    import sink_window_video_b200.sequence_parallel as sp
    K, V = _chunk(23 + P, T, H)
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    ws = lib.new_workspace(T, H)
    full = lib.ChunkBuffer(T, H)
    lib.quantize_chunk(Kd, Vd, full, ws)
    bounds = sp.shard_bounds(T, P)
    stats = [lib.chunk_stats(Kd[t0:t1], Vd[t0:t1], ws) for t0, t1 in bounds]
    psum, pmin, pmax = (torch.cat([s[i] for s in stats]) for i in range(3))
    vmax = torch.stack([s[3] for s in stats]).max(dim=0).values
    k_mean, scales = lib.chunk_finalize(psum, pmin, pmax, vmax, T, H, ws)
    torch.cuda.synchronize()
    assert torch.equal(k_mean.view(torch.int32), full.k_mean.view(torch.int32))
    assert torch.equal(scales.view(torch.int32), full.tensor_scales.view(torch.int32))
    locals_ = []
    for t0, t1 in bounds:
        b = lib.ChunkBuffer(t1 - t0, H)
        lib.chunk_encode(Kd[t0:t1], Vd[t0:t1], k_mean, scales, b)
        locals_.append(b)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    for h0, h1 in sp.head_bounds(H, P):
        for name in ("k_codes", "k_scales", "v_codes", "v_scales"):
            got = sp.assemble_head_shard([getattr(b, name)[h0:h1] for b in locals_])
            assert torch.equal(got, getattr(full, name)[h0:h1]), (P, h0, name)


@pytest.mark.parametrize("P,T,H,zero", [(2, 7040, 24, False), (3, 7040, 24, False),
                                         (8, 7040, 24, False), (3, 200, 6, True)])
def test_head_parallel_quantization_equals_one_gpu(lib, P, T, H, zero):
    """Head parallelism, the ranks emulated one after another: each rank's
    heads through nvfp4kv_chunk_stats and nvfp4kv_chunk_amax, the maximum of
    the ranks' amaxes (the all-reduce) into nvfp4kv_tensor_scales_from_amax,
    then nvfp4kv_chunk_encode of the rank's heads.  Every rank's codes, scales
    and mean equal those heads of the one-GPU quantization bit for bit, and its
    tensor scales the whole chunk's.  zero: rank 0's heads are all zero, so
    its own amaxes are 0 (an all-zero tensor's scale would be 1)."""
    import torch
    import sink_window_video_b200.sequence_parallel as sp
    K, V = _chunk(51 + P, T, H)
    if zero:
        K[:, : H // P] = 0
        V[:, : H // P] = 0
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    ws = lib.new_workspace(T, H)
    full = lib.ChunkBuffer(T, H)
    lib.quantize_chunk(Kd, Vd, full, ws)
    bounds = sp.head_bounds(H, P)
    ranks, amaxes = [], []
    for h0, h1 in bounds:
        Kh, Vh = Kd[:, h0:h1].contiguous(), Vd[:, h0:h1].contiguous()
        psum, pmin, pmax, vmax = lib.chunk_stats(Kh, Vh, ws)
        b = lib.ChunkBuffer(T, h1 - h0)
        _, amax = lib.chunk_amax(psum, pmin, pmax, vmax, T, h1 - h0, ws, k_mean=b.k_mean)
        ranks.append((Kh, Vh, b))
        amaxes.append(amax)
    if zero:
        torch.cuda.synchronize()
        assert float(amaxes[0].abs().max()) == 0.0
    A = torch.stack(amaxes).max(dim=0).values
    for Kh, Vh, b in ranks:
        lib.tensor_scales_from_amax(A, b.tensor_scales)
        lib.chunk_encode(Kh, Vh, b.k_mean, b.tensor_scales, b)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    for (h0, h1), (_, _, b) in zip(bounds, ranks):
        for name in ("k_codes", "k_scales", "v_codes", "v_scales"):
            assert torch.equal(getattr(b, name), getattr(full, name)[h0:h1]), (P, h0, name)
        assert torch.equal(b.k_mean.view(torch.int32), full.k_mean[h0:h1].view(torch.int32))
        assert torch.equal(b.tensor_scales.view(torch.int32), full.tensor_scales.view(torch.int32))


def test_tensor_scales_from_amax(lib):
    import torch
    amax = torch.tensor([0.0, 2688.0], dtype=torch.float32, device="cuda")
    s = lib.tensor_scales_from_amax(amax)
    amax2 = torch.tensor([1e-30, 3.0e38], dtype=torch.float32, device="cuda")
    s2 = lib.tensor_scales_from_amax(amax2)
    torch.cuda.synchronize()
    assert s.tolist() == [1.0, 1.0]
    want = (np.float32(1e-30) / np.float32(2688), np.float32(3.0e38) / np.float32(2688))
    assert s2.cpu().numpy().tolist() == [float(w) for w in want]


def _head_chunk(lib, full, h0, h1):
    b = lib.ChunkBuffer(full.T_c, h1 - h0)
    for name in ("k_codes", "k_scales", "v_codes", "v_scales", "k_mean"):
        getattr(b, name).copy_(getattr(full, name)[h0:h1])
    b.tensor_scales.copy_(full.tensor_scales)
    return b


def test_head_shard_attention_matches_oracle(lib, orc):
    import torch
    import sink_window_video_b200.sequence_parallel as sp
    T, H, P = 448, 4, 2
    ws = lib.new_workspace(T, H)
    fulls, qs = [], []
    for c in range(2):
        K, V = _chunk(31 + c, T, H)
        b = lib.ChunkBuffer(T, H)
        lib.quantize_chunk(dev_bf16(K), dev_bf16(V), b, ws)
        fulls.append(b)
        qs.append(orc.quantize_chunk(K, V))
    Q = synth.gaussian_bf16(33, 0, 0, synth.T_Q, (T, H, 128))
    for h0, h1 in sp.head_bounds(H, P):
        chunks = [_head_chunk(lib, f, h0, h1) for f in fulls]
        Qh = np.ascontiguousarray(Q[:, h0:h1])
        O = torch.empty(Qh.shape, dtype=torch.float32, device="cuda")
        lib.attention(chunks, dev_bf16(Qh), O, lib.new_workspace(T, h1 - h0))
        torch.cuda.synchronize()
        sl = slice(h0, h1)
        ref_chunks = [dict(q, k_codes=q["k_codes"][sl], k_scales=q["k_scales"][sl],
                           k_mean=q["k_mean"][sl], v_codes=q["v_codes"][sl],
                           v_scales=q["v_scales"][sl]) for q in qs]
        assert_attention_close(host_bf16_to_f64(O), orc.attention_f64(ref_chunks, Qh),
                               f"heads {h0}-{h1}")


def test_end_to_end_through_a_one_rank_group(lib):
    """quantize_chunk_sp and attention_sp with a real (one-rank) NCCL group:
    identical cache bytes and output to the one-GPU calls."""
    import datetime
    import os
    import socket
    import torch
    import torch.distributed as dist
    import sink_window_video_b200.sequence_parallel as sp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        T, H = 448, 4
        ws = lib.new_workspace(T, H)
        chunks_sp, chunks_one = [], []
        for c in range(2):
            K, V = _chunk(41 + c, T, H)
            Kd, Vd = dev_bf16(K), dev_bf16(V)
            chunks_sp.append(sp.quantize_chunk_sp(Kd, Vd, T, ws))
            b = lib.ChunkBuffer(T, H)
            lib.quantize_chunk(Kd, Vd, b, ws)
            chunks_one.append(b)
        for a, b in zip(chunks_sp, chunks_one):
            assert torch.equal(a.base, b.base)
        Qd = dev_bf16(synth.gaussian_bf16(43, 0, 0, synth.T_Q, (T, H, 128)))
        O_sp = sp.attention_sp(Qd, chunks_sp, T, ws, o_dtype=torch.float32)
        O_one = torch.empty((T, H, 128), dtype=torch.float32, device="cuda")
        lib.attention(chunks_one, Qd, O_one, ws)
        torch.cuda.synchronize()
        assert torch.equal(O_sp, O_one)
        # head parallelism through the same group: one rank holds every head
        for c in range(2):
            K, V = _chunk(41 + c, T, H)
            hp = sp.quantize_chunk_heads(dev_bf16(K), dev_bf16(V), ws)
            torch.cuda.synchronize()
            assert torch.equal(hp.base, chunks_one[c].base)
    finally:
        dist.destroy_process_group()
