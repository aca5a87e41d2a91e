"""The exchange steps of the sequence-parallel cache (sink_window_video_b200/
sequence_parallel.py) with real collectives: 2 and 3 gloo ranks on CPU.  The
data are the oracle's: the full chunk quantized in one piece, cut into token
shards as each rank's encoder would produce them.  Checked: the gathered
segment statistics equal those of the whole chunk (token order), every rank's
head shard equals those heads of the one-piece quantization byte for byte,
queries and outputs round-trip between token and head shards, and (head
parallelism) the all-reduced amaxes of the ranks' own heads are the whole
chunk's, whose quotients by 2688 are its tensor scales."""
import os
import socket

import numpy as np
import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _segment_stats(K):
    """Per 64-token segment: fp32 column sums in token order, bf16 min / max."""
    import synth
    T = K.shape[0]
    f = synth.bf16_bits_to_f32(K).reshape(T, -1)
    nseg = (T + 63) // 64
    psum = np.zeros((nseg, f.shape[1]), np.float32)
    pmin = np.zeros((nseg, f.shape[1]), np.float32)
    pmax = np.zeros((nseg, f.shape[1]), np.float32)
    for s in range(nseg):
        acc = np.zeros(f.shape[1], np.float32)
        for t in range(64 * s, min(64 * s + 64, T)):
            acc = (acc + f[t]).astype(np.float32)
        psum[s], pmin[s], pmax[s] = acc, f[64 * s:64 * s + 64].min(0), f[64 * s:64 * s + 64].max(0)
    return psum, pmin, pmax


def _rank(rank, P, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=P, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import synth
        import sink_window_video_b200.sequence_parallel as sp
        T, H = 200, 6
        K = synth.k_with_offsets_bf16(17, 0, 0, (T, H, 128))
        V = synth.gaussian_bf16(17, 0, 0, synth.T_V, (T, H, 128))
        Q = synth.gaussian_bf16(17, 0, 0, synth.T_Q, (T, H, 128))
        t0, t1 = sp.shard_bounds(T, P)[rank]
        h0, h1 = sp.head_bounds(H, P)[rank]
        res = {}
        # segment statistics of the shard -> all segments, token order
        ps, pn, px = (torch.from_numpy(a) for a in _segment_stats(K[t0:t1]))
        vm = torch.tensor([float(np.abs(synth.bf16_bits_to_f32(V[t0:t1])).max())])
        gps, gpn, gpx, gvm = sp.gather_segment_stats(ps, pn, px, vm, T)
        fps, fpn, fpx = _segment_stats(K)
        res["stats"] = (np.array_equal(gps.numpy(), fps) and np.array_equal(gpn.numpy(), fpn)
                        and np.array_equal(gpx.numpy(), fpx)
                        and float(gvm[0]) == float(np.abs(synth.bf16_bits_to_f32(V)).max()))
        # this rank's encoded tokens -> its head shard
        q = oracle.quantize_chunk(K, V)
        local = {k: torch.from_numpy(np.ascontiguousarray(q[k][:, t0:t1]))
                 for k in ("k_codes", "k_scales", "v_codes", "v_scales")}
        shard = sp.exchange_to_head_shards(local, T, H)
        res["heads"] = all(np.array_equal(shard[k].numpy(), q[k][h0:h1]) for k in local)
        # queries to head shards and outputs back
        Qt = torch.from_numpy(Q.view(np.int16)).view(torch.bfloat16)
        Qh = sp.exchange_queries(Qt[t0:t1].contiguous(), T)
        res["q"] = torch.equal(Qh, Qt[:, h0:h1])
        res["o"] = torch.equal(sp.exchange_outputs(Qh, T, H), Qt[t0:t1])
        # head parallelism: this rank's heads alone -> its amaxes -> reduce_amax
        # gives the whole chunk's, and amax / 2688 its tensor scales
        qh = oracle.quantize_chunk(np.ascontiguousarray(K[:, h0:h1]), np.ascontiguousarray(V[:, h0:h1]))
        kf, vf = synth.bf16_bits_to_f32(K), synth.bf16_bits_to_f32(V)
        X = (kf[:, h0:h1] - qh["k_mean"][None]).astype(np.float32)
        amax = torch.tensor([np.abs(X).max(), np.abs(vf[:, h0:h1]).max()], dtype=torch.float32)
        sp.reduce_amax(amax)
        Xf = (kf - q["k_mean"][None]).astype(np.float32)
        res["amax"] = (np.array_equal(qh["k_mean"], q["k_mean"][h0:h1])
                       and float(amax[0]) == float(np.abs(Xf).max())
                       and float(amax[1]) == float(np.abs(vf).max())
                       and np.float32(amax[0].item()) / np.float32(2688) == np.float32(q["s_k"])
                       and np.float32(amax[1].item()) / np.float32(2688) == np.float32(q["s_v"]))
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("P", [2, 3])
def test_exchanges_reproduce_the_one_piece_layout(P):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, P, port, q)) for r in range(P)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(P):
        assert results[r] == {"stats": True, "heads": True, "q": True, "o": True,
                              "amax": True}, (r, results[r])


def test_shard_bounds_align_to_segments():
    import sink_window_video_b200.sequence_parallel as sp
    for T, P in [(7040, 2), (7040, 4), (7040, 8), (200, 3), (64, 2), (1, 1)]:
        b = sp.shard_bounds(T, P)
        assert b[0][0] == 0 and b[-1][1] == T
        assert all(x[1] == y[0] for x, y in zip(b, b[1:]))
        assert all(t0 % 64 == 0 for t0, _ in b)
    with pytest.raises(ValueError):
        sp.head_bounds(24, 5)
