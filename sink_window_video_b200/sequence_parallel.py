"""Ulysses-style sequence parallelism over the NVFP4 KV cache.

Each of P ranks (one per GPU) holds a contiguous shard of a chunk's tokens for
all heads -- K, V and Q [T_r, H, 128] bf16.  Attention needs every token of a
head, so the ranks trade tokens for heads (an all-to-all) -- and ship the cache
quantized, 4.5 bits per element instead of 16 (DeepRead page, Method >
推理基础设施: the NVFP4 cache cuts the sequence-parallel communication).

quantize_chunk_sp, per chunk:
  1. each rank: nvfp4kv_chunk_stats on its shard (K's 64-token segment sums,
     minima, maxima; max |V|);
  2. all-gather of the segment statistics (token order) and all-reduce(max) of
     max |V|;
  3. each rank: nvfp4kv_chunk_finalize -> the chunk's mean and tensor scales,
     identical on every rank;
  4. each rank: nvfp4kv_chunk_encode of its shard;
  5. all-to-all of codes and scales: rank j receives every token of heads
     [j H/P, (j+1) H/P) -- its head shard of the cache, bit-identical to those
     heads of the one-GPU quantization.
attention_sp: all-to-all of Q into head shards, sink-window attention per head
shard, all-to-all of O back into token shards.

Shards: whole 64-token segments split as evenly as possible (shard_bounds), so
that every K-smoothing segment lies in one shard.  H must divide by P.  The
collectives are torch.distributed's (NCCL between GPUs); the layout steps
between them are plain tensor reshapes.

Head parallelism (quantize_chunk_heads): each rank already holds every token
of its heads [h0, h1) (head_bounds).  The mean and the blocks are per head, so
the one exchange per chunk is an all-reduce(max) of the two amaxes that set
the tensor scales (reduce_amax); attention then runs on each rank's heads with
no exchange at all.
"""
import torch
import torch.distributed as dist

import sink_window_video_b200 as lib

SEGMENT = 64
HEAD_DIM = 128


def shard_bounds(T: int, P: int):
    """Token ranges [t0, t1) of the P ranks: the ceil(T/64) segments split as
    evenly as possible, in rank order."""
    nseg = (T + SEGMENT - 1) // SEGMENT
    return [(min(SEGMENT * (nseg * r // P), T), min(SEGMENT * (nseg * (r + 1) // P), T))
            for r in range(P)]


def head_bounds(H: int, P: int):
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    Hp = H // P
    return [(j * Hp, (j + 1) * Hp) for j in range(P)]


# ------------------------------------------------------------------ layout steps

def compact_segments(padded: torch.Tensor, counts):
    """[P * nseg_max, ...] rows gathered from P ranks (each padded to nseg_max)
    -> the ranks' real rows in rank (= token) order."""
    nmax = padded.shape[0] // len(counts)
    return torch.cat([padded[r * nmax: r * nmax + c] for r, c in enumerate(counts)])


def assemble_head_shard(blocks):
    """Per source rank r, its tokens of one head block [Hp, T_r, w] -> [Hp, T, w]."""
    return torch.cat(blocks, dim=1)


# ------------------------------------------------------------------ collectives

def _rank_world(group):
    return dist.get_rank(group), dist.get_world_size(group)


def gather_segment_stats(psum, pmin, pmax, vmax, T, group=None):
    """All ranks' segment statistics in token order, and the chunk's max |V|."""
    rank, P = _rank_world(group)
    counts = [(t1 - t0 + SEGMENT - 1) // SEGMENT for t0, t1 in shard_bounds(T, P)]
    nmax = max(counts)
    out = []
    for x in (psum, pmin, pmax):
        pad = torch.zeros((nmax,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        pad[: x.shape[0]] = x
        full = torch.empty((P * nmax,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(full, pad, group=group)
        out.append(compact_segments(full, counts))
    v = vmax.clone()
    dist.all_reduce(v, op=dist.ReduceOp.MAX, group=group)
    return out[0], out[1], out[2], v


def exchange_to_head_shards(local: dict, T: int, H: int, group=None):
    """local: this rank's {k_codes, k_scales, v_codes, v_scales}, each
    [H, T_r, w] (head-major, w bytes per token) -> this rank's head shard, each
    [H/P, T, w]: every token of heads [rank H/P, (rank+1) H/P)."""
    rank, P = _rank_world(group)
    Hp = H // P
    sizes = [t1 - t0 for t0, t1 in shard_bounds(T, P)]
    out = {}
    for name, x in local.items():
        w = x.shape[2]
        recv = torch.empty(Hp * T * w, dtype=x.dtype, device=x.device)
        dist.all_to_all_single(recv, x.contiguous().view(-1),
                               output_split_sizes=[Hp * n * w for n in sizes],
                               input_split_sizes=[Hp * x.shape[1] * w] * P, group=group)
        blocks = [b.view(Hp, n, w) for b, n in zip(torch.split(recv, [Hp * n * w for n in sizes]),
                                                   sizes)]
        out[name] = assemble_head_shard(blocks)
    return out


def exchange_queries(Q_local, T: int, group=None):
    """Q [T_r, H, d] token shard -> [T, H/P, d] head shard."""
    rank, P = _rank_world(group)
    T_r, H, d = Q_local.shape
    Hp = H // P
    sizes = [t1 - t0 for t0, t1 in shard_bounds(T, P)]
    send = torch.stack([Q_local[:, j * Hp:(j + 1) * Hp] for j in range(P)]).contiguous()
    recv = torch.empty((T, Hp, d), dtype=Q_local.dtype, device=Q_local.device)
    dist.all_to_all_single(recv.view(-1), send.view(-1),
                           output_split_sizes=[n * Hp * d for n in sizes],
                           input_split_sizes=[T_r * Hp * d] * P, group=group)
    return recv


def exchange_outputs(O_head, T: int, H: int, group=None):
    """O [T, H/P, d] head shard -> [T_r, H, d] token shard."""
    rank, P = _rank_world(group)
    _, Hp, d = O_head.shape
    bounds = shard_bounds(T, P)
    T_r = bounds[rank][1] - bounds[rank][0]
    recv = torch.empty((P, T_r, Hp, d), dtype=O_head.dtype, device=O_head.device)
    dist.all_to_all_single(recv.view(-1), O_head.contiguous().view(-1),
                           output_split_sizes=[T_r * Hp * d] * P,
                           input_split_sizes=[(t1 - t0) * Hp * d for t0, t1 in bounds], group=group)
    return recv.permute(1, 0, 2, 3).reshape(T_r, H, d)


# ------------------------------------------------------------------ the two steps

def quantize_chunk_sp(K_local, V_local, T: int, ws, group=None):
    """This rank's head shard of the quantized chunk (a ChunkBuffer of T tokens
    and H/P heads) from its token shard of K and V."""
    rank, P = _rank_world(group)
    T_r, H, d = K_local.shape
    psum, pmin, pmax, vmax = lib.chunk_stats(K_local, V_local, ws)
    psum, pmin, pmax, vmax = gather_segment_stats(psum, pmin, pmax, vmax, T, group)
    k_mean, scales = lib.chunk_finalize(psum, pmin, pmax, vmax, T, H, ws)
    local = lib.ChunkBuffer(T_r, H, d)
    lib.chunk_encode(K_local, V_local, k_mean, scales, local)
    shard = exchange_to_head_shards(
        {"k_codes": local.k_codes, "k_scales": local.k_scales,
         "v_codes": local.v_codes, "v_scales": local.v_scales}, T, H, group)
    Hp = H // P
    out = lib.ChunkBuffer(T, Hp, d)
    for name, x in shard.items():
        getattr(out, name).copy_(x)
    out.k_mean.copy_(k_mean[rank * Hp:(rank + 1) * Hp])
    out.tensor_scales.copy_(scales)
    return out


def reduce_amax(amax, group=None):
    """The chunk's [max |K - mean|, max |V|] from every rank's: all-reduce(max)
    of two floats, in place."""
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def quantize_chunk_heads(K_heads, V_heads, ws, group=None):
    """This rank's heads of the quantized chunk (a ChunkBuffer of all T tokens
    and the rank's heads) from K, V [T, h1 - h0, d] of those heads; bit-equal
    to those heads of the one-GPU quantization, with the whole chunk's tensor
    scales."""
    T, Hr, d = K_heads.shape
    psum, pmin, pmax, vmax = lib.chunk_stats(K_heads, V_heads, ws)
    out = lib.ChunkBuffer(T, Hr, d)
    _, amax = lib.chunk_amax(psum, pmin, pmax, vmax, T, Hr, ws, k_mean=out.k_mean)
    reduce_amax(amax, group)
    lib.tensor_scales_from_amax(amax, out.tensor_scales)
    lib.chunk_encode(K_heads, V_heads, out.k_mean, out.tensor_scales, out)
    return out


def attention_sp(Q_local, head_chunks, T: int, ws_head, o_dtype=torch.bfloat16, group=None):
    """Sink-window attention of this rank's token shard of Q over the head
    shards of the key chunks (as returned by quantize_chunk_sp) -> O [T_r, H, d]."""
    rank, P = _rank_world(group)
    H = Q_local.shape[1]
    Q_head = exchange_queries(Q_local, T, group)
    O_head = torch.empty(Q_head.shape, dtype=o_dtype, device=Q_local.device)
    lib.attention(head_chunks, Q_head, O_head, ws_head)
    return exchange_outputs(O_head, T, H, group)
