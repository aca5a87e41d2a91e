"""Pins of the oracle's rotary position embedding (oracle.rope).

The txtmix page "LongLive 2.0：给长视频生成补上 NVFP4 并行基础设施" names a fused
RoPE kernel (section NVFP4：一条从训练贯穿到 KV cache 的量化线) and the option
multi_shot_rope_offset (section 多 shot 一致性), but gives no rotary form, so the
oracle follows a stated reading (oracle.c, oracle_rope): a 3D rotary embedding
over (frame, row, column) with parts of 44, 42 and 42 channels and base 10000.
Parity against the pages stays unpinned; these tests pin the oracle to what a
rotation and that reading fix without restating its formula: the origin is the
identity, coordinate 1 turns the first pair by exactly 1 radian (textbook
cos 1, sin 1), each axis moves only its own channels, pair norms are kept,
dot products depend only on coordinate differences, and the recovered
frequencies form a ladder from 1 down to 1/10000 over each part.
"""
import numpy as np
import pytest

import oracle

D = 128
PARTS = ((0, 44), (44, 42), (86, 42))      # (first channel, width): frame, row, column

COS1 = 0.5403023058681398                  # cos(1 rad)
SIN1 = 0.8414709848078965                  # sin(1 rad)


def bf16_round(x):
    """fp64 values -> nearest bf16 (ties to even), via fp32 (exact for these)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u << 16).astype(np.uint32).view(np.float32).astype(np.float64)


def to_f(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_b(x):
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def random_bf16(rng, shape):
    return to_b(rng.standard_normal(shape))


def test_origin_is_identity():
    rng = np.random.default_rng(1)
    X = random_bf16(rng, (1, 3, D))
    assert np.array_equal(oracle.rope(X, 0, 22, 40), X)


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_coordinate_one_turns_the_first_pair_by_one_radian(axis):
    rows, cols = 3, 5
    t = {0: 0, 1: cols, 2: 1}[axis]             # token at coordinate 1 on `axis`, 0 elsewhere
    pos0 = 1 if axis == 0 else 0
    T = t + 1
    X = np.zeros((T, 2, D), np.uint16)
    c0 = PARTS[axis][0]
    X[t, 0, c0] = to_b(1.0)                     # e_0 of the part: (1, 0)
    X[t, 1, c0 + 1] = to_b(1.0)                 # e_1 of the part: (0, 1)
    Y = to_f(oracle.rope(X, pos0, rows, cols))[t]
    assert Y[0, c0] == bf16_round(COS1) and Y[0, c0 + 1] == bf16_round(SIN1)
    assert Y[1, c0] == bf16_round(-SIN1) and Y[1, c0 + 1] == bf16_round(COS1)
    mask = np.ones(D, bool)
    mask[c0:c0 + 2] = False
    assert not Y[:, mask].any()


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_each_axis_moves_only_its_own_channels(axis):
    rows, cols = 4, 6
    rng = np.random.default_rng(10 + axis)
    # the same vector at the origin and at coordinate 3 on `axis` only
    t = {0: 0, 1: 3 * cols, 2: 3}[axis]
    pos0 = 3 if axis == 0 else 0
    v = random_bf16(rng, (2, D))
    X = np.zeros((t + 1, 2, D), np.uint16)
    X[t] = v
    Y = oracle.rope(X, pos0, rows, cols)[t]
    c0, w = PARTS[axis]
    inside = np.zeros(D, bool)
    inside[c0:c0 + w] = True
    assert np.array_equal(Y[:, ~inside], v[:, ~inside])
    assert (Y[:, inside] != v[:, inside]).mean() > 0.5


def test_token_layout_frame_major():
    """Token t is at frame t // (rows*cols), row (t // cols) % rows, column
    t % cols: every token of a later frame equals the same token of a chunk whose
    first frame is that frame, and the first token of a frame turns only the
    frame part."""
    rows, cols, frames = 3, 4, 3
    rng = np.random.default_rng(12)
    v = random_bf16(rng, (rows * cols, 2, D))
    X = np.concatenate([v] * frames)
    Y = oracle.rope(X, 10, rows, cols)
    for f in range(frames):
        assert np.array_equal(Y[f * rows * cols:(f + 1) * rows * cols],
                              oracle.rope(v, 10 + f, rows, cols))
    first = oracle.rope(X, 0, rows, cols)[rows * cols]
    c0, w = PARTS[0]
    assert np.array_equal(first[:, c0 + w:], v[0][:, c0 + w:])


def test_pair_norms_are_kept():
    rng = np.random.default_rng(3)
    rows, cols = 5, 7
    X = random_bf16(rng, (2 * rows * cols, 4, D))
    x = to_f(X).reshape(-1, D // 2, 2)
    y = to_f(oracle.rope(X, 37, rows, cols)).reshape(-1, D // 2, 2)
    nx = np.hypot(x[..., 0], x[..., 1])
    ny = np.hypot(y[..., 0], y[..., 1])
    # four fp32 products and two sums (relative 2^-23 each) then bf16 (2^-9 each)
    assert np.all(np.abs(ny - nx) <= 2.0 ** -8 * nx + 1e-30)


def test_dot_products_depend_only_on_coordinate_differences():
    """<R(p) q, R(p') k> = <R(p + D) q, R(p' + D) k> on every axis: the shot
    offset moves a query and a key of the same shot together, and changes the
    score of a pair in different shots exactly as a longer frame distance."""
    rng = np.random.default_rng(4)
    rows, cols, frames = 6, 8, 3
    T = frames * rows * cols
    q = random_bf16(rng, (T, 2, D))
    k = random_bf16(rng, (T, 2, D))

    def scores(pos_q, pos_k, tq, tk):
        Rq = to_f(oracle.rope(q, pos_q, rows, cols))[tq]
        Rk = to_f(oracle.rope(k, pos_k, rows, cols))[tk]
        return np.einsum("thd,thd->th", Rq, Rk)

    nq = np.linalg.norm(to_f(q), axis=-1)
    nk = np.linalg.norm(to_f(k), axis=-1)
    tq = np.arange(T)
    tk = rng.permutation(T)
    base = scores(5, 2, tq, tk)
    tol = 2.0 ** -6 * nq[tq] * nk[tk]
    # shift the frame axis: both by 100, or the query's shot by an offset of 100
    assert np.all(np.abs(scores(105, 102, tq, tk) - base) <= tol)
    # the row and column axes: the same vectors moved one row and one column on
    inner = ((tq // cols) % rows < rows - 1) & (tq % cols < cols - 1) & \
            ((tk // cols) % rows < rows - 1) & (tk % cols < cols - 1)
    q2, k2 = np.zeros_like(q), np.zeros_like(k)
    q2[tq[inner] + cols + 1] = q[tq[inner]]
    k2[tk[inner] + cols + 1] = k[tk[inner]]
    Rq = to_f(oracle.rope(q2, 5, rows, cols))[tq[inner] + cols + 1]
    Rk = to_f(oracle.rope(k2, 2, rows, cols))[tk[inner] + cols + 1]
    shifted = np.einsum("thd,thd->th", Rq, Rk)
    assert inner.sum() > T // 3
    assert np.all(np.abs(shifted - base[inner]) <= tol[inner])
    # a pair in different shots: offset 100 on the query side equals frame distance + 100
    cross = scores(5 + 100, 2, tq, tk)
    plain = scores(105, 2, tq, tk)
    assert np.array_equal(cross, plain)


def recovered_frequencies(axis, n=4096):
    """Each pair's angle per unit coordinate on `axis`: the unit vector (1, 0)
    in every pair at coordinates 0..n-1, atan2 of the result unwrapped along the
    coordinate, least-squares slope."""
    rows, cols = {0: (1, 1), 1: (n, 1), 2: (1, n)}[axis]
    X = np.zeros((n, 1, D), np.uint16)
    X[:, :, 0::2] = to_b(1.0)
    Y = to_f(oracle.rope(X, 0, rows, cols))[:, 0]
    c0, w = PARTS[axis]
    phi = np.unwrap(np.arctan2(Y[:, c0 + 1:c0 + w:2], Y[:, c0:c0 + w:2]), axis=0)
    p = np.arange(n, dtype=np.float64)
    return np.array([np.polyfit(p, phi[:, i], 1)[0] for i in range(w // 2)])


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_frequency_ladder(axis):
    w = PARTS[axis][1]
    om = recovered_frequencies(axis)
    assert om.shape == (w // 2,)
    assert abs(om[0] - 1.0) < 1e-4                       # the first pair: 1 rad per step
    ratio = om[1:] / om[:-1]
    r = np.exp(np.mean(np.log(ratio)))
    assert np.all(np.abs(ratio / r - 1.0) < 2e-3)        # one constant ratio
    # w/2 steps of the ladder divide the frequency by the base: r^(w/2) = 1/10000
    assert abs(r ** (w // 2) * 1e4 - 1.0) < 1e-2


def test_rope_frame_position():
    assert [oracle.rope_frame_position(n, 8, 0, 0) for n in range(4)] == [0, 8, 16, 24]
    assert oracle.rope_frame_position(5, 8, 2, 1000) == 40 + 2000
    # offset 0: a multi-shot stream counts frames like a single shot
    assert oracle.rope_frame_position(7, 8, 3, 0) == oracle.rope_frame_position(7, 8, 0, 0)
