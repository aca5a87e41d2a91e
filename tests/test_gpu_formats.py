"""The GPU's own format conversions (the sm_100 cvt instructions the kernels use)
and the quantizer's division, element by element against the oracle, through
nvfp4kv_check_formats."""
import numpy as np
import pytest

from brute import E2M1_MAGS, E4M3_POS, midpoints_with_neighbours

pytestmark = pytest.mark.gpu


def _run(lib, op, x, out_dtype, n=None):
    import torch
    xin = torch.from_numpy(x).cuda()
    n = x.size if n is None else n
    out = torch.empty(n, dtype=out_dtype, device="cuda")
    lib.check_formats(op, xin, out, n)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_e2m1_encode_matches_oracle(lib, orc):
    import torch
    rng = np.random.default_rng(21)
    pts = midpoints_with_neighbours(E2M1_MAGS)
    y = np.concatenate([
        pts, -pts,
        np.float32([0.0, -0.0, 1e-30, -1e-30, 1e-40, -1e-40, 6.0, -6.0, 7.5, -100.0, 3e38]),
        rng.uniform(-8, 8, 4_000_000).astype(np.float32),
        (rng.standard_normal(2_000_000) * np.exp2(rng.integers(-20, 8, 2_000_000))).astype(np.float32),
    ]).astype(np.float32)
    got = _run(lib, 0, y, torch.uint8)
    want = orc.e2m1_encode(y)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. y={y[bad[:8]]} gpu={got[bad[:8]]} oracle={want[bad[:8]]}"


def test_e4m3_encode_matches_oracle(lib, orc):
    import torch
    rng = np.random.default_rng(22)
    pts = midpoints_with_neighbours(E4M3_POS)
    y = np.concatenate([
        pts, np.float32([0.0, 448.0, 463.9, 464.0, 1e6, 2.0 ** -10, 2.0 ** -11, 1e-30]),
        rng.uniform(0, 500, 2_000_000).astype(np.float32),
        np.exp2(rng.uniform(-14, 10, 2_000_000)).astype(np.float32),
    ]).astype(np.float32)
    got = _run(lib, 1, y, torch.uint8)
    want = orc.e4m3_encode(y)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. y={y[bad[:8]]} gpu={got[bad[:8]]} oracle={want[bad[:8]]}"


def test_decoders_match_oracle(lib, orc):
    import torch
    codes = np.arange(16, dtype=np.uint8)
    got = _run(lib, 2, codes, torch.float32)
    assert np.array_equal(got.view(np.uint32), orc.e2m1_decode(codes).view(np.uint32))
    b = np.arange(256, dtype=np.uint8)
    got = _run(lib, 3, b, torch.float32)
    want = orc.e4m3_decode(b)
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok].view(np.uint32), want[ok].view(np.uint32))


def test_quotient_is_correctly_rounded(lib, orc):
    """x / D as the quantizer forms it equals IEEE fp32 division (numpy) for x
    like K - mean and D = E4M3 value * tensor scale."""
    import torch
    rng = np.random.default_rng(23)
    n = 8_000_000
    x = (rng.standard_normal(n) * np.exp2(rng.integers(-8, 8, n))).astype(np.float32)
    sb = orc.e4m3_decode(rng.integers(1, 0x7F, n).astype(np.uint8))
    s = np.exp2(rng.uniform(-14, 2, n)).astype(np.float32)
    D = (sb * s).astype(np.float32)
    pairs = np.empty(2 * n, np.float32)
    pairs[0::2], pairs[1::2] = x, D
    got = _run(lib, 4, pairs, torch.float32, n=n)
    want = (x / D).astype(np.float32)
    bad = np.nonzero(got.view(np.uint32) != want.view(np.uint32))[0]
    assert bad.size == 0, f"{bad.size} quotients differ, e.g. x={x[bad[:4]]} D={D[bad[:4]]}"


def test_softmax_ex2_polynomial_within_its_bound(lib):
    """The attention softmax's 2^x on the FMA pipe (Cody-Waite style split into
    n + f, a least-squares cubic for 2^f on [-1/2, 1/2]): relative error at most
    7.6e-5 (7.504e-5 for the cubic itself, plus fp32 rounding) against exp2 in
    float64, over its input range [-125, 8] -- every integer and half-integer
    point, their fp32 neighbours, and a dense random sweep -- and inputs below
    the range are taken as -125."""
    import torch
    rng = np.random.default_rng(31)
    grid = np.arange(-250, 17, dtype=np.float64) / 2.0            # n and n + 1/2
    g32 = grid.astype(np.float32)
    pts = np.concatenate([g32, np.nextafter(g32, np.float32(-np.inf)),
                          np.nextafter(g32, np.float32(np.inf))])
    x = np.concatenate([pts, rng.uniform(-125.0, 8.0, 4_000_000).astype(np.float32),
                        rng.uniform(-1.0, 1.0, 1_000_000).astype(np.float32)])
    x = np.clip(x, np.float32(-125.0), np.float32(8.0)).astype(np.float32)
    got = _run(lib, 5, x, torch.float32).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    worst = int(np.argmax(rel))
    assert rel[worst] <= 7.6e-5, f"x={x[worst]!r}: 2^x {want[worst]!r}, got {got[worst]!r}"
    assert rel.mean() < 5e-5
    low = np.float32([-125.5, -126.0, -130.0, -1000.0])
    assert np.array_equal(_run(lib, 5, low, torch.float32),
                          _run(lib, 5, np.full(4, -125.0, np.float32), torch.float32))
