"""GPU weight / activation quantizer (nvfp4kv_quantize_matrix) against the
oracle, bit for bit: codes, scale bytes and the tensor scale, for 1D row
blocks (activations) and 2D 16 x 16 tiles (weights), at the 5B DiT's shapes
(activations [7040, 3072], weights [3072, 3072]), on ragged shapes, on zeros
and on signed zeros, bf16 subnormals and extreme magnitudes."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _matrix(seed, M, N, outlier=30.0):
    z = synth.normal(synth.stream_key(seed, 0, 0, synth.T_EXTRA), M * N).reshape(M, N)
    u = synth.uniform(synth.stream_key(seed, 0, 1, synth.T_EXTRA), M * N).reshape(M, N)
    return synth.to_bf16_bits(np.where(u < 0.01, z * outlier, z))


def _check(lib, orc, X, mode, ws=None, what="", guard=False):
    """Quantize on the GPU and compare with the oracle; with guard, every
    output sits between sentinel guards that must stay untouched."""
    import torch
    from gpu_util import Guarded
    M, N = X.shape
    ws = lib.new_matrix_workspace() if ws is None else ws
    out = lib.MatrixBuffer(M, N, mode)
    guards = []
    if guard:
        for name in ("codes", "scales", "tensor_scale"):
            t = getattr(out, name)
            g = Guarded(tuple(t.shape), t.dtype)
            setattr(out, name, g.t)
            guards.append((name, g))
    lib.quantize_matrix(_dev(X), out, ws)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    for name, g in guards:
        g.assert_intact(f"{what} {name}")
    got, ref = out.to_host(), orc.quantize_matrix(X, mode)
    assert np.float32(got["s"]) == np.float32(ref["s"]), f"{what} tensor scale"
    for k in ("scales", "codes"):
        if not np.array_equal(got[k], ref[k]):
            idx = np.argwhere(got[k] != ref[k])
            raise AssertionError(f"{what} {k}: {len(idx)} bytes differ, first at {idx[:4].tolist()}")
    return ws


@pytest.mark.parametrize("mode,M,N", [(1, 7040, 3072), (2, 3072, 3072)],
                         ids=["activations-7040x3072", "weights-3072x3072"])
def test_dit_shapes_bit_exact(lib, orc, mode, M, N):
    _check(lib, orc, _matrix(100 + mode, M, N), mode, what=f"mode {mode}")


@pytest.mark.parametrize("mode,M,N", [(1, 1, 16), (1, 7, 48), (1, 33, 272), (1, 130, 528),
                                      (2, 16, 16), (2, 48, 80), (2, 160, 304)])
def test_ragged_shapes_bit_exact(lib, orc, mode, M, N):
    _check(lib, orc, _matrix(7 + M + N, M, N), mode, what=f"{M}x{N}", guard=True)


@pytest.mark.parametrize("mode", [1, 2])
def test_degenerate_and_extreme_inputs(lib, orc, mode):
    M, N = 64, 96
    rng = np.random.default_rng(5)
    X = _matrix(77, M, N)
    f = synth.bf16_bits_to_f32(X).astype(np.float64)
    cases = [(np.zeros((M, N), np.uint16), "zeros")]
    Z = X.copy()
    Z[rng.random(X.shape) < 0.05] = 0x8000
    cases.append((Z, "signed zeros"))
    S = X.copy()
    m = rng.random(X.shape) < 0.03
    S[m] = (rng.integers(1, 0x80, m.sum()) | (rng.integers(0, 2, m.sum()) << 15)).astype(np.uint16)
    cases.append((S, "bf16 subnormals"))
    for e in (-110, 100):
        cases.append((synth.to_bf16_bits(f * 2.0 ** e), f"scaled by 2^{e}"))
    blocks = rng.random((M // 16, N // 16)) < 0.2
    cases.append((synth.to_bf16_bits(f * np.where(np.kron(blocks, np.ones((16, 16))), 2.0 ** -110, 1.0)),
                  "tiny blocks"))
    ws = None
    for X_, what in cases:
        ws = _check(lib, orc, X_, mode, ws, what)


def test_query_quantization_at_the_layer_shape(lib, orc):
    """The first step of an FP4-operand Q K^T: the layer's queries [7040, 24, 128]
    as the matrix [7040 * 24, 128], 16-element blocks along d, bit-exact against
    the oracle's quantize_queries (codes, scale bytes, tensor scale)."""
    import torch
    T_q, H = 7040, 24
    Q = synth.gaussian_bf16(800, 0, 0, synth.T_Q, (T_q, H, 128))
    ws = lib.new_matrix_workspace()
    out = lib.MatrixBuffer(T_q * H, 128, 1)
    lib.quantize_matrix(_dev(Q).view(T_q * H, 128), out, ws)
    torch.cuda.synchronize()
    assert lib.workspace_status(ws) == lib.OK
    got = out.to_host()
    ref, _ = orc.quantize_queries(Q)
    assert np.float32(got["s"]) == np.float32(ref["s"])
    assert np.array_equal(got["scales"], ref["scales"])
    assert np.array_equal(got["codes"], ref["codes"])
