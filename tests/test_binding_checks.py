"""The binding's own argument checks, which run before any device call
(CPU tensors stand in for device ones): outputs of mixed dtype or the wrong
size are refused by dequantize, and a Q or O that does not match by
attention."""
import types

import pytest


@pytest.fixture
def lib():
    """The binding module itself (no device needed for these checks)."""
    import sink_window_video_b200 as swv
    return swv


def _chunk(T_c, H, d=128):
    return types.SimpleNamespace(T_c=T_c, H=H, d=d)


def test_dequantize_refuses_mixed_dtypes(lib):
    import torch
    c = _chunk(8, 2)
    with pytest.raises(TypeError):
        lib.dequantize(c, torch.empty((8, 2, 128), dtype=torch.float32),
                       torch.empty((8, 2, 128), dtype=torch.bfloat16))


def test_dequantize_refuses_short_or_strided_outputs(lib):
    import torch
    c = _chunk(8, 2)
    with pytest.raises(ValueError):
        lib.dequantize(c, torch.empty((7, 2, 128), dtype=torch.float32))
    with pytest.raises(ValueError):
        lib.dequantize(c, V_out=torch.empty((8, 2, 256), dtype=torch.bfloat16)[:, :, :128])
    with pytest.raises(TypeError):
        lib.dequantize(c, torch.empty((8, 2, 128), dtype=torch.float16))


def test_dequantize_without_outputs_is_a_no_op(lib):
    assert lib.dequantize(_chunk(8, 2)) is None


def test_attention_refuses_mismatched_q_or_o(lib):
    import torch
    Q = torch.empty((16, 2, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):          # Q not bf16
        lib._check_qo(Q.float(), torch.empty((16, 2, 128)), 2, 128)
    with pytest.raises(ValueError):          # wrong head count
        lib._check_qo(Q, torch.empty((16, 2, 128)), 3, 128)
    with pytest.raises(ValueError):          # O too small
        lib._check_qo(Q, torch.empty((15, 2, 128)), 2, 128)
    lib._check_qo(Q, torch.empty((16, 2, 128)), 2, 128)
