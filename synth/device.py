"""The same seeded generator as synth/__init__.py, evaluated with torch on any
device (a GPU draws a 7040 x 24 x 128 chunk in milliseconds, the host version
in about a second).  It draws numbers only: SplitMix64 words used
counter-style, u = (word >> 11) 2^-53, Box-Muller normals in float64, then
float32 and bf16 by round-to-nearest-even -- the definitions the host module
states, written with 64-bit integer tensors (multiplication wraps modulo 2^64;
right shifts are made logical by masking).

The host module stays the source of every array the oracle and the parity
tests compare.  This one feeds timing runs that need many distinct chunks; its
float64 logarithm, sine and cosine may differ from the host's in the last bit,
which after rounding to bf16 almost never shows (tests/test_synth.py checks a
slice bit for bit)."""
import math

import synth


def _s64(c):
    """An unsigned 64-bit constant as the signed int64 with the same bits."""
    c &= synth._M64
    return c - (1 << 64) if c >= (1 << 63) else c


def _shr(z, s):
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def words(key, n, device, start=0):
    import torch
    i = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = i * _s64(synth.GAMMA) + _s64(key)
    z = (z ^ _shr(z, 30)) * _s64(synth._MIX1)
    z = (z ^ _shr(z, 27)) * _s64(synth._MIX2)
    return z ^ _shr(z, 31)


def uniform(key, n, device):
    import torch
    return _shr(words(key, n, device), 11).to(torch.float64) * (2.0 ** -53)


def normal(key, n, device):
    import torch
    m = (n + 1) // 2
    u = uniform(key, 2 * m, device).view(m, 2)
    r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))
    ang = (2.0 * math.pi) * u[:, 1]
    z = torch.stack((r * torch.cos(ang), r * torch.sin(ang)), dim=1).view(-1)
    return z[:n]


def to_bf16(x):
    """float64 -> float32 -> bf16, each nearest-even, as a torch.bfloat16 tensor."""
    import torch
    u = x.to(torch.float32).view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    u = _shr(u + 0x7FFF + (_shr(u, 16) & 1), 16) & 0xFFFF
    return (u - ((u >= 0x8000).to(torch.int64) << 16)).to(torch.int16).view(torch.bfloat16)


def gaussian_bf16(seed, layer, chunk, tensor, shape, device):
    n = math.prod(shape)
    return to_bf16(normal(synth.stream_key(seed, layer, chunk, tensor), n, device)).view(shape)


def k_with_offsets_bf16(seed, layer, chunk, shape, device, offset_std=2.0, outlier_p=0.01,
                        outlier_mult=20.0):
    import torch
    T, H, d = shape
    n = T * H * d
    z = normal(synth.stream_key(seed, layer, chunk, synth.T_K), n, device).view(shape)
    off = normal(synth.stream_key(seed, layer, chunk, synth.T_K_OFFSET), H * d,
                 device).view(1, H, d)
    if outlier_p > 0:
        u = uniform(synth.stream_key(seed, layer, chunk, synth.T_K_OUTLIER), n,
                    device).view(shape)
        z = torch.where(u < outlier_p, z * outlier_mult, z)
    return to_bf16(z + offset_std * off)


def quant_chunk(index, device, T_c=7040, H=24, d=128):
    """The quantize-only workload's chunk `index` (seed index + 1), as
    synth.quant_chunk draws it."""
    seed = synth.QUANT["seed_base"] + index
    shape = (T_c, H, d)
    return (k_with_offsets_bf16(seed, 0, 0, shape, device),
            gaussian_bf16(seed, 0, 0, synth.T_V, shape, device))
