"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests and
the benchmark.

This module holds no arithmetic of the method itself: it only draws numbers.
Both sides of every parity check receive the very same bf16 arrays from here.

Generator (defined here, from the published algorithms it names):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014) used counter-style: word i of a stream with key k
    is mix(k + (i + 1) * GAMMA), i.e. the i-th output of SplitMix64 seeded k.
  * uniform double u = (word >> 11) * 2^-53 in [0, 1).
  * standard normals by the Box-Muller transform (1958) on consecutive pairs:
    r = sqrt(-2 ln(1 - u0)), z0 = r cos(2 pi u1), z1 = r sin(2 pi u1), in double.
  * values are formed in double, rounded to float32, then to bf16, each
    round-to-nearest-even.
Stream keys: key(seed, layer, chunk, tensor) = mix(mix(mix(seed ^ A) ^ layer*B)
^ chunk*C) ^ tensor, with fixed odd constants A, B, C (below).

Workload recipes: the shapes stand in for the K/V/Q activations of a 5B video
DiT at 1280x704 (880 tokens per latent frame, 8 frames per chunk = 7040 tokens,
24 heads, head dim 128).  Real activations are not available; the recipes
below give them the structure the quantizer has to cope with: per-channel
offsets (what K-smoothing removes) and sparse outliers.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_KA = 0xD1B54A32D192ED03
_KB = 0xABC98388FB8FAC03
_KC = 0x8CB92BA72F3D8DD7

# tensor ids of the streams
T_K, T_V, T_Q, T_K_OFFSET, T_K_OUTLIER, T_EXTRA = 1, 2, 3, 4, 5, 6


def _mix_scalar(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * _MIX1) & _M64
    z = ((z ^ (z >> 27)) * _MIX2) & _M64
    return z ^ (z >> 31)


def stream_key(seed: int, layer: int = 0, chunk: int = 0, tensor: int = 0) -> int:
    k = _mix_scalar(seed ^ _KA)
    k = _mix_scalar(k ^ ((layer * _KB) & _M64))
    k = _mix_scalar(k ^ ((chunk * _KC) & _M64))
    return (k ^ tensor) & _M64


_PARALLEL_MIN = 1 << 20
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1))
    return _POOL


def _split(n: int, f):
    """Evaluate f(start, count) over index ranges of [0, n) (in threads when n is
    large) and concatenate; the result does not depend on the split."""
    if n < _PARALLEL_MIN:
        return f(0, n)
    parts = min(16, os.cpu_count() or 1)
    step = -(-n // parts)
    step += step & 1                      # keep Box-Muller pairs inside one part
    ranges = [(a, min(step, n - a)) for a in range(0, n, step)]
    return np.concatenate(list(_pool().map(lambda r: f(*r), ranges)))


def words(key: int, n: int, start: int = 0) -> np.ndarray:
    """SplitMix64 outputs start .. start+n-1 of the stream seeded with key."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z = np.uint64(key) + i * np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MIX2)
        z = z ^ (z >> np.uint64(31))
    return z


def _uniform_range(key, start, n):
    return (words(key, n, start) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def uniform(key: int, n: int) -> np.ndarray:
    return _split(n, lambda a, c: _uniform_range(key, a, c))


def _normal_range(key, start, n):
    # start is even: pair k of the stream uses words 2k and 2k+1
    m = (n + 1) // 2
    u = _uniform_range(key, start, 2 * m)
    u0, u1 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u0))
    ang = 2.0 * np.pi * u1
    z = np.empty(2 * m, np.float64)
    z[0::2] = r * np.cos(ang)
    z[1::2] = r * np.sin(ang)
    return z[:n]


def normal(key: int, n: int) -> np.ndarray:
    """n standard normals (float64) by Box-Muller on consecutive uniform pairs."""
    return _split(n, lambda a, c: _normal_range(key, a, c))


def _bf16_range(x):
    f = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32)
    u = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (u >> np.uint32(16)).astype(np.uint16)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """double -> float32 -> bf16 bit patterns (uint16), each nearest-even."""
    x = np.asarray(x)
    flat = x.reshape(-1)
    return _split(flat.size, lambda a, c: _bf16_range(flat[a:a + c])).reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ recipes

def gaussian_bf16(seed, layer, chunk, tensor, shape, offset_channel=None, offset=0.0):
    """N(0,1) bf16 tensor of the given [T, H, d] shape; optionally one channel
    (index into d) shifted by `offset` in every head and token."""
    n = int(np.prod(shape))
    z = normal(stream_key(seed, layer, chunk, tensor), n).reshape(shape)
    if offset_channel is not None:
        z[..., offset_channel] += offset
    return to_bf16_bits(z)


def k_with_offsets_bf16(seed, layer, chunk, shape, offset_std=2.0, outlier_p=0.01,
                        outlier_mult=20.0):
    """K recipe: N(0,1) noise, a per-(head, channel) offset ~ N(0, offset_std^2)
    shared by all tokens of the chunk, and a fraction outlier_p of elements whose
    noise is multiplied by outlier_mult."""
    T, H, d = shape
    n = T * H * d
    z = normal(stream_key(seed, layer, chunk, T_K), n).reshape(shape)
    off = normal(stream_key(seed, layer, chunk, T_K_OFFSET), H * d).reshape(1, H, d)
    if outlier_p > 0:
        u = uniform(stream_key(seed, layer, chunk, T_K_OUTLIER), n).reshape(shape)
        z = np.where(u < outlier_p, z * outlier_mult, z)
    return to_bf16_bits(z + offset_std * off)


# Configurations (sizes of the 5B DiT stand-in).
TINY = dict(name="tiny", H=2, d=128, T_c=32, chunks=4, S_g=1, S_s=1, W=2, seed=0)
QUANT = dict(name="quantize-only", H=24, d=128, T_c=7040, chunks=100, seed_base=1)
ATTN = dict(name="one-layer attention", H=24, d=128, T_c=7040, S_g=1, S_s=1, W=3, seed=2,
            appended=10, shot_start=4)
ROLLOUT = dict(name="30-layer rollout", layers=30, H=24, d=128, T_c=7040, chunks=16,
               S_g=1, S_s=1, W=4, seed=3, switches=(), outlier_mult=20.0)
MULTISHOT = dict(name="multi-shot long stream", layers=30, H=24, d=128, T_c=7040, chunks=64,
                 S_g=1, S_s=1, W=4, seed=4, switches=(12, 28, 45), outlier_mult=50.0)


def tiny_chunk(chunk: int):
    """Tiny config: K, V, Q ~ N(0,1) with channel 7 shifted by +8, seed 0."""
    c = TINY
    shape = (c["T_c"], c["H"], c["d"])
    return tuple(gaussian_bf16(c["seed"], 0, chunk, t, shape, offset_channel=7, offset=8.0)
                 for t in (T_K, T_V, T_Q))


def quant_chunk(index: int, T_c=7040, H=24, d=128):
    """Quantize-only config, chunk `index` (0-based, seed index+1): K with
    offsets and 1% outliers x20, V ~ N(0,1)."""
    seed = QUANT["seed_base"] + index
    shape = (T_c, H, d)
    K = k_with_offsets_bf16(seed, 0, 0, shape)
    V = gaussian_bf16(seed, 0, 0, T_V, shape)
    return K, V


def layer_chunk(cfg: dict, layer: int, chunk: int, T_c=None, H=None, d=None):
    """K, V, Q for (layer, chunk) of the attention / rollout configs: K with
    per-channel offsets and outliers (cfg's multiplier), V and Q ~ N(0,1)."""
    T_c = T_c or cfg["T_c"]
    H = H or cfg["H"]
    d = d or cfg["d"]
    shape = (T_c, H, d)
    mult = cfg.get("outlier_mult", 20.0)
    K = k_with_offsets_bf16(cfg["seed"], layer, chunk, shape, outlier_mult=mult)
    V = gaussian_bf16(cfg["seed"], layer, chunk, T_V, shape)
    Q = gaussian_bf16(cfg["seed"], layer, chunk, T_Q, shape)
    return K, V, Q
