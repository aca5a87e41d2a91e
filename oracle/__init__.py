"""Python access to the C oracle (test infrastructure).

The oracle is a plain, slow CPU reference for the NVFP4 KV-cache quantizer and
the multi-shot sink-window attention (see oracle.c for the definition and the
sources it follows).  Only the test suite, the smoke check and the CPU-baseline
leg of the benchmark use it; the CUDA library never imports it.

Arrays are numpy; bf16 tensors travel as uint16 bit patterns.
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None


class OracleChunk(ctypes.Structure):
    """Host view of one quantized chunk, the layout of oracle.c's oracle_chunk."""
    _fields_ = [
        ("k_codes", ctypes.c_void_p),
        ("k_scales", ctypes.c_void_p),
        ("k_mean", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p),
        ("v_scales", ctypes.c_void_p),
        ("s_k", ctypes.c_float),
        ("s_v", ctypes.c_float),
        ("T", ctypes.c_int),
    ]


def lib():
    """Load (building first if needed) liboracle.so."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_encode.argtypes = [f32]
        L.oracle_e2m1_decode.restype = f32
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [f32]
        L.oracle_e4m3_decode.restype = f32
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        for name in ("oracle_e2m1_encode_array", "oracle_e2m1_decode_array",
                     "oracle_e4m3_encode_array", "oracle_e4m3_decode_array",
                     "oracle_f32_to_bf16_array"):
            getattr(L, name).argtypes = [vp, vp, sz]
            getattr(L, name).restype = None
        L.oracle_k_mean.argtypes = [vp, i32, i32, i32, vp]
        L.oracle_quantize_tensor.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp]
        L.oracle_quantize_chunk.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        L.oracle_dequantize_tensor.argtypes = [vp, vp, vp, f32, i32, i32, i32, vp]
        L.oracle_keyset.restype = i32
        L.oracle_keyset.argtypes = [ctypes.c_int64, i32, i32, i32, ctypes.c_int64, vp]
        L.oracle_attention_f64.argtypes = [vp, i32, i32, i32, vp, i32, vp, i32,
                                           ctypes.c_double, vp]
        L.oracle_attention_f64_fq.argtypes = [vp, i32, i32, i32, vp, i32, vp, i32,
                                              ctypes.c_double, vp]
        L.oracle_chunk_payload_bytes.restype = sz
        L.oracle_chunk_payload_bytes.argtypes = [i32, i32, i32]
        L.oracle_quantize_matrix.restype = i32
        L.oracle_quantize_matrix.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
        L.oracle_dequantize_matrix.argtypes = [vp, vp, f32, i32, i32, i32, vp]
        L.oracle_rope.argtypes = [vp, i32, i32, i32, ctypes.c_int64, i32, i32, vp]
        L.oracle_rope_cos_sin.argtypes = [ctypes.c_int64, i32, i32, vp, vp]
        L.oracle_set_threads.argtypes = [i32]
        L.oracle_get_threads.restype = i32
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def set_threads(n: int):
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# ---------------------------------------------------------------- formats

def e2m1_encode(y) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_ptr(y), _ptr(out), y.size)
    return out


def e2m1_decode(q) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    out = np.empty(q.shape, np.float32)
    lib().oracle_e2m1_decode_array(_ptr(q), _ptr(out), q.size)
    return out


def e4m3_encode(y) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(y), _ptr(out), y.size)
    return out


def e4m3_decode(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, np.float32)
    lib().oracle_e4m3_decode_array(_ptr(b), _ptr(out), b.size)
    return out


def f32_to_bf16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- quantizer

def k_mean(K: np.ndarray) -> np.ndarray:
    K = np.ascontiguousarray(K, dtype=np.uint16)
    T, H, d = K.shape
    mean = np.empty((H, d), np.float32)
    lib().oracle_k_mean(_ptr(K), T, H, d, _ptr(mean))
    return mean


def quantize_tensor(X: np.ndarray, smooth: bool):
    """Quantize one [T, H, d] bf16 tensor.  Returns a dict with codes [H,T,d/2],
    scales [H,T,d/16], mean [H,d] (K only, else None), s (float) and choice
    [H,T,d/16] (1 where the 4-target encoding was kept)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    T, H, d = X.shape
    codes = np.empty((H, T, d // 2), np.uint8)
    scales = np.empty((H, T, d // 16), np.uint8)
    choice = np.empty((H, T, d // 16), np.uint8)
    mean = np.empty((H, d), np.float32) if smooth else None
    s = np.zeros(1, np.float32)
    lib().oracle_quantize_tensor(_ptr(X), T, H, d, _ptr(mean), _ptr(codes), _ptr(scales),
                                 _ptr(s), _ptr(choice))
    return dict(codes=codes, scales=scales, mean=mean, s=float(s[0]), choice=choice)


def quantize_chunk(K: np.ndarray, V: np.ndarray):
    """Quantize one chunk's K (with K-smoothing) and V.  Returns a dict with
    k_codes, k_scales, v_codes, v_scales, k_mean, s_k, s_v (and the choices)."""
    k = quantize_tensor(K, smooth=True)
    v = quantize_tensor(V, smooth=False)
    return dict(k_codes=k["codes"], k_scales=k["scales"], k_mean=k["mean"], s_k=k["s"],
                v_codes=v["codes"], v_scales=v["scales"], s_v=v["s"],
                k_choice=k["choice"], v_choice=v["choice"], T=K.shape[0])


def dequantize_tensor(codes, scales, mean, s, T, H, d) -> np.ndarray:
    """fp32 [T, H, d] reconstruction: decode(q) * (decode(sb) * s) (+ mean)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    if mean is not None:
        mean = np.ascontiguousarray(mean, dtype=np.float32)
    out = np.empty((T, H, d), np.float32)
    lib().oracle_dequantize_tensor(_ptr(codes), _ptr(scales), _ptr(mean), float(s),
                                   T, H, d, _ptr(out))
    return out


def dequantize_chunk(q):
    H, T, _ = q["k_codes"].shape
    d = q["k_mean"].shape[1]
    Kh = dequantize_tensor(q["k_codes"], q["k_scales"], q["k_mean"], q["s_k"], T, H, d)
    Vh = dequantize_tensor(q["v_codes"], q["v_scales"], None, q["s_v"], T, H, d)
    return Kh, Vh


MATRIX_1D, MATRIX_2D = 1, 2


def quantize_matrix(X: np.ndarray, mode: int):
    """NVFP4 quantization of a bf16 matrix X [M, N] with Four-Over-Six: mode 1
    (activations) 16-element row blocks, mode 2 (weights) 16 x 16 tiles.
    Returns dict codes [M, N/2], scales ([M, N/16] or [M/16, N/16]), s, choice."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    M, N = X.shape
    brows = M if mode == MATRIX_1D else M // 16
    codes = np.zeros((M, N // 2), np.uint8)
    scales = np.zeros((brows, N // 16), np.uint8)
    choice = np.zeros((brows, N // 16), np.uint8)
    s = np.zeros(1, np.float32)
    if lib().oracle_quantize_matrix(_ptr(X), M, N, mode, _ptr(codes), _ptr(scales), _ptr(s),
                                    _ptr(choice)) != 0:
        raise ValueError(f"shape {X.shape} is not tiled by mode {mode}")
    return dict(codes=codes, scales=scales, s=float(s[0]), choice=choice)


def dequantize_matrix(q: dict, mode: int) -> np.ndarray:
    M, N2 = q["codes"].shape
    out = np.zeros((M, 2 * N2), np.float32)
    lib().oracle_dequantize_matrix(_ptr(np.ascontiguousarray(q["codes"])),
                                   _ptr(np.ascontiguousarray(q["scales"])), q["s"], M, 2 * N2,
                                   mode, _ptr(out))
    return out


def payload_bytes(T, H, d) -> int:
    return int(lib().oracle_chunk_payload_bytes(T, H, d))


# ---------------------------------------------------------------- key set

def keyset(n: int, S_g: int, S_s: int, W: int, s_begin: int):
    ids = np.zeros(max(1, S_g + S_s + W), np.int64)
    cnt = lib().oracle_keyset(int(n), int(S_g), int(S_s), int(W), int(s_begin), _ptr(ids))
    return [int(x) for x in ids[:cnt]]


# ---------------------------------------------------------------- attention

def _chunk_array(chunks):
    keep = []
    arr = (OracleChunk * max(1, len(chunks)))()
    for i, c in enumerate(chunks):
        parts = [np.ascontiguousarray(c[k]) for k in
                 ("k_codes", "k_scales", "k_mean", "v_codes", "v_scales")]
        keep.append(parts)
        arr[i] = OracleChunk(*(p.ctypes.data for p in parts), float(c["s_k"]),
                             float(c["s_v"]), int(c["k_codes"].shape[1]))
    return arr, keep


def _attention(fn, chunks, Q, rows, scale):
    T_q, H, d = Q.shape
    arr, keep = _chunk_array(chunks)
    if rows is None:
        rows_arr = None
        n_rows = T_q
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int32)
        n_rows = rows_arr.size
    out = np.zeros((n_rows, H, d), np.float64)
    if not (scale > 0):
        scale = 1.0 / math.sqrt(d)
    fn(arr, len(chunks), H, d, _ptr(Q), T_q, _ptr(rows_arr), n_rows, float(scale), _ptr(out))
    del keep
    return out


def attention_f64(chunks, Q: np.ndarray, rows=None, scale: float = 0.0) -> np.ndarray:
    """Float64 attention of Q [T_q, H, d] (bf16 bits) over the listed quantized
    chunks (dicts as returned by quantize_chunk, in key order).  rows: query rows
    to evaluate (None = all).  Returns [n_rows, H, d] float64."""
    Q = np.ascontiguousarray(Q, dtype=np.uint16)
    return _attention(lib().oracle_attention_f64, chunks, Q, rows, scale)


def attention_f64_fq(chunks, Qf: np.ndarray, rows=None, scale: float = 0.0) -> np.ndarray:
    """attention_f64 for queries given as fp32 values [T_q, H, d]."""
    Qf = np.ascontiguousarray(Qf, dtype=np.float32)
    return _attention(lib().oracle_attention_f64_fq, chunks, Qf, rows, scale)


def quantize_queries(Q: np.ndarray):
    """NVFP4 of the queries for an FP4-operand S = Q K^T ("2605-LongLive2"
    DeepRead page, Method > 推理基础设施: W4A4 on Blackwell, FP4 GEMMs in place of
    BF16 ones; Method > 训练基础设施: activations in 1D blocks): Q [T_q, H, d]
    (bf16 bits) as the matrix [T_q * H, d], 16-element blocks along d -- the
    contraction -- with Four-Over-Six and one FP32 tensor scale (quantize_matrix,
    MATRIX_1D).  Returns (the quantize_matrix dict, Q_hat [T_q, H, d] fp32)."""
    Q = np.ascontiguousarray(Q, dtype=np.uint16)
    T_q, H, d = Q.shape
    q = quantize_matrix(Q.reshape(T_q * H, d), MATRIX_1D)
    return q, dequantize_matrix(q, MATRIX_1D).reshape(T_q, H, d)


def attention_f64_fp4q(chunks, Q: np.ndarray, rows=None, scale: float = 0.0) -> np.ndarray:
    """Float64 attention with the queries replaced by their NVFP4 reconstruction
    (quantize_queries): the reference for an FP4-operand Q K^T over the cache."""
    _, Qh = quantize_queries(Q)
    return attention_f64_fq(chunks, Qh, rows, scale)


def rope(X: np.ndarray, frame_pos0: int, rows: int, cols: int) -> np.ndarray:
    """3D rotary position embedding of one chunk's queries or keys, X [T, H, d]
    bf16 bits -> bf16 bits (oracle_rope in oracle.c states the reading: the
    txtmix page "LongLive 2.0：给长视频生成补上 NVFP4 并行基础设施", sections
    NVFP4 and 多 shot 一致性, names a fused RoPE kernel and the multi-shot RoPE
    offset but not the rotary form).  Token t of the chunk sits at frame
    frame_pos0 + t // (rows*cols), row (t // cols) % rows, column t % cols."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    T, H, d = X.shape
    Y = np.empty_like(X)
    lib().oracle_rope(_ptr(X), T, H, d, int(frame_pos0), rows, cols, _ptr(Y))
    return Y


def rope_cos_sin(p: int, i: int, w: int):
    """(cos, sin) of pair i's angle p * 10000^(-2i/w), each rounded once from
    double to fp32 (the values oracle_rope turns that pair by), as float32."""
    c = np.zeros(1, np.float32)
    s = np.zeros(1, np.float32)
    lib().oracle_rope_cos_sin(int(p), int(i), int(w), _ptr(c), _ptr(s))
    return c[0], s[0]


def rope_frame_position(chunk: int, frames_per_chunk: int, shot: int, offset: int) -> int:
    """Frame coordinate of chunk `chunk`'s first frame in a multi-shot stream:
    the frames before it, plus multi_shot_rope_offset once per shot switch
    before it (`shot` switches; the txtmix page, 多 shot 一致性: the offset keeps
    the positions of different shots apart).  offset 0 is plain frame counting."""
    return chunk * frames_per_chunk + shot * offset
