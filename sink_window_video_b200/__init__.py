"""Python binding of libnvfp4kv (NVFP4 KV cache + multi-shot sink-window
attention for B200).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch provides device memory and streams.  The binding fails
loudly when the compiled library is missing; there is no fallback path.

The names mirror the C ABI in include/nvfp4kv.h.
"""
import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4kv.so")

OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_EMPTY_KEYSET, \
    ERR_CUDA, ERR_DEVICE_TIMEOUT = range(8)
STATUS_NAMES = ["OK", "ERR_INVALID_ARG", "ERR_ALIGNMENT", "ERR_UNSUPPORTED", "ERR_CAPACITY",
                "ERR_EMPTY_KEYSET", "ERR_CUDA", "ERR_DEVICE_TIMEOUT"]
MAX_KEY_CHUNKS = 32
HEAD_DIM = 128
F32, BF16 = 0, 1              # nvfp4kv_dtype

_lib = None


class NvFp4KvError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{where}: {name}")


class ChunkView(ctypes.Structure):
    """nvfp4kv_chunk_view: device pointers to one quantized chunk."""
    _fields_ = [("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("k_mean", ctypes.c_void_p), ("tensor_scales", ctypes.c_void_p)]


class RopeView(ctypes.Structure):
    """nvfp4kv_rope_view: a chunk's rotation table (device) and token grid."""
    _fields_ = [("table", ctypes.c_void_p), ("frames", ctypes.c_int),
                ("rows", ctypes.c_int), ("cols", ctypes.c_int)]


class KVCacheConfig(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("T_c", ctypes.c_int), ("S_g", ctypes.c_int), ("S_s", ctypes.c_int),
                ("W", ctypes.c_int)]


def load():
    """Load libnvfp4kv.so (built by sink_window_video_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python sink_window_video_b200/build.py` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                             ctypes.c_float)
    st = ctypes.c_int
    cv = ctypes.POINTER(ChunkView)
    cfgp = ctypes.POINTER(KVCacheConfig)
    rv = ctypes.POINTER(RopeView)
    sigs = {
        "nvfp4kv_chunk_bytes": (sz, [i32, i32, i32]),
        "nvfp4kv_chunk_view_init": (st, [vp, i32, i32, i32, cv]),
        "nvfp4kv_workspace_bytes": (sz, [i32, i32, i32]),
        "nvfp4kv_workspace_init": (st, [vp, sz, vp]),
        "nvfp4kv_workspace_status": (st, [vp, vp]),
        "nvfp4kv_quantize_chunk": (st, [vp, vp, i32, i32, i32, cv, vp, vp]),
        "nvfp4kv_quantize_chunk_noalloc": (st, [vp, vp, i32, i32, i32, cv, vp]),
        "nvfp4kv_dequantize": (st, [cv, i32, i32, i32, vp, vp, i32, vp]),
        "nvfp4kv_attention": (st, [cv, i32, i32, i32, i32, vp, i32, vp, i32, f32, vp, vp]),
        "nvfp4kv_attention_launches": (i32, [i32, i32, i32, i32, i32]),
        "nvfp4kv_fp4q_bytes": (sz, [i32, i32, i32]),
        "nvfp4kv_attention_fp4q": (st, [cv, i32, i32, i32, i32, vp, i32, vp, i32, f32, vp, vp,
                                        vp]),
        "nvfp4kv_attention_fp4q_launches": (i32, [i32, i32, i32, i32, i32]),
        "nvfp4kv_matrix_workspace_bytes": (sz, []),
        "nvfp4kv_rope_frame_position": (ctypes.c_longlong, [ctypes.c_longlong, i32,
                                                            ctypes.c_longlong,
                                                            ctypes.c_longlong]),
        "nvfp4kv_rope_table_bytes": (sz, [i32, i32, i32]),
        "nvfp4kv_rope_table": (st, [ctypes.c_longlong, i32, i32, i32, vp, vp]),
        "nvfp4kv_rope": (st, [vp, vp, i32, i32, i32, rv, vp]),
        "nvfp4kv_quantize_chunk_rope": (st, [vp, vp, i32, i32, i32, rv, cv, vp, vp]),
        "kvcache_append_rope": (st, [vp, i32, vp, vp, rv, vp]),
        "nvfp4kv_chunk_stats": (st, [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
        "nvfp4kv_chunk_finalize": (st, [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]),
        "nvfp4kv_chunk_amax": (st, [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]),
        "nvfp4kv_tensor_scales_from_amax": (st, [vp, vp, vp]),
        "nvfp4kv_chunk_encode": (st, [vp, vp, i32, i32, i32, vp, vp, cv, vp]),
        "nvfp4kv_quantize_matrix": (st, [vp, i32, i32, i32, vp, vp, vp, vp, vp]),
        "kvcache_pool_bytes": (sz, [cfgp]),
        "kvcache_create": (st, [cfgp, vp, vp, ctypes.POINTER(vp)]),
        "kvcache_destroy": (None, [vp]),
        "kvcache_append": (st, [vp, i32, vp, vp, vp]),
        "kvcache_rebind_shot_sink": (st, [vp, i64]),
        "kvcache_keyset": (st, [vp, i32, ctypes.POINTER(i64), ctypes.POINTER(i32)]),
        "kvcache_num_chunks": (st, [vp, i32, ctypes.POINTER(i64)]),
        "kvcache_chunk_view": (st, [vp, i32, i64, cv]),
        "kvcache_advance": (st, [vp, i32, cv]),
        "kvcache_state_bytes": (sz, [vp]),
        "kvcache_get_state": (st, [vp, vp, sz]),
        "kvcache_set_state": (st, [vp, vp, sz]),
        "sink_window_attention": (st, [vp, i32, vp, i32, vp, i32, f32, vp]),
        "kvcache_check_status": (st, [vp, vp]),
        "nvfp4kv_check_formats": (st, [i32, vp, vp, sz, vp]),
        "nvfp4kv_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status, where):
    if status != OK:
        raise NvFp4KvError(status, where)


def _ptr(x):
    """Device address of a torch tensor (or an int / None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"output dtype {t.dtype} is not float32 or bfloat16")


def _check_qo(Q, O, H, d):
    """Q: contiguous bf16 [T_q, H, d]; O: contiguous, same element count."""
    import torch
    if Q.dtype != torch.bfloat16 or Q.dim() != 3 or tuple(Q.shape[1:]) != (H, d) \
            or not Q.is_contiguous():
        raise ValueError(f"Q must be a contiguous bf16 [T_q, {H}, {d}] tensor, "
                         f"got {Q.dtype} {tuple(Q.shape)}")
    if not O.is_contiguous() or O.numel() != Q.numel():
        raise ValueError(f"O of shape {tuple(O.shape)} does not match Q {tuple(Q.shape)}")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def version() -> str:
    return load().nvfp4kv_version().decode()


# ------------------------------------------------------------------ sizes

def chunk_bytes(T_c, H, d=HEAD_DIM) -> int:
    return int(load().nvfp4kv_chunk_bytes(T_c, H, d))


def chunk_stats(K, V, ws, stream=None):
    """Per-shard statistics of the sequence-parallel quantizer: psum [nseg][H*d]
    fp32, pmin / pmax [nseg][H*d] bf16, vmax [1] fp32."""
    import torch
    T, H, d = K.shape
    nseg = (T + 63) // 64
    psum = torch.empty((nseg, H * d), dtype=torch.float32, device=K.device)
    pmin = torch.empty((nseg, H * d), dtype=torch.bfloat16, device=K.device)
    pmax = torch.empty((nseg, H * d), dtype=torch.bfloat16, device=K.device)
    vmax = torch.empty(1, dtype=torch.float32, device=K.device)
    _check(load().nvfp4kv_chunk_stats(_ptr(K), _ptr(V), T, H, d, _ptr(psum), _ptr(pmin),
                                      _ptr(pmax), _ptr(vmax), _ptr(ws), _stream(stream)),
           "nvfp4kv_chunk_stats")
    return psum, pmin, pmax, vmax


def chunk_finalize(psum, pmin, pmax, vmax, T, H, ws, d=HEAD_DIM, stream=None):
    """Mean [H][d] and tensor scales [2] of a chunk from all of its segments'
    statistics (token order) and its max |V|."""
    import torch
    k_mean = torch.empty((H, d), dtype=torch.float32, device=psum.device)
    scales = torch.empty(2, dtype=torch.float32, device=psum.device)
    _check(load().nvfp4kv_chunk_finalize(_ptr(psum), _ptr(pmin), _ptr(pmax), psum.shape[0], T,
                                         H, d, _ptr(vmax), _ptr(k_mean), _ptr(scales), _ptr(ws),
                                         _stream(stream)),
           "nvfp4kv_chunk_finalize")
    return k_mean, scales


def chunk_amax(psum, pmin, pmax, vmax, T, H, ws, d=HEAD_DIM, k_mean=None, stream=None):
    """Mean [H][d] (into k_mean when given) and the two amaxes [max |K - mean|,
    max |V|] of a chunk, or of a head shard of it, from its segments'
    statistics and its max |V|."""
    import torch
    if k_mean is None:
        k_mean = torch.empty((H, d), dtype=torch.float32, device=psum.device)
    amax = torch.empty(2, dtype=torch.float32, device=psum.device)
    _check(load().nvfp4kv_chunk_amax(_ptr(psum), _ptr(pmin), _ptr(pmax), psum.shape[0], T, H, d,
                                     _ptr(vmax), _ptr(k_mean), _ptr(amax), _ptr(ws),
                                     _stream(stream)),
           "nvfp4kv_chunk_amax")
    return k_mean, amax


def tensor_scales_from_amax(amax, out=None, stream=None):
    """[s_K, s_V] = amax / 2688 (1 for a zero amax), on the device."""
    import torch
    if out is None:
        out = torch.empty(2, dtype=torch.float32, device=amax.device)
    _check(load().nvfp4kv_tensor_scales_from_amax(_ptr(amax), _ptr(out), _stream(stream)),
           "nvfp4kv_tensor_scales_from_amax")
    return out


def chunk_encode(K, V, k_mean, tensor_scales, out: "ChunkBuffer", stream=None):
    """Codes and block scales of a token shard with the chunk's mean and scales."""
    T, H, d = K.shape
    _check(load().nvfp4kv_chunk_encode(_ptr(K), _ptr(V), T, H, d, _ptr(k_mean),
                                       _ptr(tensor_scales), ctypes.byref(out.view),
                                       _stream(stream)),
           "nvfp4kv_chunk_encode")


BLOCKS_1D, TILES_2D = 1, 2


class MatrixBuffer:
    """Device buffers of a quantized [M, N] matrix: codes [M, N/2] (uint8),
    scales ([M, N/16] for 1D blocks, [M/16, N/16] for 2D tiles), tensor scale."""

    def __init__(self, M, N, mode, device="cuda"):
        import torch
        self.M, self.N, self.mode = M, N, mode
        brows = M if mode == BLOCKS_1D else M // 16
        self.codes = torch.zeros((M, N // 2), dtype=torch.uint8, device=device)
        self.scales = torch.zeros((brows, N // 16), dtype=torch.uint8, device=device)
        self.tensor_scale = torch.zeros(1, dtype=torch.float32, device=device)

    def to_host(self):
        return dict(codes=self.codes.cpu().numpy(), scales=self.scales.cpu().numpy(),
                    s=float(self.tensor_scale[0].item()))


def new_matrix_workspace(device="cuda", stream=None):
    import torch
    ws = torch.zeros(int(load().nvfp4kv_matrix_workspace_bytes()), dtype=torch.uint8,
                     device=device)
    workspace_init(ws, stream)
    return ws


def quantize_matrix(X, out: "MatrixBuffer", ws, stream=None):
    """NVFP4 quantization of a bf16 [M, N] matrix with Four-Over-Six (1D row
    blocks or 2D 16 x 16 tiles, out.mode)."""
    M, N = X.shape
    _check(load().nvfp4kv_quantize_matrix(_ptr(X), M, N, out.mode, _ptr(out.codes),
                                          _ptr(out.scales), _ptr(out.tensor_scale), _ptr(ws),
                                          _stream(stream)),
           "nvfp4kv_quantize_matrix")


def attention_launches(n_chunks, T_c, H, T_q, d=HEAD_DIM) -> int:
    """Kernels one attention call of this shape enqueues (1, or 2 with a split tail)."""
    return int(load().nvfp4kv_attention_launches(n_chunks, T_c, H, d, T_q))


def workspace_bytes(T_c, H, d=HEAD_DIM) -> int:
    return int(load().nvfp4kv_workspace_bytes(T_c, H, d))


def chunk_view_init(base, T_c, H, d=HEAD_DIM) -> ChunkView:
    v = ChunkView()
    _check(load().nvfp4kv_chunk_view_init(_ptr(base), T_c, H, d, ctypes.byref(v)),
           "nvfp4kv_chunk_view_init")
    return v


def workspace_init(ws, stream=None):
    _check(load().nvfp4kv_workspace_init(_ptr(ws), ws.numel() * ws.element_size(),
                                         _stream(stream)), "nvfp4kv_workspace_init")


def workspace_status(ws, stream=None) -> int:
    """Synchronize and return the workspace status code and clear it: OK,
    ERR_DEVICE_TIMEOUT (a bounded wait in a kernel gave up) or ERR_UNSUPPORTED
    (an attention key set whose V tensor scales span more than 2^116)."""
    return int(load().nvfp4kv_workspace_status(_ptr(ws), _stream(stream)))


# ------------------------------------------------------------------ device buffers

class ChunkBuffer:
    """One quantized chunk in a torch uint8 device buffer, with torch views of
    its parts (codes [H, T, d/2], scales [H, T, d/16], k_mean [H, d],
    tensor_scales [2])."""

    def __init__(self, T_c, H, d=HEAD_DIM, device="cuda", buf=None):
        import torch
        self.T_c, self.H, self.d = T_c, H, d
        n = chunk_bytes(T_c, H, d)
        self.buf = buf if buf is not None else torch.zeros(n + 256, dtype=torch.uint8,
                                                           device=device)
        off = (-self.buf.data_ptr()) % 256
        self.base = self.buf[off:off + n]
        self.view = chunk_view_init(self.base, T_c, H, d)
        b0 = self.base.data_ptr()

        def part(ptr, nbytes):
            return self.base[ptr - b0: ptr - b0 + nbytes]
        nn = T_c * H * d
        self.k_codes = part(self.view.k_codes, nn // 2).view(H, T_c, d // 2)
        self.v_codes = part(self.view.v_codes, nn // 2).view(H, T_c, d // 2)
        self.k_scales = part(self.view.k_scales, nn // 16).view(H, T_c, d // 16)
        self.v_scales = part(self.view.v_scales, nn // 16).view(H, T_c, d // 16)
        self.k_mean = part(self.view.k_mean, H * d * 4).view(torch.float32).view(H, d)
        self.tensor_scales = part(self.view.tensor_scales, 8).view(torch.float32)

    def to_host(self):
        """dict of numpy arrays in the layout the oracle uses."""
        return dict(k_codes=self.k_codes.cpu().numpy(), k_scales=self.k_scales.cpu().numpy(),
                    v_codes=self.v_codes.cpu().numpy(), v_scales=self.v_scales.cpu().numpy(),
                    k_mean=self.k_mean.cpu().numpy(),
                    s_k=float(self.tensor_scales[0].item()),
                    s_v=float(self.tensor_scales[1].item()), T=self.T_c)


def new_workspace(T_c, H, d=HEAD_DIM, device="cuda", stream=None):
    """A zeroed torch uint8 workspace (256-byte aligned) for chunks of this shape."""
    import torch
    n = workspace_bytes(T_c, H, d)
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    workspace_init(ws, stream)
    return ws


# ------------------------------------------------------------------ quantizer

def quantize_chunk(K, V, out: ChunkBuffer, ws, stream=None):
    """K, V: bf16 [T_c, H, d] device tensors -> out (a ChunkBuffer)."""
    T, H, d = K.shape
    _check(load().nvfp4kv_quantize_chunk(_ptr(K), _ptr(V), T, H, d, ctypes.byref(out.view),
                                         _ptr(ws), _stream(stream)), "nvfp4kv_quantize_chunk")


# ------------------------------------------------------------------ rotary position embedding

def rope_frame_position(chunk, frames_per_chunk, shot, offset) -> int:
    """frame_pos0 of a chunk of a multi-shot stream: chunk * frames_per_chunk
    plus multi_shot_rope_offset once per shot switch before it."""
    p = int(load().nvfp4kv_rope_frame_position(int(chunk), int(frames_per_chunk), int(shot),
                                                int(offset)))
    if p < 0:
        raise NvFp4KvError(ERR_INVALID_ARG, "nvfp4kv_rope_frame_position")
    return p


class RopeTable:
    """A chunk's rotation table on the device (nvfp4kv_rope_table) and the
    token grid it covers: `frames` frames of rows x cols tokens."""

    def __init__(self, frames, rows, cols, device="cuda"):
        import torch
        n = int(load().nvfp4kv_rope_table_bytes(frames, rows, cols))
        if n == 0:
            raise NvFp4KvError(ERR_INVALID_ARG, "nvfp4kv_rope_table_bytes")
        self.table = torch.empty(n // 4, dtype=torch.float32, device=device)
        self.view = RopeView(self.table.data_ptr(), frames, rows, cols)
        self.frames, self.rows, self.cols = frames, rows, cols

    def fill(self, frame_pos0, stream=None):
        """Compute the table for a chunk whose first frame is at frame_pos0."""
        _check(load().nvfp4kv_rope_table(int(frame_pos0), self.frames, self.rows, self.cols,
                                         _ptr(self.table), _stream(stream)),
               "nvfp4kv_rope_table")
        return self


def rope(X, table: RopeTable, Y=None, stream=None):
    """Rotate bf16 [T, H, d] X into Y (a new tensor when None; Y = X in place)."""
    import torch
    T, H, d = X.shape
    if Y is None:
        Y = torch.empty_like(X)
    _check(load().nvfp4kv_rope(_ptr(X), _ptr(Y), T, H, d, ctypes.byref(table.view),
                               _stream(stream)), "nvfp4kv_rope")
    return Y


def quantize_chunk_rope(K, V, table: RopeTable, out: ChunkBuffer, ws, stream=None):
    """quantize_chunk of (K rotated by `table`, V), the rotation fused."""
    T, H, d = K.shape
    _check(load().nvfp4kv_quantize_chunk_rope(_ptr(K), _ptr(V), T, H, d,
                                              ctypes.byref(table.view), ctypes.byref(out.view),
                                              _ptr(ws), _stream(stream)),
           "nvfp4kv_quantize_chunk_rope")


def quantize_chunk_noalloc(K, V, out: ChunkBuffer, stream=None):
    """quantize_chunk without a workspace: the library's compiled-in scratch
    (chunks whose scratch exceeds it are refused with ERR_CAPACITY)."""
    T, H, d = K.shape
    _check(load().nvfp4kv_quantize_chunk_noalloc(_ptr(K), _ptr(V), T, H, d,
                                                 ctypes.byref(out.view), _stream(stream)),
           "nvfp4kv_quantize_chunk_noalloc")


def dequantize(chunk: ChunkBuffer, K_out=None, V_out=None, stream=None):
    """Write de-quantized [T_c, H, d] K and/or V: contiguous tensors of one
    dtype (float32 or bf16), the dtype the library writes both in."""
    outs = [t for t in (K_out, V_out) if t is not None]
    if not outs:
        return
    dtype = _dtype_code(outs[0])
    for t in outs:
        if _dtype_code(t) != dtype:
            raise TypeError("K_out and V_out must have the same dtype")
        if not t.is_contiguous() or t.numel() != chunk.T_c * chunk.H * chunk.d:
            raise ValueError(f"output of shape {tuple(t.shape)} is not a contiguous "
                             f"[{chunk.T_c}, {chunk.H}, {chunk.d}] tensor")
    _check(load().nvfp4kv_dequantize(ctypes.byref(chunk.view), chunk.T_c, chunk.H, chunk.d,
                                     _ptr(K_out), _ptr(V_out), dtype, _stream(stream)),
           "nvfp4kv_dequantize")


def attention(chunks, Q, O, ws, softmax_scale=0.0, stream=None):
    """O = softmax(scale Q K^T) V over the listed chunks (ChunkBuffer or ChunkView)."""
    views = [c.view if hasattr(c, "view") else c for c in chunks]
    arr = (ChunkView * max(1, len(views)))(*views)
    first = chunks[0] if chunks else None
    T_c = first.T_c if hasattr(first, "T_c") else 0
    T_q, H, d = Q.shape
    _check_qo(Q, O, H, d)
    _check(load().nvfp4kv_attention(arr, len(views), T_c, H, d, _ptr(Q), T_q, _ptr(O),
                                    _dtype_code(O), float(softmax_scale), _ptr(ws),
                                    _stream(stream)),
           "nvfp4kv_attention")


def fp4q_bytes(T_q, H, d=HEAD_DIM) -> int:
    return int(load().nvfp4kv_fp4q_bytes(T_q, H, d))


def _up256(x):
    return (x + 255) // 256 * 256


class Fp4QBuffer:
    """Device buffer for the NVFP4 queries of attention_fp4q, with views of its
    parts: codes [T_q * H, d/2], scales [T_q * H, d/16] (uint8), tensor_scale
    [1] (float32)."""

    def __init__(self, T_q, H, d=HEAD_DIM, device="cuda"):
        import torch
        n = fp4q_bytes(T_q, H, d)
        if n == 0:
            raise ValueError(f"unsupported query shape ({T_q}, {H}, {d})")
        self.T_q, self.H, self.d = T_q, H, d
        self.buf = torch.zeros(n, dtype=torch.uint8, device=device)
        R = T_q * H
        o_s = _up256(R * d // 2)
        o_t = o_s + _up256(R * d // 16)
        self.codes = self.buf[:R * d // 2].view(R, d // 2)
        self.scales = self.buf[o_s:o_s + R * d // 16].view(R, d // 16)
        self.tensor_scale = self.buf[o_t:o_t + 4].view(torch.float32)

    def to_host(self):
        return dict(codes=self.codes.cpu().numpy(), scales=self.scales.cpu().numpy(),
                    s=float(self.tensor_scale[0].item()))


def attention_fp4q(chunks, Q, O, qbuf: Fp4QBuffer, ws, softmax_scale=0.0, stream=None):
    """attention with the queries quantized to NVFP4 (into qbuf) and Q K^T on
    the block-scaled FP4 tensor cores."""
    views = [c.view if hasattr(c, "view") else c for c in chunks]
    arr = (ChunkView * max(1, len(views)))(*views)
    first = chunks[0] if chunks else None
    T_c = first.T_c if hasattr(first, "T_c") else 0
    T_q, H, d = Q.shape
    _check_qo(Q, O, H, d)
    if (qbuf.T_q, qbuf.H, qbuf.d) != (T_q, H, d):
        raise ValueError(f"query buffer for ({qbuf.T_q}, {qbuf.H}, {qbuf.d}), "
                         f"queries of shape {tuple(Q.shape)}")
    _check(load().nvfp4kv_attention_fp4q(arr, len(views), T_c, H, d, _ptr(Q), T_q, _ptr(O),
                                         _dtype_code(O), float(softmax_scale), _ptr(qbuf.buf),
                                         _ptr(ws), _stream(stream)),
           "nvfp4kv_attention_fp4q")


def attention_fp4q_launches(n_chunks, T_c, H, T_q, d=HEAD_DIM) -> int:
    """Kernels one attention_fp4q call enqueues (2, or 3 with a split tail)."""
    return int(load().nvfp4kv_attention_fp4q_launches(n_chunks, T_c, H, d, T_q))


def check_formats(op, inp, out, n=None, stream=None):
    n = inp.numel() if n is None else n
    _check(load().nvfp4kv_check_formats(op, _ptr(inp), _ptr(out), n, _stream(stream)),
           "nvfp4kv_check_formats")


# ------------------------------------------------------------------ cache

class KVCache:
    """kvcache over torch-allocated device memory (pool + workspace)."""

    def __init__(self, layers, H, T_c, S_g, S_s, W, d=HEAD_DIM, device="cuda", pool=None,
                 ws=None):
        import torch
        L = load()
        self.cfg = KVCacheConfig(layers, H, d, T_c, S_g, S_s, W)
        self.T_c, self.H, self.d, self.layers = T_c, H, d, layers
        n = int(L.kvcache_pool_bytes(ctypes.byref(self.cfg)))
        if n == 0:
            raise NvFp4KvError(ERR_INVALID_ARG, "kvcache_pool_bytes")
        self.pool = pool if pool is not None else torch.empty(n, dtype=torch.uint8, device=device)
        self.ws = ws if ws is not None else torch.zeros(workspace_bytes(T_c, H, d),
                                                        dtype=torch.uint8, device=device)
        self._h = ctypes.c_void_p()
        _check(L.kvcache_create(ctypes.byref(self.cfg), _ptr(self.pool), _ptr(self.ws),
                                ctypes.byref(self._h)), "kvcache_create")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.kvcache_destroy(h)
            self._h = None

    def append(self, layer, K, V, stream=None):
        _check(load().kvcache_append(self._h, layer, _ptr(K), _ptr(V), _stream(stream)),
               "kvcache_append")

    def append_rope(self, layer, K, V, table: "RopeTable", stream=None):
        _check(load().kvcache_append_rope(self._h, layer, _ptr(K), _ptr(V),
                                          ctypes.byref(table.view), _stream(stream)),
               "kvcache_append_rope")

    def advance(self, layer):
        v = ChunkView()
        _check(load().kvcache_advance(self._h, layer, ctypes.byref(v)), "kvcache_advance")
        return v

    def rebind_shot_sink(self, first_chunk_of_shot):
        _check(load().kvcache_rebind_shot_sink(self._h, int(first_chunk_of_shot)),
               "kvcache_rebind_shot_sink")

    def keyset(self, layer):
        ids = (ctypes.c_int64 * MAX_KEY_CHUNKS)()
        cnt = ctypes.c_int()
        _check(load().kvcache_keyset(self._h, layer, ids, ctypes.byref(cnt)), "kvcache_keyset")
        return [int(ids[i]) for i in range(cnt.value)]

    def num_chunks(self, layer):
        n = ctypes.c_int64()
        _check(load().kvcache_num_chunks(self._h, layer, ctypes.byref(n)), "kvcache_num_chunks")
        return int(n.value)

    def chunk_view(self, layer, chunk) -> ChunkView:
        v = ChunkView()
        _check(load().kvcache_chunk_view(self._h, layer, int(chunk), ctypes.byref(v)),
               "kvcache_chunk_view")
        return v

    def chunk(self, layer, chunk) -> ChunkBuffer:
        """Torch views of a stored chunk (device memory of the pool)."""
        v = self.chunk_view(layer, chunk)
        off = v.k_codes - self.pool.data_ptr()
        buf = ChunkBuffer.__new__(ChunkBuffer)
        n = chunk_bytes(self.T_c, self.H, self.d)
        ChunkBuffer.__init__(buf, self.T_c, self.H, self.d, buf=self.pool[off:off + n])
        return buf

    def attention(self, layer, Q, O, softmax_scale=0.0, stream=None):
        T_q = Q.shape[0]
        _check_qo(Q, O, self.H, self.d)
        _check(load().sink_window_attention(self._h, layer, _ptr(Q), T_q, _ptr(O),
                                            _dtype_code(O), float(softmax_scale),
                                            _stream(stream)),
               "sink_window_attention")

    def check_status(self, stream=None) -> int:
        return int(load().kvcache_check_status(self._h, _stream(stream)))

    def get_state(self) -> bytes:
        """The cache's bookkeeping (kvcache_get_state); with a copy of
        self.pool it is a checkpoint."""
        L = load()
        n = int(L.kvcache_state_bytes(self._h))
        buf = ctypes.create_string_buffer(n)
        _check(L.kvcache_get_state(self._h, buf, n), "kvcache_get_state")
        return buf.raw

    def set_state(self, state: bytes):
        """Restore bookkeeping saved by get_state (self.pool must hold the saved
        pool's bytes)."""
        buf = ctypes.create_string_buffer(state, len(state))
        _check(load().kvcache_set_state(self._h, buf, len(state)), "kvcache_set_state")


def default_scale(d=HEAD_DIM):
    return 1.0 / math.sqrt(d)
