"""Helpers for the GPU parity tests: host arrays <-> torch device tensors and the
attention error metrics of the parity bar (relative L2 <= 1e-2 and max-abs
<= 2e-2 against the float64 oracle)."""
import numpy as np

REL_L2_TOL = 1e-2
MAX_ABS_TOL = 2e-2


def dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_to_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


host_bf16_to_f64 = host_to_f64


def attention_errors(out: np.ndarray, ref: np.ndarray):
    diff = out - ref
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    return rel, float(np.abs(diff).max())


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x|: the most that rounding x to bf16 moves it."""
    a = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(a)) - 8)


def assert_attention_close(out, ref, what="", bf16_output=False):
    """rel-L2 <= 1e-2 and |out - ref| <= 2e-2 element-wise; a bf16 output may in
    addition carry its own rounding, half a bf16 ulp of the value."""
    rel, _ = attention_errors(out, ref)
    err = np.abs(out - ref)
    allow = MAX_ABS_TOL + (bf16_half_ulp(np.maximum(np.abs(ref), np.abs(out)))
                           if bf16_output else 0.0)
    worst = float((err - allow).max())
    assert rel <= REL_L2_TOL and worst <= 0, \
        f"{what}: rel-L2 {rel:.3e}, max-abs {err.max():.3e} (excess {worst:.3e})"
    return rel, float(err.max())


def sample_rows(T: int, n_random: int = 48, seed: int = 0):
    """First/last rows, tile edges of 64 and 128, and random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, T - 1}
    for tile in (64, 128):
        for e in range(tile, T, tile * 7):
            rows |= {e - 1, e}
    rows |= set(rng.integers(0, T, n_random).tolist())
    return sorted(r for r in rows if 0 <= r < T)


# ------------------------------------------------------------------ output canaries

SENTINEL = 0xA5
GUARD_BYTES = 4096


class Guarded:
    """A device tensor of `shape` and `dtype` with GUARD_BYTES of sentinel bytes
    right before and after it (its own bytes start as the sentinel too)."""

    def __init__(self, shape, dtype):
        import torch
        self.nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.big = torch.full((2 * GUARD_BYTES + self.nbytes,), SENTINEL, dtype=torch.uint8,
                              device="cuda")
        self.t = self.big[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(shape)

    def assert_intact(self, what=""):
        b = self.big.cpu().numpy()
        head, tail = b[:GUARD_BYTES], b[GUARD_BYTES + self.nbytes:]
        assert (head == SENTINEL).all() and (tail == SENTINEL).all(), \
            f"{what}: a store landed outside the output " \
            f"(guard bytes changed before: {int((head != SENTINEL).sum())}, " \
            f"after: {int((tail != SENTINEL).sum())})"


class GuardedChunk:
    """A ChunkBuffer carved from a sentinel-filled buffer with GUARD_BYTES on
    either side; every byte outside the six parts' exact extents (the guards
    and the alignment padding between parts) must stay the sentinel."""

    def __init__(self, lib, T, H):
        import torch
        n = lib.chunk_bytes(T, H)
        self.big = torch.full((2 * GUARD_BYTES + n + 256,), SENTINEL, dtype=torch.uint8,
                              device="cuda")
        self.chunk = lib.ChunkBuffer(T, H, buf=self.big[GUARD_BYTES:GUARD_BYTES + n + 256])

    def assert_intact(self, what=""):
        c = self.chunk
        mask = np.ones(self.big.numel(), bool)
        b0 = self.big.data_ptr()
        for t in (c.k_codes, c.v_codes, c.k_scales, c.v_scales, c.k_mean, c.tensor_scales):
            a = t.data_ptr() - b0
            mask[a:a + t.numel() * t.element_size()] = False
        rest = self.big.cpu().numpy()[mask]
        bad = int((rest != SENTINEL).sum())
        assert bad == 0, f"{what}: {bad} bytes outside the chunk's parts changed"
