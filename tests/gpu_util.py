"""Helpers for the GPU parity tests: host arrays <-> torch device tensors and the
attention error metrics of the parity bar (relative L2 <= 1e-2 and max-abs
<= 2e-2 against the float64 oracle)."""
import numpy as np

REL_L2_TOL = 1e-2
MAX_ABS_TOL = 2e-2


def dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bf16_to_f64(t) -> np.ndarray:
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def attention_errors(out: np.ndarray, ref: np.ndarray):
    diff = out - ref
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    return rel, float(np.abs(diff).max())


def assert_attention_close(out, ref, what=""):
    rel, mx = attention_errors(out, ref)
    assert rel <= REL_L2_TOL and mx <= MAX_ABS_TOL, f"{what}: rel-L2 {rel:.3e}, max-abs {mx:.3e}"
    return rel, mx


def sample_rows(T: int, n_random: int = 48, seed: int = 0):
    """First/last rows, tile edges of 64 and 128, and random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, T - 1}
    for tile in (64, 128):
        for e in range(tile, T, tile * 7):
            rows |= {e - 1, e}
    rows |= set(rng.integers(0, T, n_random).tolist())
    return sorted(r for r in rows if 0 <= r < T)
