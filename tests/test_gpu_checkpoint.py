"""Checkpoint and resume of the cache (kvcache_get_state / kvcache_set_state plus
a copy of the pool): a cache rebuilt from a checkpoint over a copied pool
continues the stream exactly as the original does -- the same key sets and
bit-identical attention outputs -- and matches the float64 oracle."""
import numpy as np
import pytest

import synth
from gpu_util import assert_attention_close, dev_bf16

pytestmark = pytest.mark.gpu


def test_resume_from_checkpoint_continues_identically(lib, orc):
    import torch
    T_c, H, S_g, S_s, W = 64, 2, 1, 1, 2
    a = lib.KVCache(1, H, T_c, S_g, S_s, W)
    q = {}
    chunk = lambda n: (synth.k_with_offsets_bf16(40 + n, 0, n, (T_c, H, 128)),
                       synth.gaussian_bf16(40 + n, 0, n, synth.T_V, (T_c, H, 128)))
    for n in range(5):
        if n == 3:
            a.rebind_shot_sink(3)
        K, V = chunk(n)
        a.append(0, dev_bf16(K), dev_bf16(V))
        q[n] = orc.quantize_chunk(K, V)
    torch.cuda.synchronize()
    state = a.get_state()
    b = lib.KVCache(1, H, T_c, S_g, S_s, W, pool=a.pool.clone())
    b.set_state(state)
    assert b.keyset(0) == a.keyset(0) and b.num_chunks(0) == a.num_chunks(0)
    for n in (5, 6):
        K, V = chunk(n)
        for c in (a, b):
            c.append(0, dev_bf16(K), dev_bf16(V))
        q[n] = orc.quantize_chunk(K, V)
        assert a.keyset(0) == b.keyset(0)
        Q = synth.gaussian_bf16(60 + n, 0, n, synth.T_Q, (T_c, H, 128))
        outs = []
        for c in (a, b):
            O = torch.empty((T_c, H, 128), dtype=torch.float32, device="cuda")
            c.attention(0, dev_bf16(Q), O)
            torch.cuda.synchronize()
            assert c.check_status() == lib.OK
            outs.append(O.cpu().numpy())
        assert np.array_equal(outs[0].view(np.uint32), outs[1].view(np.uint32))
        ids = b.keyset(0)
        assert_attention_close(outs[1].astype(np.float64), orc.attention_f64([q[i] for i in ids], Q),
                               f"resumed cache, chunk {n}")
