"""Write tiny_chunk0_digest.json: SHA-256 digests of the oracle's quantization
of chunk 0 of the tiny configuration (H=2, d=128, T_c=32, seed 0).

Calls only oracle/ and synth/.  Rerun only after a change to the oracle's
arithmetic that a cited passage (or its stated reading) justifies.
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402


def digest():
    K, V, _ = synth.tiny_chunk(0)
    q = oracle.quantize_chunk(K, V)
    out = {"_source": "oracle quantization of tiny-config chunk 0 (make_tiny_digest.py)"}
    for k in ("k_codes", "k_scales", "v_codes", "v_scales", "k_mean"):
        out[k] = hashlib.sha256(q[k].tobytes()).hexdigest()
    out["s_k"] = float(q["s_k"])
    out["s_v"] = float(q["s_v"])
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_chunk0_digest.json"), "w") as f:
        json.dump(digest(), f, indent=1)
        f.write("\n")
