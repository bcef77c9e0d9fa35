"""Writes tiny_oracle_regression.npz: the oracle's outputs for the tiny
workload (T=64, H=256, E=8, I=128, top-2, seed 0, logit gap enforced):
a hash of the inputs, the routing, and y for the first 8 tokens.

Calls only the oracle and the seeded input generator.  Run from the
repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_regression.npz")


def compute():
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(cfg)
    oracle.enforce_logit_gap(inp)
    ref = oracle.layer_forward(inp.x, inp.w_router, inp.bias, inp.w_gate_up, inp.w_down, cfg.k)
    import hashlib
    x_sha = np.frombuffer(hashlib.sha256(inp.x.tobytes()).digest(), np.uint8)
    return dict(x_sha256=x_sha, ids=ref["ids"], w=ref["w"], offsets=ref["offsets"],
                sorted_token_ids=ref["sorted_token_ids"], y8=ref["y"][:8])


if __name__ == "__main__":
    np.savez_compressed(OUT, **compute())
    print("wrote", OUT)
