"""Shared helpers of the GPU parity tests: moving the generator's host arrays
to the device and comparing results with the oracle under the layer's
stated tolerances."""
from __future__ import annotations

import numpy as np

# Output tolerance of the layer (bf16 weights and activations, fp32
# accumulation): max |dy| <= 2e-2 * max |y_ref| and relative Frobenius error
# <= 5e-3.  Expected error: two bf16 roundings (h and y), each ~2^-8/sqrt(3)
# relative RMS, give ~0.32% -- inside 0.5% with margin.
Y_MAX_REL = 2e-2
Y_FRO_REL = 5e-3
# Routing weights: fp32 logits differ from the float64 oracle by ~1e-6 at
# H = 8192 (fp32 accumulation of products of size ~0.02); a weight moves by
# at most about twice the largest logit error, so 5e-5 absolute is a wide
# margin that still catches any wrong softmax or renormalisation.
W_ABS = 5e-5


def torch():
    import torch as _t
    return _t


def dev_bf16(bits: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(t.bfloat16).cuda()


def dev_f32(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_i32(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def host_f64(t_) -> np.ndarray:
    return t_.float().cpu().numpy().astype(np.float64)


def rel_errors(got: np.ndarray, ref: np.ndarray) -> tuple[float, float]:
    d = got - ref
    max_rel = float(np.abs(d).max() / max(np.abs(ref).max(), 1e-30))
    fro_rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))
    return max_rel, fro_rel


def assert_close_output(got: np.ndarray, ref: np.ndarray, what: str = "y") -> None:
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    max_rel, fro_rel = rel_errors(got, ref)
    assert max_rel <= Y_MAX_REL and fro_rel <= Y_FRO_REL, \
        f"{what}: max|d|/max|ref| = {max_rel:.3e} (<= {Y_MAX_REL}), rel Frobenius = {fro_rel:.3e} (<= {Y_FRO_REL})"
