"""Logit-gap guarantee for parity inputs -- TEST INFRASTRUCTURE ONLY.

Bit-exact routing needs every token's top-k to be decided by a margin far
above fp32 rounding: the GPU computes logits in fp32, the oracle in float64.
A token passes when, among its k+1 largest float64 selection keys (the
logits with their bias; sigmoid(logit) + bias under sigmoid scoring), every
adjacent pair differs by at least ``gap``; this fixes both the selected set
and its descending order.  Failing rows of x are redrawn from fresh
counter keys of the seeded generator until every token passes.
"""
from __future__ import annotations

import numpy as np

import synth

from .moe_oracle import router_logits, selection_keys


def bad_gap_rows(x_bits, w_router, bias, k, gap, scoring="softmax") -> np.ndarray:
    l = selection_keys(router_logits(x_bits, w_router, None), bias, scoring)
    m = min(k + 1, l.shape[1])
    top = -np.sort(-l, axis=1)[:, :m]
    if m < 2:
        return np.zeros(0, np.int64)
    d = top[:, :-1] - top[:, 1:]
    return np.nonzero(d.min(axis=1) < gap)[0]


def enforce_logit_gap(inputs: "synth.Inputs", gap: float | None = None, max_attempts: int = 64,
                      scoring: str = "softmax") -> int:
    """Redraw rows of inputs.x in place until every token has the gap.
    Returns the number of row redraws (also stored in inputs.redraws)."""
    gap = synth.gap_target() if gap is None else gap
    cfg = inputs.cfg
    total = 0
    for attempt in range(1, max_attempts + 1):
        bad = bad_gap_rows(inputs.x, inputs.w_router, inputs.bias, cfg.k, gap, scoring)
        if bad.size == 0:
            inputs.redraws += total
            return total
        synth.redraw_x_rows(cfg, inputs.x, bad, attempt)
        total += int(bad.size)
    raise RuntimeError("logit gap not reached after %d attempts" % max_attempts)
