"""Seeded synthetic inputs for the routed-expert MoE layer.

This module is the one piece shared by the CUDA path's tests/bench and the
CPU oracle.  It draws random tensors and nothing else: it holds none of the
layer's arithmetic (no logits, no softmax, no top-k, no FFN).

Generator: numpy's SFC64 bit generator (Doty-Humphrey's Small Fast Chaotic
PRNG) keyed by numpy's SeedSequence hash of (seed, tensor id, slice index),
followed by numpy's ziggurat ``standard_normal``.  Every slice (one expert's
weight matrix, one row block of ``x``) has its own counter key, so any slice
can be regenerated on its own -- a parity test can rebuild exactly the
experts a sampled token touches without drawing the whole weight set.

bf16 tensors are produced by drawing fp32 normals, scaling, and rounding to
bf16 with round-to-nearest-even; they are returned as ``uint16`` bit
patterns, which both sides read byte for byte.

Workload shapes and distributions follow the configurations quoted with the
layer's headline metric (tiny, Qwen-3.5-like decode/prefill, Ling-like skewed
prefill with a shared expert, small-batch decode sweep).  The pages'
workloads are 8K-in/1K-out prefill and 1K-in/8K-out decode (pwwt.cn page,
sec. 5.1) on 512-expert top-10 and 256-expert top-8 + shared-expert models
(pwwt.cn sec. 2-4; lumevalley.com page, intro); no dataset is involved.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

__all__ = [
    "Config", "CONFIGS", "TID", "bf16_from_f32", "normal_bf16", "normal_f32",
    "uniform_bf16", "Inputs", "make_inputs", "zipf_bias", "redraw_x_rows",
    "fill_expert_weights", "fp8_e4m3_codes", "e8m0_scale_codes", "mx_expert_weights", "MX_BLOCK",
]

# Tensor ids: the second word of every counter key.
TID = dict(x=1, w_router=2, w_gate_up=3, w_down=4, w_sh_gate_up=5, w_sh_down=6,
           x_redraw=7, h_stage=8, topk_w_stage=9, misc=10,
           mx_gate_up=11, mx_down=12, mx_gate_up_scale=13, mx_down_scale=14)


@dataclass(frozen=True)
class Config:
    """Shape and distribution of one MoE-layer workload.

    T tokens, hidden H, E routed experts, expert intermediate I, top-k,
    optional shared expert with intermediate I_s (0 = none), and the router
    bias recipe ("none" or "zipf:<s>", bias_e = -s*ln(e+1)).
    """
    name: str
    T: int
    H: int
    E: int
    I: int
    k: int
    I_s: int = 0
    bias: str = "none"
    x_std: float = 1.0
    w_std: float = 0.02
    router_std: float = 0.02
    seed: int = 0
    note: str = field(default="", compare=False)

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)

    @property
    def has_shared(self) -> bool:
        return self.I_s > 0


CONFIGS: dict[str, Config] = {
    c.name: c for c in [
        Config("tiny", T=64, H=256, E=8, I=128, k=2,
               note="T=64, H=256, E=8, I=128, top-2; x~N(0,1) bf16, router N(0,.02) f32, "
                    "experts N(0,.02) bf16, seed 0, no shared expert"),
        Config("qwen_decode_t512", T=512, H=4096, E=512, I=1024, k=10,
               note="decode step, one token per request; ~12.9 GB expert weights; HBM-bound"),
        Config("qwen_prefill_t8192", T=8192, H=4096, E=512, I=1024, k=10,
               note="prefill chunk; same weights as the decode config; 81,920 permuted rows"),
        Config("ling_skewed_t4096", T=4096, H=8192, E=256, I=2048, k=8, I_s=2048,
               bias="zipf:1.2",
               note="top-8 + always-active shared expert; per-expert router bias "
                    "-1.2*ln(rank) so a few hot experts draw most tokens"),
        *[Config(f"sweep_decode_t{t}", T=t, H=4096, E=256, I=1536, k=8,
                 note="small-batch decode sweep: few experts active, pure weight streaming")
          for t in (1, 4, 16, 64)],
        # Reduced expert counts with the per-expert row counts of the decode
        # (~10 rows) and prefill (~160 rows) shapes: 1.6 GB of weights, larger
        # than L2 but small enough for multi-pass profiler captures.
        Config("prof_decode_e64", T=64, H=4096, E=64, I=1024, k=10,
               note="profiling case: decode-like rows per expert, 64 experts"),
        Config("prof_prefill_e64", T=1024, H=4096, E=64, I=1024, k=10,
               note="profiling case: prefill-like rows per expert, 64 experts"),
    ]
}


def bf16_from_f32(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even); returns uint16 bits.

    Inputs are finite normals, so no NaN special case is needed.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).copy()
    u += ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return (u >> 16).astype(np.uint16)


def _gen(seed: int, tid: int, idx: int) -> np.random.Generator:
    return np.random.Generator(np.random.SFC64(np.random.SeedSequence([seed, tid, idx])))


def normal_f32(seed: int, tid: int, idx: int, shape, std: float) -> np.ndarray:
    a = _gen(seed, tid, idx).standard_normal(int(np.prod(shape)), dtype=np.float32)
    a *= np.float32(std)
    return a.reshape(shape)


def normal_bf16(seed: int, tid: int, idx: int, shape, std: float) -> np.ndarray:
    return bf16_from_f32(normal_f32(seed, tid, idx, shape, std)).reshape(shape)


def uniform_bf16(seed: int, tid: int, idx: int, shape, lo: float, hi: float) -> np.ndarray:
    a = _gen(seed, tid, idx).uniform(lo, hi, int(np.prod(shape))).astype(np.float32)
    return bf16_from_f32(a).reshape(shape)


def zipf_bias(E: int, s: float) -> np.ndarray:
    """Router bias for the skewed config: bias_e = -s * ln(rank_e), rank_e = e + 1.

    The log of the Zipf normaliser is the same for every expert, so it is
    left out (a constant logit shift changes neither softmax nor top-k).
    """
    return (-s * np.log(np.arange(1, E + 1, dtype=np.float64))).astype(np.float32)


def _bias(cfg: Config) -> np.ndarray | None:
    if cfg.bias == "none":
        return None
    kind, _, arg = cfg.bias.partition(":")
    if kind == "zipf":
        return zipf_bias(cfg.E, float(arg))
    raise ValueError(f"unknown bias recipe {cfg.bias!r}")


_X_BLOCK = 256  # x is drawn in blocks of rows, each block its own counter key


def make_x(cfg: Config) -> np.ndarray:
    T, H = cfg.T, cfg.H
    out = np.empty((T, H), np.uint16)
    for b in range(0, T, _X_BLOCK):
        n = min(_X_BLOCK, T - b)
        out[b:b + n] = normal_bf16(cfg.seed, TID["x"], b // _X_BLOCK, (_X_BLOCK, H), cfg.x_std)[:n]
    return out


def redraw_x_rows(cfg: Config, x: np.ndarray, rows, attempt: int) -> None:
    """Replace the given rows of x (in place) with fresh draws.

    Row r on attempt a comes from counter key (seed, x_redraw, a*2^32 + r), so
    the result depends only on which rows are redrawn and how often -- never on
    the CUDA path.  Which rows to redraw is decided by the caller.
    """
    for r in rows:
        x[r] = normal_bf16(cfg.seed, TID["x_redraw"], (attempt << 32) | int(r), (cfg.H,), cfg.x_std)


def expert_gate_up(cfg: Config, e: int) -> np.ndarray:
    """W_gate_up[e] as [H, 2I] bf16 bits; columns [0,I) gate, [I,2I) up."""
    return normal_bf16(cfg.seed, TID["w_gate_up"], e, (cfg.H, 2 * cfg.I), cfg.w_std)


def expert_down(cfg: Config, e: int) -> np.ndarray:
    """W_down[e] as [I, H] bf16 bits."""
    return normal_bf16(cfg.seed, TID["w_down"], e, (cfg.I, cfg.H), cfg.w_std)


def fill_expert_weights(cfg: Config, which: str, out: np.ndarray, experts=None,
                        threads: int | None = None) -> None:
    """Fill ``out`` ([E, H, 2I] for "gate_up", [E, I, H] for "down", uint16)
    expert by expert, on a thread pool (numpy's generators release the GIL)."""
    fn = {"gate_up": expert_gate_up, "down": expert_down}[which]
    experts = range(cfg.E) if experts is None else experts
    threads = threads or min(32, os.cpu_count() or 1)

    def one(e):
        out[e] = fn(cfg, e)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(one, experts))


# ---------------------------------------------------------------- block-scaled fp8 weights
# Codes only: random bit fields, no quantisation of any real-valued tensor.
MX_BLOCK = 32  # weights along the reduction dimension that share one scale


def fp8_e4m3_codes(seed: int, tid: int, idx: int, shape, exp_lo: int = 3, exp_hi: int = 9) -> np.ndarray:
    """Random FP8 E4M3 bytes: sign bit uniform, exponent field uniform in
    [exp_lo, exp_hi], mantissa field uniform in [0, 7]; exp_hi <= 14 keeps
    every code finite."""
    if not 0 <= exp_lo <= exp_hi <= 14:
        raise ValueError("exponent field range must lie in [0, 14]")
    g = _gen(seed, tid, idx)
    n = int(np.prod(shape))
    sign = g.integers(0, 2, n, dtype=np.uint8)
    expo = g.integers(exp_lo, exp_hi + 1, n, dtype=np.uint8)
    mant = g.integers(0, 8, n, dtype=np.uint8)
    return ((sign << 7) | (expo << 3) | mant).astype(np.uint8).reshape(shape)


def e8m0_scale_codes(seed: int, tid: int, idx: int, shape, lo: int = 118, hi: int = 122) -> np.ndarray:
    """Random E8M0 scale bytes (power-of-two exponents, bias 127), uniform in [lo, hi]."""
    if not 0 <= lo <= hi <= 254:
        raise ValueError("scale codes must lie in [0, 254]")
    return _gen(seed, tid, idx).integers(lo, hi + 1, int(np.prod(shape)), dtype=np.uint8).reshape(shape)


def mx_expert_weights(cfg: Config, e: int, which: str) -> tuple[np.ndarray, np.ndarray]:
    """One expert's block-scaled fp8 weights: codes [K, N] uint8 and scale codes
    [K / MX_BLOCK, N] uint8, K the reduction dimension (gate_up: K = H,
    N = 2I; down: K = I, N = H).  Magnitudes come out near the bf16 weights'
    (exponent fields 3..9 times scales 2^-9..2^-5)."""
    K, N = {"gate_up": (cfg.H, 2 * cfg.I), "down": (cfg.I, cfg.H)}[which]
    if K % MX_BLOCK:
        raise ValueError("reduction dimension must be a multiple of the scale block")
    codes = fp8_e4m3_codes(cfg.seed, TID["mx_" + which], e, (K, N))
    scales = e8m0_scale_codes(cfg.seed, TID["mx_" + which + "_scale"], e, (K // MX_BLOCK, N))
    return codes, scales


@dataclass
class Inputs:
    """All layer inputs as host arrays; bf16 tensors are uint16 bit patterns."""
    cfg: Config
    x: np.ndarray                   # [T, H] bf16
    w_router: np.ndarray            # [H, E] f32
    bias: np.ndarray | None         # [E] f32 or None
    w_gate_up: np.ndarray | None    # [E, H, 2I] bf16 (None when not materialised)
    w_down: np.ndarray | None       # [E, I, H] bf16
    w_sh_gate_up: np.ndarray | None  # [H, 2 I_s] bf16
    w_sh_down: np.ndarray | None     # [I_s, H] bf16
    redraws: int = 0                # rows of x replaced by redraw_x_rows


def make_inputs(cfg: Config, experts: bool = True, threads: int | None = None) -> Inputs:
    """Draw every input of ``cfg``.  With experts=False the routed expert
    weights are left out (callers then draw single experts on demand)."""
    x = make_x(cfg)
    w_router = normal_f32(cfg.seed, TID["w_router"], 0, (cfg.H, cfg.E), cfg.router_std)
    wgu = wd = None
    if experts:
        wgu = np.empty((cfg.E, cfg.H, 2 * cfg.I), np.uint16)
        wd = np.empty((cfg.E, cfg.I, cfg.H), np.uint16)
        fill_expert_weights(cfg, "gate_up", wgu, threads=threads)
        fill_expert_weights(cfg, "down", wd, threads=threads)
    sgu = sd = None
    if cfg.has_shared:
        sgu = normal_bf16(cfg.seed, TID["w_sh_gate_up"], 0, (cfg.H, 2 * cfg.I_s), cfg.w_std)
        sd = normal_bf16(cfg.seed, TID["w_sh_down"], 0, (cfg.I_s, cfg.H), cfg.w_std)
    return Inputs(cfg, x, w_router, _bias(cfg), wgu, wd, sgu, sd)


def gap_target() -> float:
    """Minimum gap between adjacent logits among each token's top k+1."""
    return 1e-3


def describe(cfg: Config) -> str:
    return (f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} I={cfg.I} k={cfg.k}"
            + (f" I_s={cfg.I_s}" if cfg.I_s else "") + f" bias={cfg.bias} seed={cfg.seed}")


def expert_weight_bytes(cfg: Config) -> int:
    return cfg.E * 3 * cfg.H * cfg.I * 2


def _check():  # pragma: no cover - quick manual sanity
    c = CONFIGS["tiny"]
    i = make_inputs(c)
    assert i.x.shape == (c.T, c.H) and math.isfinite(float(i.w_router.sum()))
