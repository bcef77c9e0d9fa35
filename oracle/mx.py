"""Block-scaled FP8 expert weights for the CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU legs may import this
module; it shares no code with the CUDA library.

The weight format (a layer variant with the expert weights stored in 8 bits;
the Qwen-Ironwood page, sec. 6, audits accumulation across FP8 scaling blocks,
and the Ironwood handbook page runs Microscaling formats on Ironwood):

- Element: FP8 E4M3 as defined by the Open Compute Project's 8-bit floating
  point specification -- 1 sign bit, 4 exponent bits with bias 7, 3
  mantissa bits; exponent field 0 encodes subnormals (m/8 * 2^-6); the one
  pattern with all exponent and mantissa bits set is NaN; there are no
  infinities, so the largest finite magnitude is 1.75 * 2^8 = 448.
- Scale: E8M0 as defined by the OCP Microscaling (MX) specification -- an
  unsigned 8-bit power-of-two exponent with bias 127 (2^(c-127)); 0xFF is
  NaN.
- Block: one scale per 32 consecutive weights along the reduction dimension
  (K) of each output column, so a [K, N] weight matrix carries scales
  [K/32, N].

Dequantised weight  W[k, n] = e4m3(code[k, n]) * e8m0(scale[k // 32, n]),
in float64.  A product of a 4-significant-bit value and a power of two is
exactly representable in bf16 whenever it lies in bf16's normal range, so
the layer on these weights is the bf16-weight layer of ``moe_oracle`` on
exactly those values.
"""
from __future__ import annotations

import numpy as np

__all__ = ["e4m3_to_f64", "e8m0_to_f64", "mx_dequant", "MX_BLOCK", "TEST_INFRASTRUCTURE_ONLY"]

TEST_INFRASTRUCTURE_ONLY = True
MX_BLOCK = 32


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode FP8 E4M3 bytes from their bit fields (sign, exponent, mantissa)."""
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    subnormal = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, subnormal, normal)
    return np.where((e == 15) & (m == 7), np.nan, v)


def e8m0_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode E8M0 scale bytes: 2^(c - 127); 0xFF is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    return np.where(c == 255, np.nan, np.exp2(c - 127.0))


def mx_dequant(codes: np.ndarray, scales: np.ndarray, block: int = MX_BLOCK) -> np.ndarray:
    """W [..., K, N] float64 from codes [..., K, N] and scales [..., K/block, N]:
    every weight times the scale of its K block."""
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    K = codes.shape[-2]
    if K % block or scales.shape[-2] != K // block or scales.shape[-1] != codes.shape[-1] \
            or scales.shape[:-2] != codes.shape[:-2]:
        raise ValueError("scales must be [..., K/block, N] for codes [..., K, N]")
    return e4m3_to_f64(codes) * np.repeat(e8m0_to_f64(scales), block, axis=-2)
