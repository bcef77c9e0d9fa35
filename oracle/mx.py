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

Quantisation (for operands that must be brought into the format, e.g. token
rows if the tensor cores take both operands in fp8), following the OCP MX
specification's conversion of a block: the shared exponent is
floor(log2(max |v|)) minus the element format's largest exponent (8 for
E4M3); every element is divided by that power of two, rounded to the
nearest E4M3 value (ties to even mantissa) and, if its magnitude exceeds
448, clamped to 448.  An all-zero block takes the smallest scale.

Dequantised weight  W[k, n] = e4m3(code[k, n]) * e8m0(scale[k // 32, n]),
in float64.  A product of a 4-significant-bit value and a power of two is
exactly representable in bf16 whenever it lies in bf16's normal range, so
the layer on these weights is the bf16-weight layer of ``moe_oracle`` on
exactly those values.
"""
from __future__ import annotations

import numpy as np

__all__ = ["e4m3_to_f64", "e8m0_to_f64", "mx_dequant", "e4m3_encode", "mx_quantize", "MX_BLOCK",
           "TEST_INFRASTRUCTURE_ONLY"]

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


E4M3_MAX = 448.0
E4M3_EMAX = 8


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code of each float64 value (ties to the even mantissa),
    magnitudes above 448 clamped to 448; the sign of zero is kept."""
    v = np.asarray(v, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("NaN has no place in a quantised operand")
    a = np.abs(v)
    sign = np.signbit(v).astype(np.int64) << 7
    frac, ex = np.frexp(a)                    # a = frac * 2^ex, frac in [0.5, 1)
    e = ex - 1                                # a = (2 frac) * 2^e, 2 frac in [1, 2)
    normal = (e >= -6) & (a > 0)
    # normal range: 3 mantissa bits; a carry out of the mantissa bumps the exponent
    q = np.round((2.0 * frac - 1.0) * 8.0).astype(np.int64)
    carry = q == 8
    e_n = np.where(carry, e + 1, e)
    q_n = np.where(carry, 0, q)
    code_n = ((e_n + 7) << 3) | q_n
    # subnormal range: multiples of 2^-9 (a count of 8 is the smallest normal, code 0x08)
    code_s = np.round(a / 2.0 ** -9).astype(np.int64)
    code = np.where(normal, code_n, code_s)
    code = np.where((a > E4M3_MAX) | (code > 0x7E), 0x7E, code)
    return (sign | code).astype(np.uint8)


def mx_quantize(v: np.ndarray, block: int = MX_BLOCK) -> tuple[np.ndarray, np.ndarray]:
    """Codes [..., K, N] and E8M0 scale codes [..., K/block, N] of values
    [..., K, N], one scale per block of `block` values along K."""
    v = np.asarray(v, dtype=np.float64)
    K = v.shape[-2]
    if K % block:
        raise ValueError("K must be a multiple of the block")
    blocks = v.reshape(v.shape[:-2] + (K // block, block, v.shape[-1]))
    amax = np.abs(blocks).max(axis=-2)                       # [..., K/block, N]
    _, ex = np.frexp(amax)
    shared = np.where(amax > 0, ex - 1 - E4M3_EMAX, -127)     # floor(log2 amax) - emax
    shared = np.clip(shared, -127, 127)
    scaled = blocks / np.exp2(shared.astype(np.float64))[..., None, :]
    codes = e4m3_encode(scaled).reshape(v.shape)
    return codes, (shared + 127).astype(np.uint8)
