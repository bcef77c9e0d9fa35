"""Pins for the block-scaled FP8 weight decoding of the CPU oracle: values
worked by hand from the formats' bit layouts, all 256 codes against
PyTorch's own float8 dtypes (a library decoder), the block structure of the
scales, and the claim that the dequantised weights are exact bf16 values (so
the layer on them is the bf16 layer on those values)."""
import numpy as np
import pytest
import torch

import synth
from oracle import moe_oracle as om
from oracle import mx


def test_e4m3_values_worked_by_hand():
    # sign | exponent (bias 7) | mantissa
    cases = {
        0x00: 0.0,
        0x38: 1.0,             # 0 0111 000
        0x30: 0.5,             # 0 0110 000
        0x3C: 1.5,             # 0 0111 100
        0x44: 3.0,             # 0 1000 100
        0xC0: -2.0,            # 1 1000 000
        0x7E: 448.0,           # 0 1111 110: largest finite
        0x08: 2.0 ** -6,       # smallest normal
        0x01: 2.0 ** -9,       # smallest subnormal: 1/8 * 2^-6
        0x07: 7 * 2.0 ** -9,   # largest subnormal
        0x77: 240.0,           # 0 1110 111: 1.875 * 2^7
    }
    got = mx.e4m3_to_f64(np.array(list(cases), np.uint8))
    assert got.tolist() == list(cases.values())
    neg0 = mx.e4m3_to_f64(np.array([0x80], np.uint8))[0]
    assert neg0 == 0.0 and np.signbit(neg0)
    assert np.isnan(mx.e4m3_to_f64(np.array([0x7F, 0xFF], np.uint8))).all()
    assert not np.isnan(mx.e4m3_to_f64(np.array([0x7E, 0x78, 0xFE], np.uint8))).any()


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = mx.e4m3_to_f64(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])
    # positive codes increase strictly; negative codes mirror them
    pos = got[:0x7F]
    assert np.all(np.diff(pos) > 0)
    np.testing.assert_array_equal(got[0x80:0xFF], -pos)


def test_e8m0_values_and_all_codes_match_torch():
    assert mx.e8m0_to_f64(np.array([127, 128, 126, 0, 254], np.uint8)).tolist() == \
        [1.0, 2.0, 0.5, 2.0 ** -127, 2.0 ** 127]
    assert np.isnan(mx.e8m0_to_f64(np.array([255], np.uint8))[0])
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = mx.e8m0_to_f64(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    np.testing.assert_array_equal(got[:255], want[:255])


def test_dequant_scales_act_on_their_k_block_only():
    K, N = 96, 5
    codes = synth.fp8_e4m3_codes(0, 99, 0, (K, N))
    scales = np.full((K // 32, N), 127, np.uint8)
    base = mx.mx_dequant(codes, scales)
    np.testing.assert_array_equal(base, mx.e4m3_to_f64(codes))   # unit scales: plain decode
    b, n = 1, 3
    s2 = scales.copy()
    s2[b, n] = 127 + 3                                            # x8 on one block of one column
    got = mx.mx_dequant(codes, s2)
    changed = np.zeros((K, N), bool)
    changed[32 * b:32 * (b + 1), n] = True
    np.testing.assert_array_equal(got[changed], 8 * base[changed])
    np.testing.assert_array_equal(got[~changed], base[~changed])
    with pytest.raises(ValueError):
        mx.mx_dequant(codes, scales[:2])
    with pytest.raises(ValueError):
        mx.mx_dequant(codes[:90], scales)
    # leading (expert) dimensions broadcast block by block
    codes3 = np.stack([codes, codes])
    scales3 = np.stack([scales, s2])
    out = mx.mx_dequant(codes3, scales3)
    np.testing.assert_array_equal(out[0], base)
    np.testing.assert_array_equal(out[1], got)


def test_dequantised_weights_are_exact_bf16_values():
    codes = np.arange(256, dtype=np.uint8).reshape(256, 1).repeat(32, axis=0).reshape(256 * 32, 1)
    finite = ~np.isnan(mx.e4m3_to_f64(codes[:, 0]))
    codes = codes[finite]
    codes = codes[: (len(codes) // 32) * 32]
    for sc in (127 - 60, 127 - 9, 127, 127 + 40):
        scales = np.full((len(codes) // 32, 1), sc, np.uint8)
        w = mx.mx_dequant(codes, scales)
        back = om.bf16_to_f64(synth.bf16_from_f32(w.astype(np.float32)))
        np.testing.assert_array_equal(back, w)


def test_exact_bf16_range_of_the_scale_codes():
    """Every finite E4M3 value times 2^(c - 127) is a bf16 number exactly for
    scale codes 3..246, and for no wider range: below 3 the smallest values
    (2^-9 * 2^(c-127)) fall under bf16's least subnormal step 2^-133; above
    246 the largest (448 * 2^(c-127)) pass bf16's largest finite value
    (1.9921875 * 2^127).  Checked over all 254 finite codes and all 255
    finite scale codes by widening back from bf16."""
    codes = np.arange(256, dtype=np.uint8)
    vals = mx.e4m3_to_f64(codes)
    vals = vals[~np.isnan(vals)]
    assert len(vals) == 254
    exact = []
    for c in range(255):
        w = vals * 2.0 ** (c - 127)
        back = torch.from_numpy(w).float().to(torch.bfloat16).double().numpy()
        exact.append(bool(np.array_equal(back, w)))
    assert [c for c in range(255) if exact[c]] == list(range(3, 247))
    # the two limits, worked by hand
    assert 2.0 ** -9 * 2.0 ** (2 - 127) == 2.0 ** -134 < 2.0 ** -133
    assert 448 * 2.0 ** (247 - 127) == 1.75 * 2.0 ** 128 > 1.9921875 * 2.0 ** 127


def test_mx_layer_is_bf16_layer_on_the_same_values():
    """The layer on dequantised fp8 weights equals the oracle's bf16-weight
    layer fed the same values as bf16 bit patterns (exact, no tolerance)."""
    cfg = synth.Config("mx_small", T=24, H=256, E=4, I=128, k=2)
    inp = synth.make_inputs(cfg, experts=False)
    gu = [synth.mx_expert_weights(cfg, e, "gate_up") for e in range(cfg.E)]
    dn = [synth.mx_expert_weights(cfg, e, "down") for e in range(cfg.E)]
    w_gu = np.stack([mx.mx_dequant(c, s) for c, s in gu])
    w_dn = np.stack([mx.mx_dequant(c, s) for c, s in dn])
    assert w_gu.shape == (cfg.E, cfg.H, 2 * cfg.I) and w_dn.shape == (cfg.E, cfg.I, cfg.H)
    assert 0.005 < w_gu.std() < 0.2                 # magnitudes near the bf16 weights'
    y_mx = om.layer_forward(inp.x, inp.w_router, None, w_gu, w_dn, cfg.k)["y"]
    bits_gu = synth.bf16_from_f32(w_gu.astype(np.float32)).reshape(w_gu.shape)
    bits_dn = synth.bf16_from_f32(w_dn.astype(np.float32)).reshape(w_dn.shape)
    y_bf = om.layer_forward(inp.x, inp.w_router, None, bits_gu, bits_dn, cfg.k)["y"]
    np.testing.assert_array_equal(y_mx, y_bf)


def test_fp8_code_generator_is_finite_keyed_and_in_range():
    a = synth.fp8_e4m3_codes(0, 11, 5, (64, 64))
    b = synth.fp8_e4m3_codes(0, 11, 5, (64, 64))
    c = synth.fp8_e4m3_codes(0, 11, 6, (64, 64))
    np.testing.assert_array_equal(a, b)
    assert (a != c).any()
    e = (a >> 3) & 0xF
    assert e.min() >= 3 and e.max() <= 9
    assert not np.isnan(mx.e4m3_to_f64(a)).any()
    with pytest.raises(ValueError):
        synth.fp8_e4m3_codes(0, 11, 5, (4,), exp_hi=15)
    s = synth.e8m0_scale_codes(0, 13, 0, (8, 8))
    assert s.min() >= 118 and s.max() <= 122


# ---------------------------------------------------------------- quantisation (E4M3 encode, MX blocks)

def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = mx.e4m3_to_f64(codes)
    ok = ~np.isnan(vals)
    np.testing.assert_array_equal(mx.e4m3_encode(vals[ok]), codes[ok])   # -0 keeps its sign bit
    with pytest.raises(ValueError):
        mx.e4m3_encode(np.array([np.nan]))


def test_e4m3_encode_ties_and_saturation_worked_by_hand():
    cases = {
        1.0625: 0x38,           # halfway 1.0 | 1.125 -> even mantissa 000
        1.1875: 0x3A,           # halfway 1.125 | 1.25 -> even mantissa 010
        2.0 ** -10: 0x00,       # halfway 0 | 2^-9 -> 0
        3 * 2.0 ** -11: 0x01,   # 0.75 * 2^-9 -> 2^-9
        15 * 2.0 ** -10: 0x08,  # halfway 7*2^-9 | 2^-6 -> the smallest normal (even)
        440.0: 0x7E,            # nearest is 448
        470.0: 0x7E,            # above 448: clamped
        1e6: 0x7E,
        -500.0: 0xFE,
        -3.3: 0xC5,             # 1 1000 101 = -3.25
    }
    got = mx.e4m3_encode(np.array(list(cases)))
    assert [hex(c) for c in got] == [hex(c) for c in cases.values()]


def test_e4m3_encode_matches_torch_below_its_overflow():
    """PyTorch's float8_e4m3fn cast rounds to nearest-even too; it turns
    magnitudes from 464 up into NaN, where the MX rule clamps, so the
    comparison stays below 464."""
    rng = np.random.default_rng(41)
    v = rng.uniform(-463.9, 463.9, 200_000) * np.exp2(rng.integers(-16, 1, 200_000))
    v = v.astype(np.float32)
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(mx.e4m3_encode(v.astype(np.float64)), want)


def test_mx_quantize_scale_rule():
    v = np.zeros((96, 4))
    v[:32, 0] = np.linspace(-1.0, 1.0, 32)           # amax 1: floor(log2 1) - 8 = -8
    v[32:64, 1] = 448.0 * 4 * np.sign(np.arange(32) - 15.5)   # amax 448 * 2^2: exact
    v[64:, 2] = 500.0                                # amax 500: shared exponent 0, 500 clamps to 448
    codes, scales = mx.mx_quantize(v)
    assert scales[0, 0] == 127 - 8 and scales[1, 1] == 127 + 2 and scales[2, 2] == 127
    assert scales[1, 0] == 0 and scales[0, 3] == 0     # all-zero blocks take the smallest scale
    deq = mx.mx_dequant(codes, scales)
    np.testing.assert_array_equal(deq[32:64, 1], v[32:64, 1])
    assert np.all(deq[64:, 2] == 448.0)
    assert np.all(deq[:, 3] == 0.0) and np.all(codes[:, 3] == 0)


def test_mx_quantize_error_bound():
    """Three mantissa bits: relative error <= 2^-4 in the normal range, and
    absolute error <= half a subnormal step (2^-10 of the scale) below it."""
    rng = np.random.default_rng(42)
    v = rng.standard_normal((256, 16)) * np.exp2(rng.integers(-20, 20, (8, 1, 16))).repeat(32, axis=0).reshape(256, 16)
    codes, scales = mx.mx_quantize(v)
    deq = mx.mx_dequant(codes, scales)
    X = np.repeat(mx.e8m0_to_f64(scales), 32, axis=0)
    p = np.abs(v) / X
    normal = (p >= 2.0 ** -6) & (p <= 448.0)
    assert np.all(np.abs(deq - v)[normal] <= 2.0 ** -4 * np.abs(v)[normal])
    sub = p < 2.0 ** -6
    assert np.all(np.abs(deq - v)[sub] <= 2.0 ** -10 * X[sub])
    assert np.all(p <= 512.0)                          # the largest element of a block scales into [256, 512)
