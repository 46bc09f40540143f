"""Pins of the oracle's FP8 E4M3 comparator (reading R8: the lossy
alternative of the summary's chapter "Lossless or FP8").

* the format's defining values (OCP 8-bit floating point, E4M3): 448, 1.0,
  the smallest normal 2^-6, the subnormals m * 2^-9, NaN = S.1111.111;
* every finite code encodes back to itself;
* round to nearest with ties to the even code, saturation at +-448;
* agreement with torch's own float8_e4m3fn conversion on random values;
* attention over E4M3 pools equals the bf16 attention when the scaled codes
  are exactly bf16 values.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import zfsynth


def test_defining_values():
    d = oracle.e4m3_decode
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert d(0x38) == 1.0 and d(0x30) == 0.5 and d(0xC0) == -2.0
    assert d(0x08) == 2.0 ** -6                        # smallest normal
    assert d(0x01) == 2.0 ** -9 and d(0x07) == 7 * 2.0 ** -9   # subnormals
    assert d(0x00) == 0.0 and math.copysign(1.0, d(0x80)) == -1.0
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))
    # 0x78..0x7E: exponent field 15 is a normal binade except the NaN code
    assert d(0x78) == 256.0 and d(0x7D) == 416.0


def test_every_finite_code_round_trips():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = oracle.e4m3_decode(c)
        assert oracle.e4m3_encode(v) == c


def test_ties_to_even_and_saturation():
    e = oracle.e4m3_encode
    assert e(2.0 ** -10) == 0x00          # half of the smallest subnormal -> 0 (even)
    assert e(3 * 2.0 ** -10) == 0x02      # between 1 and 2 subnormal steps -> 2 (even)
    assert e(1.0625) == 0x38              # between 1.0 (m=0) and 1.125 (m=1) -> 1.0
    assert e(1.1875) == 0x3A              # between 1.125 (m=1) and 1.25 (m=2) -> 1.25
    assert e(0.96875) == 0x38             # across a binade: 0.9375 (0x37) vs 1.0 (0x38)
    assert e(1.05) == 0x38 and e(1.07) == 0x39   # nearest: 1.0 vs 1.125
    assert e(464.0) == 0x7E and e(1e9) == 0x7E and e(-1e9) == 0xFE
    assert e(float("inf")) == 0x7E and e(float("-inf")) == 0xFE
    assert e(float("nan")) == 0x7F


def test_agrees_with_torch_float8_e4m3fn():
    """Random values, every exact midpoint between neighbouring finite codes
    (the ties, of either sign) and NaN, against torch's own conversion."""
    rng = np.random.default_rng(7)
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-3, 2, 20000),
                        rng.uniform(-447, 447, 5000), mids, -mids, [np.nan]]).astype(np.float32)
    assert np.array_equal(x[25000:25000 + mids.size].astype(np.float64), mids)   # ties are exact in fp32
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_quantize_uses_the_single_precision_product():
    rng = np.random.default_rng(8)
    w = zfsynth.to_bf16_bits(rng.standard_normal(4096).astype(np.float32) * 30)
    inv = np.float32(1.0 / 0.37)
    codes = oracle.fp8_quantize(w, inv)
    prod = zfsynth.bf16_bits_to_f32(w) * inv                 # numpy float32 multiply
    assert np.array_equal(codes, np.array([oracle.e4m3_encode(float(p)) for p in prod], dtype=np.uint8))


def test_fp8_attention_equals_bf16_attention_on_exact_values():
    """With a power-of-two scale every scaled code is a bf16 value, so the
    E4M3 attention must equal the bf16 attention on those values exactly."""
    case = zfsynth.make_case("fp8-pin", B=3, Hq=8, Hkv=2, ctx=[40, 17, 64], sigma=0.5, seed=11)
    rng = np.random.default_rng(12)
    shape = case.k_pool.shape
    k_codes = rng.integers(0, 256, size=shape, dtype=np.uint8)
    v_codes = rng.integers(0, 256, size=shape, dtype=np.uint8)
    for c in (k_codes, v_codes):                            # no NaN codes
        c[(c & 0x7F) == 0x7F] = 0x38
    ks, vs = 2.0 ** -3, 2.0 ** 2
    kv = oracle.fp8_dequantize(k_codes, ks).astype(np.float32)
    vv = oracle.fp8_dequantize(v_codes, vs).astype(np.float32)
    k_bf = zfsynth.to_bf16_bits(kv).reshape(shape)
    v_bf = zfsynth.to_bf16_bits(vv).reshape(shape)
    assert np.array_equal(zfsynth.bf16_bits_to_f32(k_bf), kv)  # exact in bf16
    a = oracle.attention(case.q, k_bf, v_bf, case.page_table, case.seq_lens, case.sm_scale)
    b = oracle.attention_fp8(case.q, k_codes, v_codes, ks, vs, case.page_table, case.seq_lens, case.sm_scale)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
