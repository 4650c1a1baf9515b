"""Pins for the oracle's OFP8 E4M3 decode / encode / absmax scaling.

Checked against: the format's printed special values (tests/golden, cited there),
PyTorch's float8_e4m3fn conversions for in-range values (a library routine that
shares nothing with this repo), exact midpoints between neighbouring codes
(ties go to the even mantissa), round trips and the format's error bound.
"Qwen/Qwen-Image-2.1" (vLLM recipe), "Prefix KV cache": the cache may be stored
in FP8 ("fp8_v": V only; "fp8": K and V)."""
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_special_values.txt")


def _all_bf16_finite():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    return vals[np.isfinite(vals)]


def test_golden_special_values():
    with open(GOLDEN) as f:
        lines = f.readlines()
    for line in lines:
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        got = oracle.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_decode_table_matches_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if math.isnan(ref[c].item()):
            assert math.isnan(got)
        else:
            assert got == ref[c].item(), c


def test_round_trip_every_finite_code():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c


def test_ties_go_to_even():
    for c in range(0x7E):
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        mid = (lo + hi) / 2.0
        assert float(np.float32(mid)) == mid
        want = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == want
        assert oracle.e4m3_encode(-mid) == want | 0x80


def test_saturation_and_signed_zero():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(464.0) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-9) == 0x80
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00  # exact tie between 0 and 2^-9 -> even
    assert oracle.e4m3_encode(1.5 * 2.0 ** -10) == 0x01


def test_encode_matches_torch_for_every_in_range_bf16():
    """All finite bf16 values with |x| <= 448 (no saturation involved) against
    torch's float32 -> float8_e4m3fn cast."""
    x = _all_bf16_finite()
    x = x[np.abs(x) <= 448.0]
    got = oracle.e4m3_encode_array(x)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)


def test_encode_matches_torch_on_scaled_values():
    """The quantiser's real inputs are x / s; check fp32 quotients of bf16 values by
    a spread of scales (in-range results only)."""
    x = _all_bf16_finite()
    x = x[np.abs(x) < 60.0]
    rng = np.random.default_rng(3)
    for amax in rng.uniform(0.5, 60.0, size=8).astype(np.float32):
        s = np.float32(amax) / np.float32(448.0)
        q = (x.astype(np.float64) / np.float64(s)).astype(np.float32)
        q = q[np.abs(q) <= 448.0]
        got = oracle.e4m3_encode_array(q)
        want = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got, want)


def test_relative_error_bound_in_normal_range():
    rng = np.random.default_rng(5)
    x = (rng.uniform(-1, 1, 20000) * np.exp2(rng.uniform(-6, 8.8, 20000))).astype(np.float32)
    x = x[(np.abs(x) >= 2.0 ** -6) & (np.abs(x) <= 448.0)]
    codes = oracle.e4m3_encode_array(x)
    dec = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    assert np.all(np.abs(dec - x) <= 2.0 ** -4 * np.abs(x))


def test_encode_is_monotone():
    x = np.sort(np.random.default_rng(6).uniform(-500, 500, 5000).astype(np.float32))
    dec = np.array([oracle.e4m3_decode(int(c)) for c in oracle.e4m3_encode_array(x)])
    assert np.all(np.diff(dec) >= 0)


def test_absmax_scale_definition():
    rng = np.random.default_rng(9)
    H, P, d = 3, 37, 16
    x = torch.from_numpy(rng.normal(0, 2.5, (P, H, d)).astype(np.float32)).to(torch.bfloat16)
    codes, scales = oracle.quantize_prefix(x, P)
    xf = x.to(torch.float32).numpy()
    for h in range(H):
        amax = np.float32(np.abs(xf[:, h]).max())
        assert scales[h] == np.float32(amax / np.float32(448.0))
        # the largest magnitude lands on the largest code
        t, c = np.unravel_index(np.abs(xf[:, h]).argmax(), (P, d))
        assert codes[h, t, c] & 0x7F == 0x7E
        # every code is the RNE encoding of fp32(x / s)
        q = (xf[:, h].astype(np.float64) / np.float64(scales[h])).astype(np.float32)
        assert np.array_equal(codes[h], oracle.e4m3_encode_array(q))
    zeros = torch.zeros((5, 2, 4), dtype=torch.bfloat16)
    c0, s0 = oracle.quantize_prefix(zeros, 5)
    assert np.all(s0 == 1.0) and np.all(c0 == 0)


def test_quantize_leaves_rows_beyond_prefix():
    x = torch.ones((10, 2, 4), dtype=torch.bfloat16)
    codes, _ = oracle.quantize_prefix(x, 6, cap=9)
    assert codes.shape == (2, 9, 4)
    assert np.all(codes[:, :6] == 0x7E) and np.all(codes[:, 6:] == 0)
