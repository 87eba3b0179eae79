"""Pins for the scaling-aware shift of single E4M3 codes (FP8-Flow-MoE review, section
核心方法: under power-of-two scales the row->column conversion is an exponent shift by
k = log2(Smax) - log2(S_row), with the mantissa re-formed only where the result
becomes subnormal)."""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)


@pytest.mark.parametrize("k", range(0, 41))
def test_value_rule_equals_byte_rule(k):
    """Two independent formulations inside the oracle: decode-scale-encode versus the
    exponent-field subtract with RNE right shift of the significand."""
    assert np.array_equal(oracle.shift_codes(FINITE, k, "value"), oracle.shift_codes(FINITE, k, "bytes"))


@pytest.mark.parametrize("k", range(0, 41))
def test_value_rule_equals_torch_cast(k):
    """Library reference: torch decodes the code, the product by 2^-k is exact in
    float32 for k <= 40, and torch's float8 cast rounds to nearest even."""
    vals = torch.from_numpy(FINITE.copy()).view(torch.float8_e4m3fn).to(torch.float32)
    ref = (vals * (2.0 ** -k)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.shift_codes(FINITE, k), ref)


def test_golden_examples():
    n = 0
    for line in open(os.path.join(GOLDEN, "e4m3_shift_examples.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        c, k, want = line.split()
        got = oracle.shift_codes(np.array([int(c, 16)], np.uint8), int(k))[0]
        assert got == int(want, 16), (c, k, hex(got), want)
        n += 1
    assert n >= 15


@pytest.mark.parametrize("k", range(0, 41))
def test_shift_invariants(k):
    out = oracle.shift_codes(FINITE, k)
    mag_in, mag_out = FINITE & 0x7F, out & 0x7F
    # the sign bit is untouched
    assert np.array_equal(FINITE & 0x80, out & 0x80)
    # never overflows: magnitudes only shrink (codes are ordered like magnitudes)
    assert np.all(mag_out <= mag_in)
    # k = 0 is the identity
    if k == 0:
        assert np.array_equal(out, FINITE)
    # exact whenever the shifted value is representable
    v = oracle.e4m3_decode(FINITE) * 2.0 ** -k
    rep = oracle.e4m3_decode(oracle.e4m3_encode(v)) == v
    assert np.array_equal(oracle.e4m3_decode(out)[rep], v[rep])
    # exponent fields above k stay exact with the mantissa untouched
    E = (FINITE >> 3) & 15
    big = E > k
    assert np.array_equal(out[big] & 7, FINITE[big] & 7)
    assert np.array_equal((out[big] >> 3) & 15, E[big] - k)
