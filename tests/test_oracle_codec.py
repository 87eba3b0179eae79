"""Pins for the oracle's E4M3 codec and power-of-two scale rule.

The references here are independent of the oracle's C code: PyTorch's own
``float8_e4m3fn`` conversions (a library routine), a brute-force nearest-code search,
exact closed forms, and hand-worked fixtures under tests/golden/.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def torch_decode_all():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def torch_encode_f32(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def all_bf16_f32():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    return v[np.isfinite(v)]


def test_decode_matches_torch_on_all_codes():
    ref = torch_decode_all()
    got = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ref[~nan], got[~nan])
    assert np.signbit(got[0x80]) and got[0x80] == 0.0
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_round_trip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


@pytest.mark.parametrize("shift", list(range(-40, 21, 4)) + [-1, 1, 2, 3])
def test_encode_matches_torch_on_all_bf16_scaled(shift):
    """Every finite BF16 value times 2^shift, below torch's NaN threshold (464)."""
    v = all_bf16_f32().astype(np.float64) * 2.0 ** shift
    v = v[(np.abs(v) < 464.0) & (np.abs(v) > 2.0 ** -140)]
    v = np.concatenate([v, [0.0, -0.0]])
    ref = torch_encode_f32(v.astype(np.float32))
    got = oracle.e4m3_encode(v)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, [(v[i], hex(ref[i]), hex(got[i])) for i in bad[:5]]


def brute_force_nearest(v: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 code by exhaustive search, ties to the even code (LSB 0),
    saturating magnitudes above 448; the sign bit follows the input's sign."""
    table = torch_decode_all()[:0x7F]  # magnitudes of codes 0x00..0x7E
    a = np.abs(v)
    d = np.abs(a[:, None] - table[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among equal distances prefer the code whose lowest bit is 0
    even = cand & ((np.arange(0x7F)[None, :] & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    pick = np.where(a >= 448.0, 0x7E, pick)
    return (pick | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def test_encode_matches_brute_force_nearest():
    rng = np.random.default_rng(1)
    table = torch_decode_all()[:0x7F]
    mids = (table[1:] + table[:-1]) / 2.0
    eps = np.array([0.0, 1e-9, -1e-9])
    probes = [
        rng.uniform(0, 500, 20000),
        np.exp2(rng.uniform(-14, 9, 20000)),
        (mids[:, None] + mids[:, None] * eps[None, :]).ravel(),
        table,
        np.array([448.0, 460.0, 463.9, 464.0, 470.0, 1e9, 2.0 ** -10, 2.0 ** -11, 0.0]),
    ]
    v = np.concatenate(probes)
    v = np.concatenate([v, -v])
    assert np.array_equal(oracle.e4m3_encode(v), brute_force_nearest(v))


def test_saturation():
    v = np.array([448.0, 449.0, 464.0, 480.0, 1e30, -1e30, -448.5])
    assert oracle.e4m3_encode(v).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_signed_zero():
    v = np.array([0.0, -0.0, 2.0 ** -11, -(2.0 ** -11), -(2.0 ** -10)])
    assert oracle.e4m3_encode(v).tolist() == [0x00, 0x80, 0x00, 0x80, 0x80]


# ------------------------------------------------------------------ scale rule

def load_pairs(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if line:
            rows.append(line.split())
    return rows


def test_scale_exponent_golden():
    rows = load_pairs("scale_exponent_examples.txt")
    amax = np.array([float(r[0]) for r in rows])
    want = [int(r[1]) for r in rows]
    assert oracle.scale_exponent(amax).tolist() == want


def test_scale_exponent_definition_property():
    rng = np.random.default_rng(2)
    v = all_bf16_f32().astype(np.float64)
    v = np.abs(v[v != 0])
    v = np.concatenate([v, np.exp2(rng.uniform(-120, 120, 50000)), rng.uniform(0, 1e4, 50000)])
    e = oracle.scale_exponent(v)
    for a, ee in zip(v.tolist(), e.tolist()):
        if -127 < ee < 127:
            assert a <= math.ldexp(448.0, ee) and a > math.ldexp(448.0, ee - 1), (a, ee)
        elif ee == -127:
            assert a <= math.ldexp(448.0, -127)


def test_scale_exponent_matches_stated_formula_on_bf16():
    """For BF16 amax the stated closed form S = 2^ceil(log2(amax/448)), evaluated with
    the library log2 in double, is exact (amax/448 at a power of two is exact and any
    BF16 amax above it is at least 2^-8 relatively larger)."""
    v = all_bf16_f32().astype(np.float64)
    v = np.abs(v[(v > 0) & (v < 3e38)])
    formula = np.ceil(np.log2(v / 448.0)).astype(np.int64)
    formula = np.clip(formula, -127, 127)
    assert np.array_equal(oracle.scale_exponent(v), formula)


def test_scale_exponent_zero_and_clamp():
    assert oracle.scale_exponent(np.array([0.0, 1e-45, 2.0 ** -133, 3.3e38])).tolist() == [0, -127, -127, 120]
