"""Pins for the oracle's single-pass quantizer (row-wise and column-wise layouts from one
read of X), its zero-tile option and the packed UE8M0 scale layout.

Sources: FP8-Flow-MoE review, 核心方法 (scaling-aware transpose of the row-wise result);
DeepSeek FP8 与 DeepGEMM §8 (UE8M0 scales, packed four to an int32 for the SM100 GEMM).
"""
import os

import numpy as np
import pytest

import oracle
from scaling_aware_transpose_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_packed_fixture():
    sf_rows, words = [], {}
    with open(os.path.join(GOLDEN, "packed_ue8m0_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if not line:
                continue
            if line[0] == "sf":
                sf_rows.append([int(v, 16) for v in line[1:]])
            elif line[0] == "word":
                words[(int(line[1]), int(line[2]))] = int(line[3], 16)
    return np.array(sf_rows, np.uint8), words


def test_pack_golden_example():
    sf, words = _read_packed_fixture()
    packed = oracle.pack_ue8m0(sf)
    assert packed.shape == (2, 4)
    for (g, m), w in words.items():
        assert int(packed[g, m]) == w, (g, m)
    assert len(words) == packed.size


@pytest.mark.parametrize("mn,kt", [(8, 4), (12, 56), (128, 16), (5, 7), (3, 1), (256, 64)])
def test_pack_matches_numpy_view(mn, kt):
    """Independent route: pad K to a multiple of 4 and rows to a multiple of 4 with zero
    bytes, reinterpret each row's bytes as little-endian uint32, transpose to MN-major."""
    rng = np.random.default_rng(mn * 100 + kt)
    sf = rng.integers(0, 255, size=(mn, kt), dtype=np.uint8)
    kp, mp = -(-kt // 4) * 4, -(-mn // 4) * 4
    padded = np.zeros((mp, kp), np.uint8)
    padded[:mn, :kt] = sf
    ref = padded.view("<u4").T
    assert np.array_equal(oracle.pack_ue8m0(sf), ref)


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(3)
    sf = rng.integers(0, 255, size=(64, 10), dtype=np.uint8)
    p = oracle.pack_ue8m0(sf)
    unpacked = np.stack([(p >> (8 * i)) & 0xFF for i in range(4)], axis=1)  # [g, 4, mn]
    unpacked = unpacked.reshape(-1, p.shape[1])[: sf.shape[1]].T.astype(np.uint8)
    assert np.array_equal(unpacked, sf)


def _with_zero_tiles(x, frac, seed, neg=False):
    """Zero whole 1x128 tiles of a bf16-bits array (optionally as -0.0)."""
    rng = np.random.default_rng(seed)
    x = x.copy()
    rows, cols = x.shape
    mask = rng.random((rows, cols // 128)) < frac
    z = np.uint16(0x8000 if neg else 0)
    x.reshape(rows, cols // 128, 128)[mask] = z
    return x, mask


def test_zero_tile_option_off_is_rowwise():
    x = synthetic.tiny()["x"]
    q0, sf0 = oracle.quantize_rowwise(x)
    q1, sf1 = oracle.quantize_rowwise_opt(x, zero_tile_min=False)
    assert np.array_equal(q0, q1) and np.array_equal(sf0, sf1)


@pytest.mark.parametrize("neg", [False, True])
def test_zero_tile_option_changes_only_zero_tile_scales(neg):
    x, mask = _with_zero_tiles(synthetic.tiny()["x"], 0.2, seed=1, neg=neg)
    q0, sf0 = oracle.quantize_rowwise(x)
    q1, sf1 = oracle.quantize_rowwise_opt(x, zero_tile_min=True)
    assert mask.any()
    assert np.array_equal(q0, q1)                       # codes of a zero tile are +-0 either way
    assert np.all(sf0[mask] == 127) and np.all(sf1[mask] == 0)
    assert np.array_equal(sf0[~mask], sf1[~mask])
    zero_codes = q1.reshape(q1.shape[0], -1, 128)[mask]
    assert np.all(zero_codes == (0x80 if neg else 0x00))


def test_composite_is_quantize_then_direct():
    x = synthetic.dense(rows=384, cols=640, seed=2)["x"]
    q, sf, qt, sft = oracle.quantize_rowwise_colwise(x, flags=0)
    rq, rsf = oracle.quantize_rowwise(x)
    rqt, rsft = oracle.direct_transpose(rq, rsf)
    for a, b in ((q, rq), (sf, rsf), (qt, rqt), (sft, rsft)):
        assert np.array_equal(a, b)
    q2, sf2, qt2, sft2 = oracle.quantize_rowwise_colwise(x, flags=0, colwise=False)
    assert qt2 is None and sft2 is None and np.array_equal(q2, rq) and np.array_equal(sf2, rsf)


def test_composite_packed_scales():
    x = synthetic.dense(rows=640, cols=384, seed=4)["x"]  # K tiles 3 (row-wise) and 5 (column-wise): ragged packing
    q, sf, qt, sft = oracle.quantize_rowwise_colwise(x, flags=oracle.SF_PACKED_UE8M0)
    rq, rsf, rqt, rsft = oracle.quantize_rowwise_colwise(x, flags=0)
    assert np.array_equal(q, rq) and np.array_equal(qt, rqt)
    assert sf.dtype == np.uint32 and sf.shape == (1, 640)
    assert sft.dtype == np.uint32 and sft.shape == (2, 384)
    for packed, bytes_ in ((sf, rsf), (sft, rsft)):
        mn, kt = bytes_.shape
        padded = np.zeros((mn, -(-kt // 4) * 4), np.uint8)
        padded[:, :kt] = bytes_
        assert np.array_equal(packed, padded.view("<u4").T)


def test_zero_tile_option_hand_worked_block():
    """One 128x128 block: rows 0..126 hold 2^-10 everywhere, row 127 is all zero.
    Row tiles: amax = 2^-10 -> e = -18 (448*2^-19 < 2^-10 <= 448*2^-18), codes
    RNE(2^-10 * 2^18 = 256) = 0x78.  Zero row: e = 0 (pages' rule) or -127 (option).
    Pages' rule: Smax exponent 0, k = 18, 256*2^-18 = 2^-10 is half the smallest
    subnormal 2^-9, ties to even -> 0x00: every value of the block is lost.
    Option: Smax exponent -18, k = 0 for the data rows -> codes unchanged, SF^T byte
    127 - 18 = 109; the zero row shifts by 109 and stays 0x00."""
    one = np.uint16(0x3A80)  # bf16 bits of 2^-10: exponent field 127 - 10 = 117 -> 117 << 7
    x = np.full((128, 128), one, np.uint16)
    x[127] = 0
    q, sf, qt, sft = oracle.quantize_rowwise_colwise(x, flags=0)
    assert np.all(q[:127] == 0x78) and np.all(sf[:127] == 127 - 18) and sf[127, 0] == 127
    assert np.all(qt == 0x00) and np.all(sft == 127)
    q, sf, qt, sft = oracle.quantize_rowwise_colwise(x, flags=oracle.ZERO_TILE_MIN_SCALE)
    assert np.all(sf[:127] == 109) and sf[127, 0] == 0
    assert np.all(qt[:, :127] == 0x78) and np.all(qt[:, 127] == 0x00) and np.all(sft == 109)


def _dec(codes):
    return oracle.e4m3_decode(codes.ravel()).reshape(codes.shape)


def test_zero_tile_option_never_farther():
    """With the option, Smax of a block is the max over its nonzero tiles (<= the max
    with zero tiles counted), so the column-wise grid 2^Smax_opt * E4M3 contains the
    default one within range: each transposed value is at least as close to the
    row-wise value it came from.  Also SF^T = max over nonzero tiles, 0 if none."""
    x = synthetic.stress(rows=512, cols=256, seed=9)["x"]
    # half the row blocks hold only small tiles (all e < 0), where zero tiles matter
    small = synthetic._bf16_bits(np.random.default_rng(7).standard_normal((256, 256)).astype(np.float32) * 2.0**-12)
    x[256:] = small
    x, mask = _with_zero_tiles(x, 0.05, seed=2)
    x[:128, :128] = 0  # one entirely zero block
    q, sf = oracle.quantize_rowwise_opt(x, zero_tile_min=True)
    _, _, qt0, sft0 = oracle.quantize_rowwise_colwise(x, flags=0)
    _, _, qt1, sft1 = oracle.quantize_rowwise_colwise(x, flags=oracle.ZERO_TILE_MIN_SCALE)
    rows, cols = x.shape
    zero = np.abs(_dec(q)).reshape(rows, cols // 128, 128).max(axis=2) == 0
    e = sf.astype(np.int64)
    e_nz = np.where(zero, -1, e).reshape(rows // 128, 128, cols // 128).max(axis=1)  # [nb, nt]
    want = np.where(e_nz < 0, 0, e_nz)
    assert np.array_equal(sft1, np.repeat(want.T, 128, axis=0))
    v = (_dec(q) * np.exp2(e.repeat(128, axis=1) - 127)).T          # row-wise values, [cols, rows]
    v0 = _dec(qt0) * np.exp2(sft0.astype(np.int64).repeat(128, axis=1) - 127)
    v1 = _dec(qt1) * np.exp2(sft1.astype(np.int64).repeat(128, axis=1) - 127)
    assert np.all(np.abs(v1 - v) <= np.abs(v0 - v))
    assert np.abs(v1 - v).sum() < np.abs(v0 - v).sum()            # and strictly better somewhere
