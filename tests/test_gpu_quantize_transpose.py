"""GPU parity: row-wise quantization, direct transpose and the naive baseline against the
CPU oracle, byte for byte, on seeded inputs (tiny shapes, ragged tile counts, the
full dense and range-stress workloads, exhaustive code x shift sweeps, edge cases)."""
import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, dev, device_status_ok, host

pytestmark = pytest.mark.gpu


def run_quant_direct(x_bits, naive=False):
    x = dev(x_bits)
    q, sf = sat.quantize_rowwise(x)
    qt, sft = sat.direct_transpose(q, sf)
    out = {"q": host(q), "sf": host(sf), "qt": host(qt), "sft": host(sft)}
    if naive:
        nq, nsf = sat.naive_transpose(q, sf)
        out.update(nqt=host(nq), nsft=host(nsf))
    device_status_ok()
    return out


def check_against_oracle(x_bits, naive=False):
    g = run_quant_direct(x_bits, naive)
    q, sf = oracle.quantize_rowwise(x_bits)
    assert_bytes_equal(g["sf"], sf, "SF")
    assert_bytes_equal(g["q"], q, "Q")
    qt, sft = oracle.direct_transpose(q, sf)
    assert_bytes_equal(g["sft"], sft, "SF^T")
    assert_bytes_equal(g["qt"], qt, "Q^T")
    if naive:
        nqt, nsft = oracle.naive_transpose(q, sf)
        assert_bytes_equal(g["nsft"], nsft, "naive SF^T")
        assert_bytes_equal(g["nqt"], nqt, "naive Q^T")


def test_tiny_config():
    check_against_oracle(synthetic.tiny()["x"], naive=True)


# rows x cols: several tiles, block counts that leave a partial last wave of CTAs, a
# single tile, odd column-block counts
SHAPES = [(128, 128), (128, 384), (256, 640), (384, 1152), (640, 256), (1024, 1024), (1152, 896), (2048, 7168)]


@pytest.mark.parametrize("rows,cols", SHAPES)
def test_random_shapes(rows, cols):
    check_against_oracle(synthetic.scaled_normal(rows, cols, seed=rows + cols, row_sigma=2.5), naive=True)


def test_quantize_odd_rows():
    """Row-wise quantization has no 128-row rule: 1, 3 and 130 rows."""
    for rows in (1, 3, 130):
        x = synthetic.scaled_normal(rows, 384, seed=rows)
        q, sf = sat.quantize_rowwise(dev(x))
        oq, osf = oracle.quantize_rowwise(x)
        assert_bytes_equal(host(sf), osf, "SF")
        assert_bytes_equal(host(q), oq, "Q")


def test_dense_config_full():
    check_against_oracle(synthetic.dense()["x"], naive=True)


def test_stress_config_full():
    """65536 x 7168: large enough that the dense transpose takes its 256x128-tile kernel."""
    check_against_oracle(synthetic.stress()["x"])


def test_large_tile_path_wide_rows():
    """A second shape on the 256x128-tile kernel (at least eight waves of tiles): 6912 x
    28672, 224 column blocks, range-stress tiles; and 6784 rows (not a multiple of 256),
    which stays on the 128x128 kernel."""
    for rows in (6912, 6784):
        check_against_oracle(synthetic.stress(rows=rows, cols=28672, seed=rows)["x"])


def test_all_bf16_values_at_fixed_scales():
    """Every finite BF16 magnitude up to 448 * 2^E, both signs, in tiles whose first
    element pins the tile exponent to E (so every value goes through the encoder)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = synthetic.bf16_bits_to_f32(bits)
    for E in (0, -20, 7):
        lim = 448.0 * 2.0 ** E
        v = bits[np.isfinite(vals) & (np.abs(vals) <= lim)]
        n = -(-v.size // 127)
        pad = np.zeros(n * 127, np.uint16)
        pad[: v.size] = v
        head = synthetic._bf16_bits(np.full(n, lim, np.float32))
        x = np.concatenate([head[:, None], pad.reshape(n, 127)], axis=1)
        x = np.ascontiguousarray(x)  # n tiles = n rows of 128
        q, sf = sat.quantize_rowwise(dev(x))
        oq, osf = oracle.quantize_rowwise(x)
        assert np.all(osf == 127 + E)
        assert_bytes_equal(host(sf), osf, f"SF E={E}")
        assert_bytes_equal(host(q), oq, f"Q E={E}")


def test_quantize_edge_values():
    f = np.zeros((6, 256), np.float32)
    f[1, :] = -0.0                                      # all negative zero -> sf 127, codes 0x80
    f[2, 0], f[2, 1], f[2, 2] = 3.3e38, -1.0, 1e30      # near BF16 max: e = 120
    f[3, :] = 2.0 ** -133                               # BF16 subnormal floor: e clamped to -127
    f[3, 5] = -(2.0 ** -130)
    f[4, :128] = np.linspace(-448, 448, 128)            # exact-ish grid incl. ties
    f[5, 128:] = 2.0 ** -10                             # tie at half the smallest subnormal
    f[5, 128] = 448.0
    x = synthetic._bf16_bits(f)
    q, sf = sat.quantize_rowwise(dev(x))
    oq, osf = oracle.quantize_rowwise(x)
    assert_bytes_equal(host(sf), osf, "SF")
    assert_bytes_equal(host(q), oq, "Q")
    assert osf[0, 0] == 127 and osf[2, 0] == 127 + 120 and osf[3, 0] == 0


def shift_sweep_inputs():
    """Two 128x128 blocks' worth of codes: row t of block 0 shifts by k = t (t <= 40),
    every finite code appears in every row (0x7F/0xFF replaced by zeros)."""
    rows, cols = 128, 256
    codes = np.arange(256, dtype=np.uint8)
    codes[0x7F], codes[0xFF] = 0x00, 0x80
    q = np.tile(codes, (rows, 1))
    e = np.full(rows, 40, np.int64)
    e[:41] = 40 - np.arange(41)
    sf = np.repeat((e + 127).astype(np.uint8)[:, None], cols // 128, axis=1)
    return q, sf


def test_direct_exhaustive_codes_and_shifts():
    q, sf = shift_sweep_inputs()
    qt, sft = sat.direct_transpose(dev(q), dev(sf))
    device_status_ok()
    oqt, osft = oracle.direct_transpose(q, sf)
    assert_bytes_equal(host(sft), osft, "SF^T")
    assert_bytes_equal(host(qt), oqt, "Q^T")
    # and the oracle's answer here is the value rule applied code by code
    for k in range(41):
        assert np.array_equal(oqt[:, k], oracle.shift_codes(q[k], k))


def test_direct_all_zero_and_uniform_scales():
    q = np.zeros((256, 256), np.uint8)
    q[:, 7] = 0x80
    sf = np.full((256, 2), 127, np.uint8)
    qt, sft = sat.direct_transpose(dev(q), dev(sf))
    assert_bytes_equal(host(qt), q.T.copy(), "Q^T of k = 0 blocks is the byte transpose")
    assert np.all(host(sft) == 127)


# ------------------------------------------------------------------ groups

def grouped_case(sizes, cols, seed, capacity_extra=0):
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows = int(off[-1]) + capacity_extra
    x = synthetic.scaled_normal(rows, cols, seed=seed, row_sigma=2.0)
    q, sf = oracle.quantize_rowwise(x)
    return q, sf, off


@pytest.mark.parametrize("fn", ["direct", "naive"])
def test_grouped_matches_oracle(fn):
    q, sf, off = grouped_case([128, 0, 384, 256, 0, 128], 384, seed=21, capacity_extra=256)
    rows, cols = q.shape
    call = sat.direct_transpose if fn == "direct" else sat.naive_transpose
    qt, sft = call(dev(q), dev(sf), dev(off))
    device_status_ok()
    oqt, osft = (oracle.direct_transpose if fn == "direct" else oracle.naive_transpose)(q, sf, off)
    n = int(off[-1])
    assert_bytes_equal(host(qt)[: cols * n], oqt[: cols * n], "grouped Q^T")
    assert_bytes_equal(host(sft)[: cols * n // 128], osft[: cols * n // 128], "grouped SF^T")


def test_grouped_single_group_equals_dense():
    x = synthetic.scaled_normal(512, 256, seed=22)
    q, sf = sat.quantize_rowwise(dev(x))
    qt, sft = sat.direct_transpose(q, sf)
    off = torch.tensor([0, 512], dtype=torch.int32, device="cuda")
    gqt, gsft = sat.direct_transpose(q, sf, off)
    assert torch.equal(gqt.view(256, 512), qt) and torch.equal(gsft.view(256, 4), sft)


@pytest.mark.parametrize("bad", [[0, 100, 256], [0, 256, 128, 256], [128, 256], [0, 1024]])
def test_bad_group_offsets_set_device_status(bad):
    q = torch.zeros((512, 256), dtype=torch.uint8, device="cuda")
    sf = torch.full((512, 2), 127, dtype=torch.uint8, device="cuda")
    off = torch.tensor(bad, dtype=torch.int32, device="cuda")
    sat.direct_transpose(q, sf, off)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_SHAPE
    sat.naive_transpose(q, sf, off)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_SHAPE
    assert sat.fp8q_last_device_status() == 0  # read-and-clear


def test_empty_inputs_are_noops():
    z = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q, sf = sat.quantize_rowwise(z)
    assert q.shape == (0, 256)
    qt, sft = sat.direct_transpose(q, sf)
    assert qt.shape == (256, 0)
    device_status_ok()


# ------------------------------------------------------------------ 50 random small shapes

def _random_shapes(n=50, seed=123):
    rng = np.random.default_rng(seed)
    return [(128 * int(rng.integers(1, 9)), 128 * int(rng.integers(1, 9)), int(rng.integers(0, 1 << 30)))
            for _ in range(n)]


@pytest.mark.parametrize("rows,cols,seed", _random_shapes())
def test_fifty_random_small_shapes(rows, cols, seed):
    """T, H in {128..1024} (multiples of 128), seeded; every step of the path (quantize,
    direct, naive, single pass) against the oracle.  Inputs alternate between the dense
    and the range-stress recipes."""
    if seed % 2:
        x = synthetic.stress(rows=rows, cols=cols, seed=seed % 1000)["x"]
    else:
        x = synthetic.scaled_normal(rows, cols, seed=seed % 1000, row_sigma=2.0)
    check_against_oracle(x, naive=True)
    q, sf, qt, sft = sat.quantize_rowwise_colwise(dev(x))
    oq, osf, oqt, osft = oracle.quantize_rowwise_colwise(x)
    assert_bytes_equal(host(q), oq, "single-pass Q")
    assert_bytes_equal(host(sf), osf, "single-pass SF")
    assert_bytes_equal(host(qt), oqt, "single-pass Q^T")
    assert_bytes_equal(host(sft), osft, "single-pass SF^T")
