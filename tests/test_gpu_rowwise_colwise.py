"""GPU parity of the single-pass quantizer (row-wise and column-wise layouts from one read
of X) against the CPU oracle, byte for byte: every option combination, ragged packed
scale layouts, row-wise-only mode with odd row counts, an exhaustive code x shift sweep,
edge values and the full dense and range-stress workloads."""
import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, dev, device_status_ok, host

pytestmark = pytest.mark.gpu

FLAGS = [0, sat.ZERO_TILE_MIN_SCALE, sat.SF_PACKED_UE8M0, sat.ZERO_TILE_MIN_SCALE | sat.SF_PACKED_UE8M0]


def _u32(t):
    return host(t).view(np.uint32) if t.dtype == torch.int32 else host(t)


def check(x_bits, flags=0, colwise=True, what=""):
    q, sf, qt, sft = sat.quantize_rowwise_colwise(dev(x_bits), flags=flags, colwise=colwise)
    device_status_ok()
    oq, osf, oqt, osft = oracle.quantize_rowwise_colwise(x_bits, flags=flags, colwise=colwise)
    assert_bytes_equal(_u32(sf), osf, f"SF {what} flags={flags}")
    assert_bytes_equal(host(q), oq, f"Q {what} flags={flags}")
    if colwise:
        assert_bytes_equal(_u32(sft), osft, f"SF^T {what} flags={flags}")
        assert_bytes_equal(host(qt), oqt, f"Q^T {what} flags={flags}")
    else:
        assert qt is None and sft is None


def with_zero_tiles(x, frac, seed):
    rng = np.random.default_rng(seed)
    x = x.copy()
    rows, cols = x.shape
    t = x.reshape(rows, cols // 128, 128)
    m = rng.random((rows, cols // 128))
    t[m < frac / 2] = 0
    t[(m >= frac / 2) & (m < frac)] = 0x8000  # -0.0
    return x


@pytest.mark.parametrize("flags", FLAGS)
def test_tiny_config(flags):
    check(synthetic.tiny()["x"], flags, what="tiny")


# several blocks, K tile counts not a multiple of 4 in either layout (ragged packed
# words), a single block, wide and tall shapes
SHAPES = [(128, 128), (128, 384), (256, 640), (384, 1152), (640, 256), (1152, 896), (2048, 7168)]


@pytest.mark.parametrize("rows,cols", SHAPES)
@pytest.mark.parametrize("flags", FLAGS)
def test_random_shapes(rows, cols, flags):
    x = synthetic.scaled_normal(rows, cols, seed=rows * 3 + cols, row_sigma=2.5)
    check(with_zero_tiles(x, 0.1, seed=rows), flags, what=f"{rows}x{cols}")


@pytest.mark.parametrize("flags", FLAGS)
def test_small_blocks_with_zero_rows(flags):
    """Blocks of small values (all e < 0) with zero tiles: the case the zero-tile option
    changes, plus a block that is entirely zero."""
    rng = np.random.default_rng(5)
    f = rng.standard_normal((512, 512)).astype(np.float32) * np.float32(2.0 ** -14)
    f[::7] = 0.0
    f[128:256, 128:256] = 0.0
    f[300, 256:384] = -0.0
    check(synthetic._bf16_bits(f), flags, what="small blocks")


@pytest.mark.parametrize("flags", [0, sat.SF_PACKED_UE8M0, sat.ZERO_TILE_MIN_SCALE | sat.SF_PACKED_UE8M0])
def test_rowwise_only_odd_rows(flags):
    """Without Q^T there is no 128-row rule: 1, 3, 130 and 257 rows (padding rows of the
    packed layout must come out as zero words)."""
    for rows in (1, 3, 130, 257):
        x = with_zero_tiles(synthetic.scaled_normal(rows, 640, seed=rows), 0.1, seed=rows)
        check(x, flags, colwise=False, what=f"rows={rows}")


def test_exhaustive_codes_and_shifts():
    """Row t (t <= 40) of the block has scale exponent 40 - t, so its codes shift by
    k = t; each row holds every finite code (0x7F/0xFF replaced by zeros), and each row
    tile holds +-448 so that its exponent is exactly the chosen one."""
    codes = np.arange(256, dtype=np.uint8)
    codes[0x7F], codes[0xFF] = 0x00, 0x80
    vals = oracle.e4m3_decode(codes)
    e = np.full(128, 40, np.int64)
    e[:41] = 40 - np.arange(41)
    f = (vals[None, :] * np.exp2(e.astype(np.float64))[:, None]).astype(np.float32)
    x = synthetic._bf16_bits(f)
    assert np.array_equal(synthetic.bf16_bits_to_f32(x), f)  # exact in bf16
    for flags in FLAGS:
        check(x, flags, what="sweep")
    _, sf, qt, _ = oracle.quantize_rowwise_colwise(x)
    assert np.array_equal(sf[:, 0].astype(np.int64) - 127, e)
    for k in range(41):
        assert np.array_equal(qt[:128, k], oracle.shift_codes(codes[:128], k))


def test_edge_values():
    f = np.zeros((128, 256), np.float32)
    f[1, :] = -0.0
    f[2, 0], f[2, 1], f[2, 2] = 3.3e38, -1.0, 1e30
    f[3, :] = 2.0 ** -133
    f[3, 5] = -(2.0 ** -130)
    f[4, :128] = np.linspace(-448, 448, 128)
    f[5, 128:] = 2.0 ** -10
    f[5, 128] = 448.0
    x = synthetic._bf16_bits(f)
    for flags in FLAGS:
        check(x, flags, what="edges")


def test_equals_quantize_then_direct_on_gpu():
    """Same bytes as the two separate library calls on the dense workload's shape."""
    x = dev(synthetic.dense(rows=1024)["x"])
    q, sf, qt, sft = sat.quantize_rowwise_colwise(x)
    rq, rsf = sat.quantize_rowwise(x)
    rqt, rsft = sat.direct_transpose(rq, rsf)
    for a, b in ((q, rq), (sf, rsf), (qt, rqt), (sft, rsft)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("flags", [0, sat.ZERO_TILE_MIN_SCALE | sat.SF_PACKED_UE8M0])
def test_dense_config_full(flags):
    check(synthetic.dense()["x"], flags, what="dense 8192x7168")


def test_stress_config_full():
    check(synthetic.stress()["x"], sat.ZERO_TILE_MIN_SCALE, what="stress 65536x7168")


def test_empty_is_noop():
    z = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q, sf, qt, sft = sat.quantize_rowwise_colwise(z)
    assert q.shape == (0, 256) and qt.shape == (256, 0)
    device_status_ok()
