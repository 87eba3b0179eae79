"""GPU parity of the MX-granularity path (1x32 scaling tiles, 32x32 transpose blocks)
against the CPU oracle, byte for byte: ragged shapes, the dense and range-stress
workloads at full size, an exhaustive code x shift sweep and edge values."""
import numpy as np
import pytest

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, dev, device_status_ok, host

pytestmark = pytest.mark.gpu


def check(x_bits, transpose=True, what=""):
    q, sf = sat.quantize_rowwise_mx32(dev(x_bits))
    oq, osf = oracle.quantize_rowwise_g(x_bits, 32)
    assert_bytes_equal(host(sf), osf, f"SF {what}")
    assert_bytes_equal(host(q), oq, f"Q {what}")
    if transpose:
        qt, sft = sat.direct_transpose_mx32(q, sf)
        oqt, osft = oracle.direct_transpose_g(oq, osf, 32)
        assert_bytes_equal(host(sft), osft, f"SF^T {what}")
        assert_bytes_equal(host(qt), oqt, f"Q^T {what}")
    device_status_ok()


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (384, 1152), (1024, 2048), (2048, 7168)])
def test_shapes(rows, cols):
    check(synthetic.stress(rows=rows, cols=cols, seed=rows + cols)["x"], what=f"{rows}x{cols}")


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 96), (130, 160), (7, 7168 + 32)])
def test_quantize_ragged(rows, cols):
    """The quantizer alone needs only cols % 32 == 0: odd rows, tile counts that are not a
    multiple of a warp's 16 tiles."""
    x = synthetic.scaled_normal(rows, 128 * (cols // 128 + 1), seed=rows, row_sigma=3.0)[:, :cols]
    check(np.ascontiguousarray(x), transpose=False, what=f"{rows}x{cols}")


def test_tiny_config():
    check(synthetic.tiny()["x"], what="tiny")


def test_dense_config_full():
    check(synthetic.dense()["x"], what="dense")


def test_stress_config_full():
    check(synthetic.stress()["x"], what="stress")


def test_exhaustive_codes_and_shifts():
    codes = np.arange(256, dtype=np.uint8)
    codes[0x7F], codes[0xFF] = 0x00, 0x80
    q = np.tile(codes, (128, 1))
    e = np.full(128, 31, np.int64)
    e[:32] = 31 - np.arange(32)
    sf = np.repeat((e + 127).astype(np.uint8)[:, None], 8, axis=1)
    qt, sft = sat.direct_transpose_mx32(dev(q), dev(sf))
    oqt, osft = oracle.direct_transpose_g(q, sf, 32)
    assert_bytes_equal(host(sft), osft, "SF^T")
    assert_bytes_equal(host(qt), oqt, "Q^T")
    for k in range(32):
        assert np.array_equal(oqt[:, k], oracle.shift_codes(codes, k))


def test_edge_values():
    f = np.zeros((128, 256), np.float32)
    f[1, :] = -0.0
    f[2, 0], f[2, 33], f[2, 70] = 3.3e38, -1.0, 1e30
    f[3, :] = 2.0 ** -133
    f[4, :128] = np.linspace(-448, 448, 128)
    f[5, 128:] = 2.0 ** -10
    f[5, 128::32] = 448.0
    check(synthetic._bf16_bits(f), what="edges")
