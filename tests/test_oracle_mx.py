"""Pins for the oracle's tile-size-generic quantize and direct transpose, used at the
MX granularity (1x32 tiles, 32x32 blocks): the low-precision format table (MXFP8 = E4M3
elements with one power-of-two scale per 32 elements) and the FP8-Flow-MoE review's
future work (the scaling-aware layout conversion carried to MX formats)."""
import numpy as np
import pytest
import torch

import oracle
from scaling_aware_transpose_b200 import synthetic


def fp8_decode_t(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)


def library_quantize(x_bits, G):
    """torch: amax per 1xG tile, S = 2^ceil(log2(amax/448)) (S = 1 for zero tiles), cast."""
    x = torch.from_numpy(synthetic.bf16_bits_to_f32(x_bits)).to(torch.float64)
    rows, cols = x.shape
    t = x.reshape(rows, cols // G, G)
    amax = t.abs().amax(dim=2)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax)).clamp(-127, 127)
    q = (t * torch.exp2(-e)[:, :, None]).to(torch.float32).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).reshape(rows, cols).numpy(), (e + 127).to(torch.uint8).numpy()


def library_direct(q, sf, G):
    rows, cols = q.shape
    nb, nt = rows // G, cols // G
    e = torch.from_numpy(sf.astype(np.int64) - 127)
    emax = e.reshape(nb, G, nt).amax(dim=1)
    k = emax.repeat_interleave(G, dim=0) - e
    v = fp8_decode_t(q) * torch.exp2(-k.to(torch.float64)).repeat_interleave(G, dim=1)
    qt = v.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy().T.copy()
    sft = np.repeat((emax + 127).numpy().astype(np.uint8).T, G, axis=0)
    return qt, sft


@pytest.mark.parametrize("maker", [lambda: synthetic.tiny()["x"], lambda: synthetic.stress(rows=256, cols=384, seed=2)["x"],
                                   lambda: synthetic.dense(rows=384, cols=256, seed=1)["x"]])
def test_tile_128_is_the_pinned_path(maker):
    x = maker()
    q, sf = oracle.quantize_rowwise_g(x, 128)
    rq, rsf = oracle.quantize_rowwise(x)
    assert np.array_equal(q, rq) and np.array_equal(sf, rsf)
    qt, sft = oracle.direct_transpose_g(q, sf, 128)
    rqt, rsft = oracle.direct_transpose(rq, rsf)
    assert np.array_equal(qt, rqt) and np.array_equal(sft, rsft)


@pytest.mark.parametrize("seed,rows,cols", [(0, 64, 96), (3, 256, 512), (7, 96, 160)])
def test_mx32_matches_library_recipe(seed, rows, cols):
    x = synthetic.stress(rows=rows, cols=cols if cols % 128 == 0 else 128 * (cols // 128 + 1), seed=seed)["x"][:, :cols]
    x = np.ascontiguousarray(x)
    q, sf = oracle.quantize_rowwise_g(x, 32)
    lq, lsf = library_quantize(x, 32)
    assert np.array_equal(sf, lsf) and np.array_equal(q, lq)
    qt, sft = oracle.direct_transpose_g(q, sf, 32)
    lqt, lsft = library_direct(q, sf, 32)
    assert np.array_equal(sft, lsft) and np.array_equal(qt, lqt)


def test_mx32_equal_subtile_exponents_reduce_to_128():
    """When the four 1x32 sub-tiles of every 1x128 tile have the same exponent (here every
    sub-tile holds one element of magnitude 400 * 2^r), the codes agree with the 1x128
    quantization and the scales are the 1x128 scales repeated four times."""
    rng = np.random.default_rng(4)
    f = rng.uniform(-1, 1, size=(64, 256)).astype(np.float32) * 300
    f[:, ::32] = 400.0
    f *= np.exp2(rng.integers(-6, 6, size=(64, 1))).astype(np.float32)
    x = synthetic._bf16_bits(f)
    q32, sf32 = oracle.quantize_rowwise_g(x, 32)
    q128, sf128 = oracle.quantize_rowwise(x)
    assert np.array_equal(q32, q128) and np.array_equal(sf32, np.repeat(sf128, 4, axis=1))


def test_mx32_exhaustive_codes_and_shifts():
    """Rows t = 0..31 of a 32x32 block row hold every finite code (8 column blocks) at
    scale exponent 31 - t, so row t shifts by k = t."""
    codes = np.arange(256, dtype=np.uint8)
    codes[0x7F], codes[0xFF] = 0x00, 0x80
    q = np.tile(codes, (32, 1))
    sf = np.repeat((127 + 31 - np.arange(32)).astype(np.uint8)[:, None], 8, axis=1)
    qt, sft = oracle.direct_transpose_g(q, sf, 32)
    assert np.all(sft == 127 + 31)
    for k in range(32):
        assert np.array_equal(qt[:, k], oracle.shift_codes(codes, k))


def test_mx32_uniform_scales_are_a_byte_transpose():
    rng = np.random.default_rng(1)
    q = rng.integers(0, 0x7E, size=(96, 64), dtype=np.uint8)
    sf = np.full((96, 2), 120, np.uint8)
    qt, sft = oracle.direct_transpose_g(q, sf, 32)
    assert np.array_equal(qt, q.T) and np.all(sft == 120)


def test_mx32_shape_rules():
    with pytest.raises(oracle.OracleError):
        oracle.quantize_rowwise_g(np.zeros((4, 48), np.uint16), 32)
    with pytest.raises(oracle.OracleError):
        oracle.direct_transpose_g(np.zeros((48, 64), np.uint8), np.zeros((48, 2), np.uint8), 32)
