"""Pins for the oracle's row-wise 1x128 quantization (DeepSeek FP8 与 DeepGEMM §3:
per token per 128 channels, online amax; FP8-Flow-MoE review 关键观察: power-of-two
scales)."""
import os

import numpy as np
import torch

import oracle
from scaling_aware_transpose_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def library_quantize(x_bits: np.ndarray):
    """The stated recipe with library primitives: torch amax per 1x128 tile,
    S = 2^ceil(log2(amax/448)) in float64 (S = 1 for zero tiles), x/S exact in float32,
    torch's float8_e4m3fn cast (round to nearest even)."""
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    rows, cols = x.shape
    t = x.reshape(rows, cols // 128, 128)
    amax = t.abs().amax(dim=2)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax))
    e = e.clamp(-127, 127)
    scaled = (t * torch.exp2(-e)[:, :, None]).to(torch.float32)
    q = scaled.to(torch.float8_e4m3fn).view(torch.uint8).reshape(rows, cols).numpy()
    sf = (e + 127).to(torch.uint8).numpy()
    return q, sf


def test_matches_library_recipe_tiny():
    x = synthetic.tiny()["x"]
    q, sf = oracle.quantize_rowwise(x)
    rq, rsf = library_quantize(x)
    assert np.array_equal(sf, rsf)
    assert np.array_equal(q, rq)


def test_matches_library_recipe_random_shapes():
    for seed, (r, c) in enumerate([(1, 128), (3, 384), (130, 256), (64, 1024)]):
        x = synthetic.scaled_normal(r, c, seed=seed + 10, row_sigma=3.0)
        q, sf = oracle.quantize_rowwise(x)
        rq, rsf = library_quantize(x)
        assert np.array_equal(sf, rsf) and np.array_equal(q, rq)


def test_golden_tiles():
    for line in open(os.path.join(GOLDEN, "quantize_examples.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        amax, probe, e, ca, cp = line.split()
        vals = np.zeros(128, np.float32)
        vals[0], vals[1] = float(amax), float(probe)
        q, sf = oracle.quantize_rowwise(bf16_bits(vals).reshape(1, 128))
        assert int(sf[0, 0]) - 127 == int(e)
        assert q[0, 0] == int(ca, 16) and q[0, 1] == int(cp, 16), line
        assert np.all(q[0, 2:] == 0)


def test_representable_tile_reproduces_codes():
    """A tile whose values are all E4M3 values with amax = 448 is reproduced byte for
    byte (e = 0, every value exact)."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    rng = np.random.default_rng(3)
    for _ in range(20):
        tile = rng.choice(codes, 128)
        tile[rng.integers(128)] = 0x7E
        vals = oracle.e4m3_decode(tile).astype(np.float32)
        q, sf = oracle.quantize_rowwise(bf16_bits(vals).reshape(1, 128))
        assert sf[0, 0] == 127
        # -0 and +0 both decode to zero; compare values, and bytes elsewhere
        nz = vals != 0
        assert np.array_equal(q[0][nz], tile[nz])


def test_max_code_band_and_zero_tiles():
    x = synthetic.stress(rows=256, cols=1024, seed=4)["x"]
    q, sf = oracle.quantize_rowwise(x)
    mags = (q & 0x7F).reshape(256, 8, 128).max(axis=2)
    xz = (x.reshape(256, 8, 128) & 0x7FFF).max(axis=2) == 0
    assert np.all(sf[xz] == 127) and np.all(mags[xz] == 0)
    assert np.all((mags[~xz] >= 0x76) & (mags[~xz] <= 0x7E))
