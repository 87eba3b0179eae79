"""The seeded input generators: deterministic, the stated shapes, and the stated
distribution features (row factors, outlier channels, tile amax range, zero tiles,
Zipf routing)."""
import numpy as np

from scaling_aware_transpose_b200 import synthetic


def f32(bits):
    return synthetic.bf16_bits_to_f32(bits)


def test_deterministic_and_seeded():
    a = synthetic.tiny(seed=0)["x"]
    assert np.array_equal(a, synthetic.tiny(seed=0)["x"])
    assert not np.array_equal(a, synthetic.tiny(seed=1)["x"])
    assert a.shape == (256, 512) and a.dtype == np.uint16


def test_dense_outlier_channels():
    d = synthetic.dense(rows=512, cols=7168)
    x = np.abs(f32(d["x"]))
    assert d["outlier_channels"].size == 7
    col = x.mean(axis=0)
    others = np.delete(col, d["outlier_channels"])
    assert col[d["outlier_channels"]].min() > 20 * np.median(others)


def test_stress_tile_amax_range_and_zero_tiles():
    d = synthetic.stress(rows=2048, cols=1024, seed=3)
    t = np.abs(f32(d["x"])).reshape(2048, 8, 128).max(axis=2)
    z = d["zero_tiles"]
    assert np.all(t[z] == 0) and 0.002 < z.mean() < 0.03
    nz = t[~z]
    lg = np.log2(nz)
    assert lg.min() >= -20.01 and lg.max() <= 12.01
    assert lg.min() < -19 and lg.max() > 11  # the range is covered


def test_swiglu_row_factor_shared():
    d = synthetic.swiglu(rows=64, cols=2048, seed=4)
    g, u = np.abs(f32(d["gate"])), np.abs(f32(d["up"]))
    r = np.corrcoef(np.log(g.mean(axis=1)), np.log(u.mean(axis=1)))[0, 1]
    assert r > 0.95


def test_zipf_topk_distinct_and_skewed():
    rng = np.random.default_rng(5)
    idx = synthetic.zipf_topk(4096, 32, 8, rng)
    assert idx.shape == (4096, 8) and idx.dtype == np.int32
    assert all(len(set(r)) == 8 for r in idx[:500].tolist())
    counts = np.bincount(idx.ravel(), minlength=32)
    assert counts[0] > counts[15] > counts[31]
    assert counts.sum() == 4096 * 8


def test_moe_combine_inputs():
    d = synthetic.moe_combine(tokens=300, hidden=256, rows=2500, topk=8, seed=2)
    assert d["y"].shape == (2500, 256) and d["y"].dtype == np.uint16
    w = d["weights"]
    assert w.shape == (300, 8) and w.dtype == np.float32 and np.all(w > 0)
    assert np.allclose(w.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)
    again = synthetic.moe_combine(tokens=300, hidden=256, rows=2500, topk=8, seed=2)
    assert np.array_equal(again["y"], d["y"]) and np.array_equal(again["weights"], w)


def test_swiglu_wide_spans_binades_and_is_seeded():
    a = synthetic.swiglu_wide(seed=1, rows=64, cols=256)
    b = synthetic.swiglu_wide(seed=1, rows=64, cols=256)
    assert np.array_equal(a["gate"], b["gate"]) and np.array_equal(a["up"], b["up"])
    g = synthetic.bf16_bits_to_f32(a["gate"])
    assert np.isfinite(g).all() and np.abs(g).max() < 2.0 ** 121
    mag = a["gate"] & 0x7FFF
    assert (mag < 0x80).any() and (mag > 0x4300).any()   # subnormal and huge gates present
