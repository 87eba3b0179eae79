"""Pins for the oracle's fused SwiGLU+quantize (FP8-Flow-MoE review, 核心方法: Fused
SwiGLU+Quantization) and fused permute+pad+quantize (核心方法: Fused Permute+Padding;
DeepSeek FP8 与 DeepGEMM §5.6: experts' rows concatenated along M)."""
import math

import numpy as np
import pytest

import oracle
from scaling_aware_transpose_b200 import synthetic


def ulp_distance_f32(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    ia = a.astype(np.float32).view(np.int32).astype(np.int64)
    ib = b.astype(np.float32).view(np.int32).astype(np.int64)
    ia = np.where(ia < 0, -(ia & 0x7FFFFFFF), ia)
    ib = np.where(ib < 0, -(ib & 0x7FFFFFFF), ib)
    return np.abs(ia - ib)


def test_exp_spec_constants_are_derived():
    c = oracle.exp_spec_constants()
    ln2 = math.log(2.0)
    hi = np.float32(np.frombuffer(np.uint32(0x3F317200).tobytes(), np.float32)[0])
    assert c[0] == np.float32(math.log2(math.e))
    assert c[1] == hi and abs(float(hi) - ln2) < 2e-6
    assert c[2] == np.float32(ln2 - float(hi))
    for k in range(8):
        assert c[3 + k] == np.float32(1.0 / math.factorial(k))


def test_exp_spec_accuracy_vs_libm():
    """Within 2 ulp of exp over the normal-result range, measured against exp in
    double rounded once to fp32."""
    rng = np.random.default_rng(8)
    a = np.concatenate([rng.uniform(-87.0, 88.5, 400000), rng.uniform(-1, 1, 100000),
                        np.linspace(-87, 88.5, 100001)]).astype(np.float32)
    got = oracle.exp_spec(a)
    ref = np.exp(a.astype(np.float64)).astype(np.float32)
    d = ulp_distance_f32(got, ref)
    assert d.max() <= 2, float(d.max())


def test_exp_spec_special_values():
    a = np.array([0.0, 89.5, 1e30, -104.5, -1e30, 88.0, -103.0], np.float32)
    e = oracle.exp_spec(a)
    assert e[0] == 1.0 and np.isinf(e[1]) and np.isinf(e[2])
    assert e[3] == 0.0 and e[4] == 0.0
    assert np.isfinite(e[5]) and e[6] > 0  # subnormal, not flushed


def test_swiglu_special_values():
    g = np.array([0.0, 30.0, -200.0, 1.0, -1.0], np.float32)
    u = np.array([5.0, 2.0, 3.0, 1.0, 1.0], np.float32)
    y = oracle.swiglu(g, u)
    assert y[0] == 0.0
    assert y[1] == np.float32(60.0)  # silu(30) rounds to 30 in fp32
    assert y[2] == 0.0 and np.signbit(y[2])
    ref = np.array([1.0 / (1.0 + math.exp(-1.0)), -1.0 / (1.0 + math.exp(1.0))])
    assert np.allclose(y[3:], ref, rtol=3e-7)


def test_swiglu_close_to_double_reference():
    rng = np.random.default_rng(9)
    g = rng.standard_normal(200000).astype(np.float32) * 4
    u = rng.standard_normal(200000).astype(np.float32)
    y = oracle.swiglu(g, u).astype(np.float64)
    gd, ud = g.astype(np.float64), u.astype(np.float64)
    ref = gd / (1.0 + np.exp(-gd)) * ud
    assert np.all(np.abs(y - ref) <= 4 * np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64) + 1e-45)


def test_silu_closed_forms_over_every_bf16_gate():
    """On BF16 gates the spec's silu(g) = g / (1 + exp(-g)) reduces to one IEEE operation
    outside one magnitude range: below BF16 0x33C1 the denominator rounds to exactly 2
    (silu = RN(g/2)); from 89 up exp(-g) <= 2^-24 and the denominator rounds to 1
    (silu = g, true already from 16.75); from -89 down exp(-g) overflows to +inf
    (silu = -0).  These are the facts a kernel may use to tabulate only the rest; the
    thresholds are tight at the low end (0x33C1 itself breaks the first rule)."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    bits = bits[(bits & 0x7F80) != 0x7F80]
    g = (bits << 16).view(np.float32)
    s = oracle.swiglu(g, np.ones_like(g)).view(np.uint32)
    mag, neg = bits & 0x7FFF, bits >> 15
    tiny = mag < 0x33C1
    half = (g[tiny].astype(np.float64) * 0.5).astype(np.float32)   # exact product, one rounding
    assert np.array_equal(s[tiny], half.view(np.uint32))
    big_pos = (mag >= 0x4186) & (neg == 0)
    assert np.array_equal(s[big_pos], g[big_pos].view(np.uint32))
    big_neg = (mag >= 0x42B2) & (neg == 1)
    assert (s[big_neg] == 0x80000000).all()
    # the low threshold is tight: the positive gate 0x33C1 does not give RN(g/2)
    g1 = np.array([(0x33C1 << 16)], np.uint32).view(np.float32)
    assert oracle.swiglu(g1, np.ones(1, np.float32)).view(np.uint32)[0] != (g1 * np.float32(0.5)).view(np.uint32)[0]
    # and just below 89 the negative side is not yet -0
    g2 = np.array([(0xC2B1 << 16)], np.uint32).view(np.float32)
    assert oracle.swiglu(g2, np.ones(1, np.float32)).view(np.uint32)[0] != 0x80000000


def test_swiglu_quant_is_quantize_of_swiglu_then_direct():
    d = synthetic.swiglu(rows=256, cols=384, seed=10)
    q, sf, qt, sft = oracle.swiglu_quant(d["gate"], d["up"])
    g = synthetic.bf16_bits_to_f32(d["gate"])
    u = synthetic.bf16_bits_to_f32(d["up"])
    y = oracle.swiglu(g, u)
    rq, rsf = oracle.quantize_rowwise_f32(y)
    assert np.array_equal(q, rq) and np.array_equal(sf, rsf)
    dqt, dsft = oracle.direct_transpose(q, sf)
    assert np.array_equal(qt, dqt) and np.array_equal(sft, dsft)
    q2, sf2, qt2, sft2 = oracle.swiglu_quant(d["gate"], d["up"], transposed=False)
    assert qt2 is None and np.array_equal(q2, q)


# ------------------------------------------------------------------ permute

def brute_permute(x_bits, idx, E, align):
    T, K = idx.shape
    H = x_bits.shape[1]
    pairs = {e: [] for e in range(E)}
    for t in range(T):
        for s in range(K):
            pairs[int(idx[t, s])].append((t, s))
    off = [0]
    for e in range(E):
        n = len(pairs[e])
        off.append(off[-1] + (n + align - 1) // align * align)
    rmap = np.zeros(T * K, np.int32)
    for e in range(E):
        for r, (t, s) in enumerate(pairs[e]):
            rmap[t * K + s] = off[e] + r
    qx, sfx = oracle.quantize_rowwise(x_bits)
    q = np.full((off[-1], H), 0xEE, np.uint8)
    sf = np.full((off[-1], H // 128), 0xEE, np.uint8)
    for p in range(T * K):
        q[rmap[p]], sf[rmap[p]] = qx[p // K], sfx[p // K]
    for e in range(E):
        for r in range(off[e] + len(pairs[e]), off[e + 1]):
            q[r], sf[r] = 0, 127
    return q, sf, np.array(off, np.int32), rmap


@pytest.mark.parametrize("align", [1, 2, 16])
def test_permute_brute_force_tiny(align):
    rng = np.random.default_rng(11 + align)
    T, E, K, H = 8, 4, 2, 256
    x = synthetic.scaled_normal(T, H, seed=12)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    q, sf, off, rmap = oracle.permute_pad_quant(x, idx, E, align)
    bq, bsf, boff, brmap = brute_permute(x, idx, E, align)
    n = boff[-1]
    assert np.array_equal(off, boff) and np.array_equal(rmap, brmap)
    assert np.array_equal(q[:n], bq) and np.array_equal(sf[:n], bsf)
    assert np.all(q[n:] == 0xEE) and np.all(sf[n:] == 0xEE)


def _check_permute_invariants(x, idx, E, align):
    """What the permute's definition fixes, checked without re-deriving it: each expert's
    segment is its pair count rounded up to `align`, the offsets are their exclusive scan,
    every pair has its own row inside its expert's segment, rows within a segment follow
    (token, slot) order with no gap, every row holds its token's codes and scales, and the
    padding rows are zero codes with scale byte 127."""
    T, K = idx.shape
    q, sf, off, rmap = oracle.permute_pad_quant(x, idx, E, align)
    counts = np.bincount(idx.ravel(), minlength=E)
    assert counts.sum() == T * K
    sizes = np.diff(off)
    assert off[0] == 0 and np.all(sizes % align == 0) and np.all(sizes >= counts) and np.all(sizes - counts < align)
    assert np.array_equal(sizes == 0, counts == 0)
    assert len(np.unique(rmap)) == rmap.size
    e_of = idx.ravel()
    assert np.all((rmap >= off[e_of]) & (rmap < off[e_of] + counts[e_of]))
    # stable order: within an expert the rows follow (token, slot) order
    order = np.argsort(e_of, kind="stable")
    assert np.array_equal(rmap[order], np.concatenate([np.arange(off[e], off[e] + counts[e]) for e in range(E)]))
    qx, sfx = oracle.quantize_rowwise(x)
    assert np.array_equal(q[rmap], np.repeat(qx, K, axis=0))
    assert np.array_equal(sf[rmap], np.repeat(sfx, K, axis=0))
    pad = np.ones(off[-1], bool)
    pad[rmap] = False
    assert np.all(q[:off[-1]][pad] == 0) and np.all(sf[:off[-1]][pad] == 127)


def test_permute_invariants_zipf():
    d = synthetic.moe(tokens=512, hidden=256, num_experts=32, topk=8, seed=13)
    _check_permute_invariants(d["x"], d["topk_idx"], 32, 128)


@pytest.mark.parametrize("T,E,K,align", [(2048, 4096, 8, 16), (3000, 513, 3, 1), (1500, 256, 8, 128)])
def test_permute_invariants_wide_routing(T, E, K, align):
    """Routings as wide as the library accepts (4096 experts, most of them empty), expert
    counts that are not multiples of 32, ids repeated within a token."""
    rng = np.random.default_rng(T + E)
    idx = rng.integers(0, E, (T, K), dtype=np.int32)
    idx[::5, 1] = idx[::5, 0]  # the same expert twice in one token
    _check_permute_invariants(synthetic.scaled_normal(T, 128, seed=E), idx, E, align)


def test_permute_rejects_bad_index():
    x = synthetic.scaled_normal(4, 128, seed=14)
    with pytest.raises(oracle.OracleError):
        oracle.permute_pad_quant(x, np.array([[0], [1], [5], [2]], np.int32), 4, 16)


# ------------------------------------------------------------------ FP8-input permute

@pytest.mark.parametrize("T,H,K,E,align", [(64, 256, 2, 4, 16), (300, 384, 8, 32, 128), (1, 128, 1, 1, 1),
                                           (129, 128, 3, 5, 7)])
def test_fp8_permute_equals_quantize_then_permute(T, H, K, E, align):
    """Quantization is row-local, so permuting the row-wise codes and scales must give
    byte for byte what the fused BF16 permute+quantize gives (same routing, offsets,
    padding rows)."""
    d = synthetic.moe(tokens=T, hidden=H, num_experts=E, topk=K, seed=T + E)
    q, sf = oracle.quantize_rowwise(d["x"])
    a = oracle.permute_pad_fp8(q, sf, d["topk_idx"], E, align)
    b = oracle.permute_pad_quant(d["x"], d["topk_idx"], E, align)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_fp8_permute_brute_force_rows():
    """Pure-Python gather: row row_id_map[t*K+s] holds token t's codes and scales."""
    d = synthetic.moe(tokens=40, hidden=256, num_experts=3, topk=2, seed=1)
    rng = np.random.default_rng(0)
    q = rng.integers(0, 256, size=(40, 256), dtype=np.uint8)
    sf = rng.integers(100, 140, size=(40, 2), dtype=np.uint8)
    oq, osf, off, rmap = oracle.permute_pad_fp8(q, sf, d["topk_idx"], 3, 16)
    for p in range(80):
        t = p // 2
        assert np.array_equal(oq[rmap[p]], q[t]) and np.array_equal(osf[rmap[p]], sf[t])
    used = set(rmap.tolist())
    for r in range(int(off[-1])):
        if r not in used:
            assert np.all(oq[r] == 0) and np.all(osf[r] == 127)


def test_fp8_permute_bad_index():
    q = np.zeros((4, 128), np.uint8)
    sf = np.full((4, 1), 127, np.uint8)
    with pytest.raises(oracle.OracleError):
        oracle.permute_pad_fp8(q, sf, np.array([[0], [1], [9], [2]], np.int32), 4, 16)
