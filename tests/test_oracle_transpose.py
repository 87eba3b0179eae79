"""Pins for the oracle's scaling-aware direct transpose and the naive
dequant -> transpose -> requant baseline (FP8-Flow-MoE review, sections 问题与动机 and
核心方法; DeepSeek FP8 与 DeepGEMM §1: wgrad reduces over tokens, so it consumes the
column-wise layout)."""
import numpy as np
import pytest
import torch

import oracle
from scaling_aware_transpose_b200 import synthetic


def fp8_decode_t(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64)


def library_direct(q: np.ndarray, sf: np.ndarray):
    """Direct transpose from library primitives: torch decodes the codes, each 128x128
    block takes Smax = max row scale, values are divided by Smax/S_row (exact in
    float32 while the result stays above 2^-149) and torch's float8 cast rounds."""
    rows, cols = q.shape
    nb, nt = rows // 128, cols // 128
    e = torch.from_numpy(sf.astype(np.int64) - 127)                      # [rows, nt]
    emax = e.reshape(nb, 128, nt).amax(dim=1)                            # [nb, nt]
    k = emax.repeat_interleave(128, dim=0) - e                           # [rows, nt]
    v = fp8_decode_t(q) * torch.exp2(-k.to(torch.float64)).repeat_interleave(128, dim=1)
    qt = v.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy().T.copy()
    sft = np.repeat((emax + 127).numpy().astype(np.uint8).T, 128, axis=0)  # [cols, nb]
    return qt, sft


def library_naive(q: np.ndarray, sf: np.ndarray):
    """Naive path from library primitives: dequantize to BF16 (torch), transpose,
    requantize each 128-token column tile with S = 2^ceil(log2(amax/448))."""
    rows, cols = q.shape
    e = torch.from_numpy(sf.astype(np.int64) - 127).repeat_interleave(128, dim=1)
    v = (fp8_decode_t(q) * torch.exp2(e.to(torch.float64))).to(torch.float32).to(torch.bfloat16)
    vt = v.t().contiguous().to(torch.float64).reshape(cols, rows // 128, 128)
    amax = vt.abs().amax(dim=2)
    ec = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax)).clamp(-127, 127)
    qt = (vt * torch.exp2(-ec)[:, :, None]).to(torch.float32).to(torch.float8_e4m3fn)
    return qt.view(torch.uint8).reshape(cols, rows).numpy(), (ec + 127).to(torch.uint8).numpy()


@pytest.fixture(scope="module")
def tiny_q():
    x = synthetic.tiny()["x"]
    return oracle.quantize_rowwise(x)


def test_direct_matches_library_recipe(tiny_q):
    q, sf = tiny_q
    qt, sft = oracle.direct_transpose(q, sf)
    rqt, rsft = library_direct(q, sf)
    assert np.array_equal(sft, rsft)
    assert np.array_equal(qt, rqt)


def test_direct_matches_library_recipe_stress():
    x = synthetic.stress(rows=512, cols=768, seed=5)["x"]
    q, sf = oracle.quantize_rowwise(x)
    qt, sft = oracle.direct_transpose(q, sf)
    rqt, rsft = library_direct(q, sf)
    assert np.array_equal(sft, rsft) and np.array_equal(qt, rqt)


def test_naive_matches_library_recipe(tiny_q):
    q, sf = tiny_q
    qt, sft = oracle.naive_transpose(q, sf)
    rqt, rsft = library_naive(q, sf)
    assert np.array_equal(sft, rsft)
    assert np.array_equal(qt, rqt)


def test_direct_invariants(tiny_q):
    q, sf = tiny_q
    rows, cols = q.shape
    qt, sft = oracle.direct_transpose(q, sf)
    e = sf.astype(np.int64) - 127
    emax = e.reshape(rows // 128, 128, -1).max(axis=1)
    # SF^T holds the block's max row exponent, replicated over its 128 channels
    assert np.array_equal(sft.astype(np.int64) - 127, np.repeat(emax.T, 128, axis=0))
    k = np.repeat(emax, 128, axis=0) - e                     # [rows, nt]
    kk = np.repeat(k, 128, axis=1)                           # [rows, cols]
    # rows with k = 0 are a pure byte transpose
    assert np.array_equal(qt.T[kk == 0], q[kk == 0])
    # magnitudes never grow (no overflow) and the sign is kept
    assert np.all((qt.T & 0x7F) <= (q & 0x7F))
    assert np.array_equal(qt.T & 0x80, q & 0x80)
    # every value that stays representable is carried over exactly
    vin = oracle.dequant_rowwise(q, sf)
    vout = oracle.dequant_colwise(qt, sft)
    shifted = oracle.e4m3_decode(q) * np.exp2(-kk.astype(np.float64))
    rep = oracle.e4m3_decode(oracle.e4m3_encode(shifted)) == shifted
    assert np.array_equal(vout[rep], vin[rep])


def test_naive_never_farther_than_direct(tiny_q):
    """Per element, requantizing with the fresh column exponent e_c <= e_max rounds to
    a grid that contains the direct transpose's grid, so it is never farther from the
    dequantized value v (nearest on a superset)."""
    q, sf = tiny_q
    v = oracle.dequant_rowwise(q, sf)
    d = oracle.dequant_colwise(*oracle.direct_transpose(q, sf))
    n = oracle.dequant_colwise(*oracle.naive_transpose(q, sf))
    assert np.all(np.abs(v - n) <= np.abs(v - d))


def test_naive_equals_direct_when_scales_agree():
    """Special case: every row tile has e = 0 and every column tile of every block
    holds a code of magnitude >= 224, so e_c = e_max = 0 and both paths are the
    plain byte transpose."""
    rng = np.random.default_rng(6)
    rows, cols = 256, 384
    q = rng.integers(0, 0x7F, size=(rows, cols), dtype=np.uint8)
    q |= rng.integers(0, 2, size=q.shape, dtype=np.uint8) << 7
    q[::128, :] = 0x7E            # one 448 in every column tile (row 0 of each block)
    for r in range(rows):
        q[r, ::128] = 0x7E        # and one 448 in every row tile
    sf = np.full((rows, cols // 128), 127, np.uint8)
    d, dsf = oracle.direct_transpose(q, sf)
    n, nsf = oracle.naive_transpose(q, sf)
    assert np.array_equal(d, q.T) and np.array_equal(n, q.T)
    assert np.all(dsf == 127) and np.all(nsf == 127)


def test_grouped_equals_per_group_dense():
    x = synthetic.scaled_normal(640, 256, seed=7, row_sigma=2.0)
    q, sf = oracle.quantize_rowwise(x)
    off = np.array([0, 128, 128, 512, 640], np.int32)   # includes an empty group
    for fn in (oracle.direct_transpose, oracle.naive_transpose):
        qt, sft = fn(q, sf, off)
        for g in range(len(off) - 1):
            a, b = off[g], off[g + 1]
            if a == b:
                continue
            dq, ds = fn(q[a:b], sf[a:b])
            M = b - a
            assert np.array_equal(qt[256 * a: 256 * a + 256 * M].reshape(256, M), dq)
            assert np.array_equal(sft[256 * a // 128: 256 * a // 128 + 256 * M // 128].reshape(256, M // 128), ds)


def test_bad_groups_rejected():
    q = np.zeros((256, 128), np.uint8)
    sf = np.full((256, 1), 127, np.uint8)
    for off in ([0, 100, 256], [0, 256, 128], [128, 256], [0, 384]):
        with pytest.raises(oracle.OracleError):
            oracle.direct_transpose(q, sf, np.array(off, np.int32))


def test_error_report_runs(tiny_q):
    """Reported numbers (not parity): relative RMS of each column-wise result against
    the original BF16 input, and against the row-wise dequantized values."""
    q, sf = tiny_q
    x = synthetic.bf16_bits_to_f32(synthetic.tiny()["x"]).astype(np.float64)
    v = oracle.dequant_rowwise(q, sf)
    d = oracle.dequant_colwise(*oracle.direct_transpose(q, sf))
    n = oracle.dequant_colwise(*oracle.naive_transpose(q, sf))
    f = oracle.naive_fp32_colwise(v)
    for arr in (d, n, f):
        assert 0.0 <= oracle.rel_rms(arr, x) < 0.2
        assert 0.0 <= oracle.calc_diff(arr, x) < 0.05
    assert oracle.rel_rms(v, v) == 0.0


def _row_rel_rms(a, ref):
    num = np.sqrt(((a - ref) ** 2).sum(axis=1))
    den = np.sqrt((ref ** 2).sum(axis=1))
    return num[den > 0] / den[den > 0]


@pytest.mark.parametrize("recipe", ["dense", "stress"])
def test_error_report_direct_vs_double_quantization(recipe):
    """The error report on 1024 rows of the dense and range-stress recipes (reported
    numbers; run with -s to print them).  The column-wise result of the direct transpose
    stays within the row-wise quantization's own error of X, while a requantization with
    fresh non-power-of-two column scales (the double quantization the method avoids)
    adds two orders of magnitude more error relative to the row-wise values."""
    d = synthetic.dense(seed=0, rows=1024) if recipe == "dense" else synthetic.stress(seed=0, rows=1024)
    x = synthetic.bf16_bits_to_f32(d["x"]).astype(np.float64)
    q, sf = oracle.quantize_rowwise(d["x"])
    v = oracle.dequant_rowwise(q, sf)
    res = {"row-wise": v,
           "direct": oracle.dequant_colwise(*oracle.direct_transpose(q, sf)),
           "naive (pow2)": oracle.dequant_colwise(*oracle.naive_transpose(q, sf)),
           "naive (fp32 amax/448)": oracle.naive_fp32_colwise(v)}
    print(f"\n{recipe} [1024x7168]: rel RMS vs X | vs row-wise values | calc_diff vs X | per-row rel RMS vs X p50 / p99")
    for name, a in res.items():
        rr = _row_rel_rms(a, x)
        print(f"  {name:22s} {oracle.rel_rms(a, x):.4e} | {oracle.rel_rms(a, v):.4e} | {oracle.calc_diff(a, x):.3e} | "
              f"{np.percentile(rr, 50):.3e} / {np.percentile(rr, 99):.3e}")
    extra_direct = oracle.rel_rms(res["direct"], v)
    extra_fp32 = oracle.rel_rms(res["naive (fp32 amax/448)"], v)
    assert extra_direct * 100 < extra_fp32
    assert oracle.rel_rms(res["direct"], x) < oracle.rel_rms(res["naive (fp32 amax/448)"], x)
