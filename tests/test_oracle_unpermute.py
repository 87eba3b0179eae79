"""Pins for the oracle's fused unpermute + unpad (combine side of the permute:
FP8-Flow-MoE review, 核心方法, Fused Permute+Padding / Unpermute+Unpadding).

The combine's arithmetic is this library's reading (fp32 multiply-add per slot in slot
order, BF16 round-to-nearest-even); the pins check it against hand-worked values, an
independent float64 emulation of the same sequence with torch's BF16 rounding, the
permute round trip, and the exact sum within the fp32 error bound."""
import os

import numpy as np
import pytest
import torch

import oracle
from scaling_aware_transpose_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits_of(f32):
    t = torch.from_numpy(np.ascontiguousarray(f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def read_fixture():
    blocks, cur = [], None
    with open(os.path.join(GOLDEN, "unpermute_examples.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if not line:
                continue
            if line[0] == "y":
                cur = {"kind": line[1], "vals": line[2:], "cases": []}
                blocks.append(cur)
            else:
                _, name, rows, w, want = line
                cur["cases"].append((name, [int(r) for r in rows.split(",")],
                                     None if w == "none" else [float(v) for v in w.split(",")], int(want, 16)))
    return blocks


def test_golden_examples():
    n = 0
    for blk in read_fixture():
        if blk["kind"] == "bf16":
            y = np.repeat(bf16_bits_of(np.array([float(v) for v in blk["vals"]], np.float32))[:, None], 128, axis=1)
            sf = None
        else:
            pairs = [v.split(":") for v in blk["vals"]]
            y = np.repeat(np.array([int(c, 16) for c, _ in pairs], np.uint8)[:, None], 128, axis=1)
            sf = np.array([[int(s)] for _, s in pairs], np.uint8)
        for name, rows, w, want in blk["cases"]:
            wts = None if w is None else np.array([w], np.float32)
            out = oracle.unpermute_unpad(y, np.array(rows, np.int32), 2, wts, y_sf=sf)
            assert np.all(out == want), (name, hex(int(out[0, 0])), hex(want))
            n += 1
    assert n == 12


def emulate(y_f32, rmap, w):
    """The same fp32 fma chain, emulated in float64 (a*b is exact in double; the sum is
    rounded once to double, then to float32), BF16 rounding by torch."""
    T, K = rmap.shape
    acc = np.full((T, y_f32.shape[1]), -0.0, np.float32)
    for s in range(K):
        ws = np.ones(T, np.float64) if w is None else w[:, s].astype(np.float64)
        acc = (ws[:, None] * y_f32[rmap[:, s]].astype(np.float64) + acc.astype(np.float64)).astype(np.float32)
    return bf16_bits_of(acc)


@pytest.mark.parametrize("K,weighted", [(1, False), (2, True), (8, True), (8, False), (3, True)])
def test_bf16_matches_independent_emulation(K, weighted):
    T, H, R = 96, 384, 96 * K + 40
    rng = np.random.default_rng(K)
    y = synthetic.scaled_normal(R, H, seed=K, row_sigma=2.0)
    rmap = rng.permutation(R)[: T * K].astype(np.int32).reshape(T, K)   # distinct rows, 40 never read
    w = rng.dirichlet(np.ones(K), size=T).astype(np.float32) if weighted else None
    got = oracle.unpermute_unpad(y, rmap, K, w)
    want = emulate(synthetic.bf16_bits_to_f32(y), rmap, w)
    assert np.array_equal(got, want)


def test_fp8_matches_independent_emulation():
    T, H, R, K = 64, 512, 600, 4
    rng = np.random.default_rng(11)
    x = synthetic.stress(rows=R, cols=H, seed=3)["x"]
    q, sf = oracle.quantize_rowwise(x)
    rmap = rng.permutation(R)[: T * K].astype(np.int32).reshape(T, K)
    w = rng.dirichlet(np.ones(K), size=T).astype(np.float32)
    dec = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    v = (dec * np.exp2(np.repeat(sf.astype(np.float64) - 127, 128, axis=1))).astype(np.float32)
    assert np.array_equal(oracle.unpermute_unpad(q, rmap, K, w, y_sf=sf), emulate(v, rmap, w))


def test_permute_round_trip_bf16():
    """K = 1, unit weights: unpermuting the permuted rows gives X back exactly, whatever the
    padding rows hold."""
    d = synthetic.moe(tokens=200, hidden=256, num_experts=6, topk=1, seed=4)
    _, _, off, rmap = oracle.permute_pad_quant(d["x"], d["topk_idx"], 6, 16)
    R = int(off[-1])
    y = synthetic.scaled_normal(R, 256, seed=9)          # padding rows keep this noise
    y[rmap] = d["x"]
    assert np.array_equal(oracle.unpermute_unpad(y, rmap, 1), d["x"])


@pytest.mark.parametrize("seed", [5, 8])
def test_permute_round_trip_fp8(seed):
    """K = 1 on the FP8 permute output: the BF16 rounding of the row-wise dequantization
    (torch decodes the codes) - the permute's rows come back to their tokens, codes of
    -0 included."""
    d = synthetic.moe(tokens=150 * seed, hidden=384, num_experts=5, topk=1, seed=seed)
    pq, psf, off, rmap = oracle.permute_pad_quant(d["x"], d["topk_idx"], 5, 128)
    q, sf = oracle.quantize_rowwise(d["x"])
    dec = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    v = (dec * np.exp2(np.repeat(sf.astype(np.float64) - 127, 128, axis=1))).astype(np.float32)
    assert np.array_equal(oracle.unpermute_unpad(pq, rmap, 1, y_sf=psf), bf16_bits_of(v))


def test_sum_of_copies_is_k_times_row():
    """Backward of the permute (unit weights) on K identical copies: K * x, exact for
    K = 2, 4, 8 (a power-of-two multiple of a BF16 value is a BF16 value)."""
    d = synthetic.moe(tokens=64, hidden=128, num_experts=8, topk=8, seed=6)
    _, _, off, rmap = oracle.permute_pad_quant(d["x"], d["topk_idx"], 8, 16)
    y = np.zeros((int(off[-1]), 128), np.uint16)
    y[rmap] = np.repeat(d["x"], 8, axis=0)
    for K in (2, 4, 8):
        out = oracle.unpermute_unpad(y, rmap.reshape(64, 8)[:, :K], K)
        assert np.array_equal(out, bf16_bits_of(synthetic.bf16_bits_to_f32(d["x"]) * K))


def test_within_fp32_error_bound_of_exact_sum():
    T, H, K, R = 128, 256, 8, 1200
    rng = np.random.default_rng(7)
    y = synthetic.scaled_normal(R, H, seed=7, row_sigma=1.0)
    rmap = rng.permutation(R)[: T * K].astype(np.int32).reshape(T, K)
    w = rng.dirichlet(np.ones(K), size=T).astype(np.float32)
    out = synthetic.bf16_bits_to_f32(oracle.unpermute_unpad(y, rmap, K, w)).astype(np.float64)
    yv = synthetic.bf16_bits_to_f32(y).astype(np.float64)
    terms = w.astype(np.float64)[:, :, None] * yv[rmap]
    exact = terms.sum(axis=1)
    bound = K * 2.0 ** -24 * np.abs(terms).sum(axis=1) + 2.0 ** -8 * np.abs(exact) + 2.0 ** -133
    assert np.all(np.abs(out - exact) <= bound)


def test_bad_row_index_rejected():
    y = np.zeros((4, 128), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.unpermute_unpad(y, np.array([[0, 4]], np.int32), 2)
    with pytest.raises(oracle.OracleError):
        oracle.unpermute_unpad(y, np.array([[-1, 0]], np.int32), 2)
