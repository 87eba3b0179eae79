"""GPU parity: fused SwiGLU+quantize (+ direct transpose), fused permute+pad+quantize and
the grouped direct transpose on its output, against the CPU oracle, byte for byte."""
import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, dev, device_status_ok, host

pytestmark = pytest.mark.gpu


def check_swiglu(d, transposed=True):
    q, sf, qt, sft = sat.swiglu_quant(dev(d["gate"]), dev(d["up"]), transposed=transposed)
    device_status_ok()
    oq, osf, oqt, osft = oracle.swiglu_quant(d["gate"], d["up"], transposed=transposed)
    assert_bytes_equal(host(sf), osf, "SF")
    assert_bytes_equal(host(q), oq, "Q")
    if transposed:
        assert_bytes_equal(host(sft), osft, "SF^T")
        assert_bytes_equal(host(qt), oqt, "Q^T")


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (640, 1024), (1024, 2048)])
def test_swiglu_shapes(rows, cols):
    check_swiglu(synthetic.swiglu(rows=rows, cols=cols, seed=rows + 3 * cols))


def test_swiglu_rowwise_only_ragged_rows():
    check_swiglu(synthetic.swiglu(rows=300, cols=256, seed=5), transposed=False)


def test_swiglu_exp_range_edges():
    """Gate values that reach the exp spec's clamps and the division's extremes."""
    rows, cols = 128, 256
    g = np.linspace(-120, 120, rows * cols, dtype=np.float32).reshape(rows, cols)
    u = np.ones((rows, cols), np.float32)
    u[::2] = -3.0
    d = {"gate": synthetic._bf16_bits(g), "up": synthetic._bf16_bits(u)}
    check_swiglu(d)


def test_swiglu_config_full():
    check_swiglu(synthetic.swiglu())


def test_swiglu_persistent_ragged_rows():
    """More blocks than resident CTAs (each CTA loops over several), last row block ragged."""
    check_swiglu(synthetic.swiglu(rows=4100, cols=1536, seed=9), transposed=False)


def test_swiglu_every_binade():
    """Gates from BF16 subnormals to 2^127 in one tensor: tiny, tabulated and huge inputs
    mixed within warps, through the persistent loop."""
    check_swiglu(synthetic.swiglu_wide(seed=3, rows=4096, cols=2048))


# ------------------------------------------------------------------ permute

def check_permute(d, E, align):
    x, idx = d["x"], d["topk_idx"]
    q, sf, off, rmap = sat.permute_pad_quant(dev(x), dev(idx), E, align)
    device_status_ok()
    oq, osf, ooff, ormap = oracle.permute_pad_quant(x, idx, E, align)
    assert_bytes_equal(host(off), ooff, "expert offsets")
    assert_bytes_equal(host(rmap), ormap, "row_id_map")
    n = int(ooff[-1])
    assert_bytes_equal(host(sf)[:n], osf[:n], "SF")
    assert_bytes_equal(host(q)[:n], oq[:n], "Q")
    return q, sf, off, oq, osf, ooff


@pytest.mark.parametrize("tokens,hidden,E,K,align", [(8, 128, 4, 2, 16), (100, 256, 8, 2, 16),
                                                      (512, 384, 32, 8, 128), (3000, 256, 16, 4, 1),
                                                      (1500, 512, 7, 3, 64)])
def test_permute_shapes(tokens, hidden, E, K, align):
    rng = np.random.default_rng(tokens)
    d = {"x": synthetic.scaled_normal(tokens, hidden, seed=tokens + 1),
         "topk_idx": synthetic.zipf_topk(tokens, E, K, rng)}
    check_permute(d, E, align)


def test_permute_with_duplicate_and_skewed_routing():
    tokens, hidden, E = 700, 256, 5
    idx = np.zeros((tokens, 3), np.int32)
    idx[:, 1] = 0           # every token sends two slots to expert 0
    idx[::7, 2] = 4
    d = {"x": synthetic.scaled_normal(tokens, hidden, seed=9), "topk_idx": idx}
    check_permute(d, E, 128)


def test_permute_bad_index_sets_device_status():
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.tensor([[0], [1], [9], [2]], dtype=torch.int32, device="cuda")
    sat.permute_pad_quant(x, idx, 4, 16)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE


def test_permute_zero_tokens():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((0, 8), dtype=torch.int32, device="cuda")
    q, sf, off, rmap = sat.permute_pad_quant(x, idx, 32, 128)
    device_status_ok()
    assert torch.all(off == 0)


def test_moe_config_permute_then_grouped_transpose():
    """The MoE workload end to end: permute+pad(128)+quantize, then the grouped direct
    transpose on the device-resident offsets.  Every byte of every expert group's Q^T and
    SF^T (all offsets[E] rows) is compared with the oracle's grouped transpose of the
    oracle's permuted codes."""
    d = synthetic.moe()
    q, sf, off, oq, osf, ooff = check_permute(d, 32, 128)
    qt, sft = sat.direct_transpose(q, sf, off)
    device_status_ok()
    H = q.shape[1]
    n = int(ooff[-1])
    want_qt, want_sft = oracle.direct_transpose(oq, osf, ooff)
    assert_bytes_equal(host(sft).reshape(-1)[:H * n // 128], want_sft[:H * n // 128], "grouped SF^T")
    assert_bytes_equal(host(qt).reshape(-1)[:H * n], want_qt[:H * n], "grouped Q^T")


def test_bounded_wait_expires_cleanly():
    sat.fp8q_debug_expire_wait(2_000_000)  # 2 ms, nobody arrives
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_TIMEOUT
    # the context is still usable
    x = dev(synthetic.scaled_normal(128, 128, seed=1))
    q, sf = sat.quantize_rowwise(x)
    device_status_ok()


# ------------------------------------------------------------------ FP8-input permute

def check_permute_fp8(x_bits, idx, E, align):
    oq0, osf0 = oracle.quantize_rowwise(x_bits)
    q, sf, off, rmap = sat.permute_pad_fp8(dev(oq0), dev(osf0), dev(idx), E, align)
    device_status_ok()
    oq, osf, ooff, ormap = oracle.permute_pad_fp8(oq0, osf0, idx, E, align)
    assert_bytes_equal(host(off), ooff, "expert offsets")
    assert_bytes_equal(host(rmap), ormap, "row_id_map")
    n = int(ooff[-1])
    assert_bytes_equal(host(sf)[:n], osf[:n], "SF")
    assert_bytes_equal(host(q)[:n], oq[:n], "Q")
    return q, sf, off


@pytest.mark.parametrize("tokens,hidden,E,K,align", [(8, 128, 4, 2, 16), (100, 256, 8, 2, 16),
                                                      (512, 384, 32, 8, 128), (3000, 256, 16, 4, 1),
                                                      (1500, 512, 7, 3, 64)])
def test_permute_fp8_shapes(tokens, hidden, E, K, align):
    rng = np.random.default_rng(tokens + 5)
    x = synthetic.scaled_normal(tokens, hidden, seed=tokens + 2)
    check_permute_fp8(x, synthetic.zipf_topk(tokens, E, K, rng), E, align)


def test_permute_fp8_equals_fused_permute_quantize_on_gpu():
    """On the MoE workload: quantize on the GPU, permute the FP8 rows, and compare with the
    fused BF16 permute+quantize - the same bytes in every written row."""
    d = synthetic.moe()
    x, idx = dev(d["x"]), dev(d["topk_idx"])
    q0, sf0 = sat.quantize_rowwise(x)
    a = sat.permute_pad_fp8(q0, sf0, idx, 32, 128)
    b = sat.permute_pad_quant(x, idx, 32, 128)
    device_status_ok()
    n = int(b[2][-1].item())
    assert torch.equal(a[2], b[2]) and torch.equal(a[3], b[3])
    assert torch.equal(a[0][:n], b[0][:n]) and torch.equal(a[1][:n], b[1][:n])


def test_permute_fp8_moe_config_full():
    d = synthetic.moe()
    check_permute_fp8(d["x"], d["topk_idx"], 32, 128)


def test_permute_fp8_bad_index_sets_device_status():
    q = torch.zeros((4, 128), dtype=torch.uint8, device="cuda")
    sf = torch.full((4, 1), 127, dtype=torch.uint8, device="cuda")
    idx = torch.tensor([[0], [1], [9], [2]], dtype=torch.int32, device="cuda")
    sat.permute_pad_fp8(q, sf, idx, 4, 16)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE


@pytest.mark.parametrize("tokens,E,K", [(700, 300, 4), (2500, 512, 2), (1800, 513, 3), (600, 4096, 8)])
def test_permute_many_experts(tokens, E, K):
    """Routing with many experts, too wide for the fused rank kernel: the per-32-expert
    chunk scan and the eight-warp rank, with expert counts that are not multiples of 32
    (300, 513) and the 4096 maximum (one rank CTA per SM), uniform routing so most experts
    are hit."""
    rng = np.random.default_rng(E)
    idx = np.argsort(rng.random((tokens, E)), axis=1)[:, :K].astype(np.int32)
    d = {"x": synthetic.scaled_normal(tokens, 128, seed=E), "topk_idx": np.ascontiguousarray(idx)}
    check_permute(d, E, 16)
    check_permute_fp8(d["x"], d["topk_idx"], E, 16)


@pytest.mark.parametrize("tokens,E,K", [(40000, 256, 8), (16384, 4096, 8), (70000, 33, 8)])
def test_permute_wide_routing_many_chunks(tokens, E, K):
    """Hundreds of 1024-pair chunks: each warp of the chunk scan walks a range of several
    chunks in steps of eight with a ragged last step (313, 128 and 547 chunks), across
    expert blocks with a partial last block (33 experts).  The 256-expert case is the full
    top-8 routing of a 256-expert model; ids need not be distinct within a token."""
    rng = np.random.default_rng(tokens + E)
    if E <= 256:
        idx = np.argsort(rng.random((tokens, E)), axis=1)[:, :K].astype(np.int32)
    else:
        idx = rng.integers(0, E, (tokens, K), dtype=np.int32)
    d = {"x": synthetic.scaled_normal(tokens, 128, seed=E + 1), "topk_idx": np.ascontiguousarray(idx)}
    check_permute(d, E, 16)
    check_permute_fp8(d["x"], d["topk_idx"], E, 128)
