"""GPU parity of the fused unpermute + unpad (combine side of the permute) against the
CPU oracle, byte for byte: BF16 and FP8 expert rows, routing weights and unit weights,
K = 1..8 (each its own FP8 specialisation) and 12, 16, ragged hidden sizes, the FP8 bulk-copy ring
(hidden % 512 == 0, K <= 8), the permute round trip, the full MoE workload, and bad row indices reported
through the status word."""
import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, dev, device_status_ok, host

pytestmark = pytest.mark.gpu


def case(T, H, K, R, seed, fp8):
    rng = np.random.default_rng(seed)
    rmap = rng.permutation(R)[: T * K].astype(np.int32)
    w = rng.dirichlet(np.ones(K), size=T).astype(np.float32)
    if fp8:
        y, sf = oracle.quantize_rowwise(synthetic.stress(rows=R, cols=H, seed=seed)["x"])
    else:
        y, sf = synthetic.scaled_normal(R, H, seed=seed, row_sigma=2.0), None
    return y, sf, rmap, w


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("T,H,K", [(1, 128, 1), (37, 384, 2), (64, 640, 3), (40, 512, 4), (257, 256, 5), (29, 896, 6),
                                   (50, 256, 7), (100, 1152, 8), (33, 7168, 8), (45, 384, 12), (20, 1024, 16)])
def test_matches_oracle(fp8, weighted, T, H, K):
    R = T * K + 50
    y, sf, rmap, w = case(T, H, K, R, seed=T + H + K, fp8=fp8)
    w = w if weighted else None
    out = sat.unpermute_unpad(dev(y), dev(rmap), K, None if w is None else dev(w), None if sf is None else dev(sf))
    device_status_ok()
    assert_bytes_equal(host(out), oracle.unpermute_unpad(y, rmap, K, w, y_sf=sf), f"out T={T} H={H} K={K}")


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("T,H,K", [(300, 1024, 1), (149, 1024, 2), (1000, 2048, 3), (5, 1024, 5), (777, 3072, 7),
                                   (2000, 8192, 8), (160, 7168, 4), (148, 1024, 6), (600, 3584, 8), (149, 1536, 3),
                                   (77, 512, 1), (300, 2560, 6), (1000, 512, 8), (5000, 1024, 2), (3000, 1536, 8),
                                   (2000, 3584, 5)])
def test_fp8_ring_matches_oracle(weighted, T, H, K):
    """FP8 rows with top-k <= 8 and hidden % 512 == 0 take the bulk-copy ring: fewer
    tokens than SMs, exactly one per SM, and many tokens per CTA (the stages wrap
    around many times: up to 34 tokens per CTA at 5000 tokens),
    every k, hidden up to 8192; the scale rows go in 8-byte pieces when hidden % 1024 ==
    0 and in 4-byte pieces otherwise (512, 1536, 2560, 3584)."""
    R = T * K + 50
    y, sf, rmap, w = case(T, H, K, R, seed=3 * T + H + K, fp8=True)
    w = w if weighted else None
    out = sat.unpermute_unpad(dev(y), dev(rmap), K, None if w is None else dev(w), dev(sf))
    device_status_ok()
    assert_bytes_equal(host(out), oracle.unpermute_unpad(y, rmap, K, w, y_sf=sf), f"out T={T} H={H} K={K}")


def test_moe_workload_full():
    """The MoE workload end to end on the GPU: permute+pad(128)+quantize of X, then the
    combine of (a) the FP8 rows themselves with unit weights and (b) BF16 expert outputs
    with routing weights, both against the oracle."""
    d = synthetic.moe()
    x, idx = dev(d["x"]), dev(d["topk_idx"])
    E, K = d["num_experts"], d["topk_idx"].shape[1]
    pq, psf, off, rmap = sat.permute_pad_quant(x, idx, E, 128)
    R = int(off[-1].item())
    out = sat.unpermute_unpad(pq, rmap, K, None, psf)
    device_status_ok()
    hq, hsf, hmap = host(pq)[:R], host(psf)[:R], host(rmap)
    assert_bytes_equal(host(out), oracle.unpermute_unpad(hq, hmap, K, None, y_sf=hsf), "fp8 combine")
    c = synthetic.moe_combine(rows=R, topk=K)
    out = sat.unpermute_unpad(dev(c["y"]), rmap, K, dev(c["weights"]))
    device_status_ok()
    assert_bytes_equal(host(out), oracle.unpermute_unpad(c["y"], hmap, K, c["weights"]), "bf16 combine")


def test_round_trip_k1():
    d = synthetic.moe(tokens=300, hidden=512, num_experts=7, topk=1, seed=8)
    pq, psf, off, rmap = sat.permute_pad_quant(dev(d["x"]), dev(d["topk_idx"]), 7, 16)
    out = sat.unpermute_unpad(pq, rmap, 1, None, psf)
    q, sf = oracle.quantize_rowwise(d["x"])
    dec = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64)
    v = (dec * torch.exp2(torch.from_numpy(np.repeat(sf.astype(np.float64) - 127, 128, axis=1)))).to(torch.float32)
    assert_bytes_equal(host(out), v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16), "round trip")


def test_bad_row_index_sets_device_status():
    y = torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda")
    rmap = torch.tensor([0, 1, 64, 3], dtype=torch.int32, device="cuda")
    sat.unpermute_unpad(y, rmap, 2)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE
    rmap = torch.tensor([0, -5], dtype=torch.int32, device="cuda")
    sat.unpermute_unpad(y, rmap, 2)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE
    assert sat.fp8q_last_device_status() == 0


def test_bad_row_index_sets_device_status_fp8():
    """The FP8 kernels (one per top-k up to 8, a generic one above) report a bad index too."""
    q = torch.zeros((64, 256), dtype=torch.uint8, device="cuda")
    sf = torch.full((64, 2), 127, dtype=torch.uint8, device="cuda")
    for K, bad in ((2, [0, 1, 64, 3]), (8, list(range(15)) + [-1]), (12, list(range(23)) + [99])):
        rmap = torch.tensor(bad, dtype=torch.int32, device="cuda")
        sat.unpermute_unpad(q, rmap, K, None, sf)
        assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE, K
    assert sat.fp8q_last_device_status() == 0
    # the bulk-copy ring (hidden % 1024 == 0): a bad slot is skipped and reported, the rest
    # of the token still combines
    q = torch.zeros((64, 1024), dtype=torch.uint8, device="cuda")
    sf = torch.full((64, 8), 127, dtype=torch.uint8, device="cuda")
    for K, bad in ((2, [0, 1, 64, 3]), (8, list(range(15)) + [-1])):
        rmap = torch.tensor(bad, dtype=torch.int32, device="cuda")
        sat.unpermute_unpad(q, rmap, K, None, sf)
        assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE, K
    assert sat.fp8q_last_device_status() == 0


def test_empty_is_noop():
    y = torch.zeros((16, 256), dtype=torch.bfloat16, device="cuda")
    out = sat.unpermute_unpad(y, torch.empty(0, dtype=torch.int32, device="cuda"), 4)
    assert out.shape == (0, 256)
    device_status_ok()
