"""Stream order across dependent launches, checked where it could break.

Every kernel is a programmatic dependent launch: its blocks may be placed on the GPU
while the previous kernel in the stream still runs, and it waits for that kernel before
touching memory.  These tests run producer and consumer calls back to back on one stream
with two different inputs alternating through the SAME intermediate buffers and no
synchronisation, then compare every final output with the oracle.  A consumer that read
its input before the producer had finished, or a producer that overwrote an intermediate
the previous consumer was still reading, would show up as the other input's bytes.
"""
import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, dev, device_status_ok, host

pytestmark = pytest.mark.gpu

REPS = 8


def _u8(*shape):
    return torch.empty(shape, dtype=torch.uint8, device="cuda")


def test_quantize_then_direct_transpose_alternating_inputs():
    R, C = 2048, 3072
    xs = [synthetic.scaled_normal(R, C, seed=s, row_sigma=1.5) for s in (11, 12)]
    X = [dev(x) for x in xs]
    q, sf = _u8(R, C), _u8(R, C // 128)  # shared by both inputs
    outs = [(_u8(C, R), _u8(C, R // 128)) for _ in xs]
    for _ in range(REPS):
        for i in range(2):
            sat.fp8q_quantize_rowwise(X[i], R, C, q, sf)
            sat.fp8q_direct_transpose(q, sf, R, C, None, 1, outs[i][0], outs[i][1])
    device_status_ok()
    for i, x in enumerate(xs):
        oqt, osft = oracle.direct_transpose(*oracle.quantize_rowwise(x))
        assert_bytes_equal(host(outs[i][0]), oqt, f"input {i} Q^T")
        assert_bytes_equal(host(outs[i][1]), osft, f"input {i} SF^T")


def test_mx32_quantize_then_transpose_alternating_inputs():
    R, C = 1024, 2048
    xs = [synthetic.scaled_normal(R, C, seed=s, row_sigma=2.0) for s in (21, 22)]
    X = [dev(x) for x in xs]
    q, sf = _u8(R, C), _u8(R, C // 32)
    outs = [(_u8(C, R), _u8(C, R // 32)) for _ in xs]
    for _ in range(REPS):
        for i in range(2):
            sat.fp8q_quantize_rowwise_mx32(X[i], R, C, q, sf)
            sat.fp8q_direct_transpose_mx32(q, sf, R, C, outs[i][0], outs[i][1])
    device_status_ok()
    for i, x in enumerate(xs):
        oqt, osft = oracle.direct_transpose_g(*oracle.quantize_rowwise_g(x, 32), 32)
        assert_bytes_equal(host(outs[i][0]), oqt, f"input {i} MX Q^T")
        assert_bytes_equal(host(outs[i][1]), osft, f"input {i} MX SF^T")


def test_permute_grouped_transpose_combine_alternating_routings():
    """permute+pad+quantize -> grouped direct transpose -> FP8 unpermute (combine), two
    token sets with different routings sharing the permuted buffers, offsets, row ids and
    routing workspace."""
    T, H, E, K, align = 2048, 1024, 16, 4, 128
    rng = np.random.default_rng(5)
    xs = [synthetic.scaled_normal(T, H, seed=s) for s in (31, 32)]
    idxs = [synthetic.zipf_topk(T, E, K, rng) for _ in xs]
    X, IDX = [dev(x) for x in xs], [dev(i) for i in idxs]
    R = sat.permute_max_rows(T, K, E, align)
    q, sf = _u8(R, H), _u8(R, H // 128)
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rmap = torch.empty(T * K, dtype=torch.int32, device="cuda")
    ws = _u8(sat.fp8q_permute_workspace_bytes(T, K, E))
    outs = [(_u8(R * H), _u8(R * H // 128), torch.empty((T, H), dtype=torch.bfloat16, device="cuda")) for _ in xs]
    for _ in range(REPS):
        for i in range(2):
            sat.fp8q_permute_pad_quant(X[i], T, H, IDX[i], K, E, align, q, sf, R, offs, rmap, ws, ws.numel())
            sat.fp8q_direct_transpose(q, sf, R, H, offs, E, outs[i][0], outs[i][1])
            sat.fp8q_unpermute_unpad(q, sf, R, H, rmap, None, T, K, outs[i][2])
    device_status_ok()
    for i in range(2):
        oq, osf, ooff, ormap = oracle.permute_pad_quant(xs[i], idxs[i], E, align)
        n = int(ooff[-1])
        oqt, osft = oracle.direct_transpose(oq[:n], osf[:n], ooff)
        assert_bytes_equal(host(outs[i][0])[:n * H], oqt.reshape(-1)[:n * H], f"routing {i} grouped Q^T")
        assert_bytes_equal(host(outs[i][1])[:n * H // 128], osft.reshape(-1)[:n * H // 128], f"routing {i} grouped SF^T")
        want = oracle.unpermute_unpad(oq[:n], ormap, K, y_sf=osf[:n])
        assert_bytes_equal(host(outs[i][2]), want, f"routing {i} combine")
