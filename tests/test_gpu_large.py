"""Maximum sizes: a tensor of more than 2^31 elements (65664 x 33024), so every offset
past 2^31 bytes must be computed in 64 bits.  Quantize, direct transpose and the single
pass run on the whole tensor; sampled rows and 128x128 blocks - the last one at the
highest addresses among them - are checked against the oracle, and the single pass
against the two-kernel path byte for byte."""
import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, device_status_ok, host

pytestmark = pytest.mark.gpu

ROWS, COLS = 65664, 33024  # 2,168,487,936 elements


def test_beyond_2_31_elements():
    assert ROWS * COLS > 2 ** 31
    x = synthetic.device_normal(ROWS, COLS, seed=11, device="cuda", row_sigma=2.0)
    q, sf = sat.quantize_rowwise(x)
    qt, sft = sat.direct_transpose(q, sf)
    device_status_ok()
    nb, nj = ROWS // 128, COLS // 128
    blocks = [(0, 0), (nb - 1, nj - 1), (nb - 1, 0), (0, nj - 1), (nb // 2, nj // 2), (nb - 2, nj - 3)]
    for b, j in blocks:
        xs = host(x[128 * b:128 * b + 128, 128 * j:128 * j + 128].contiguous())
        oq, osf = oracle.quantize_rowwise(xs)
        assert_bytes_equal(host(q[128 * b:128 * b + 128, 128 * j:128 * j + 128].contiguous()), oq, f"Q block {b},{j}")
        assert_bytes_equal(host(sf[128 * b:128 * b + 128, j:j + 1].contiguous()), osf, f"SF block {b},{j}")
        oqt, osft = oracle.direct_transpose(oq, osf)
        got = host(qt[128 * j:128 * j + 128, 128 * b:128 * b + 128].contiguous())
        assert_bytes_equal(got, oqt, f"Q^T block {b},{j}")
        assert_bytes_equal(host(sft[128 * j:128 * j + 128, b:b + 1].contiguous()), osft, f"SF^T block {b},{j}")
    del qt, sft
    q2, sf2, qt2, sft2 = sat.quantize_rowwise_colwise(x)
    assert torch.equal(q2, q) and torch.equal(sf2, sf)
    del q2, sf2
    qt, sft = sat.direct_transpose(q, sf)
    assert torch.equal(qt2, qt) and torch.equal(sft2, sft)
    device_status_ok()
