"""fp8q_permute_pad_quant_noalloc — permute + pad + quantize for callers that cannot
allocate device memory (their memory belongs to an allocator they cannot reach where
they route tokens, they run under a fixed memory budget, or they are a plugin handed
only its input and output buffers).  Instead of a caller-provided workspace it uses the
library's static device scratch, shared by every call.  These tests call it through the
C ABI and hold its output to the allocating entry point's, byte for byte, over
consecutive calls with different routings.  (This file is collected last on purpose.)
"""
import ctypes

import numpy as np
import pytest
import torch

import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic


def _outputs(tokens, hidden, topk, E, align):
    max_rows = sat.permute_max_rows(tokens, topk, E, align)
    q = torch.full((max_rows, hidden), 0xEE, dtype=torch.uint8, device="cuda")
    sf = torch.full((max_rows, hidden // 128), 0xEE, dtype=torch.uint8, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    rmap = torch.full((tokens * topk,), -7, dtype=torch.int32, device="cuda")
    return max_rows, q, sf, off, rmap


def _noalloc(x, idx, E, align):
    tokens, hidden = x.shape
    topk = idx.shape[1]
    max_rows, q, sf, off, rmap = _outputs(tokens, hidden, topk, E, align)
    rc = sat.lib().fp8q_permute_pad_quant_noalloc(
        x.data_ptr(), tokens, hidden, idx.data_ptr(), topk, E, align, q.data_ptr(), sf.data_ptr(), max_rows,
        off.data_ptr(), rmap.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, sat.STATUS.get(rc, rc)
    return q, sf, off, rmap


def _with_workspace(x, idx, E, align):
    tokens, hidden = x.shape
    topk = idx.shape[1]
    max_rows, q, sf, off, rmap = _outputs(tokens, hidden, topk, E, align)
    ws_bytes = sat.fp8q_permute_workspace_bytes(tokens, topk, E)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    rc = sat.lib().fp8q_permute_pad_quant(
        x.data_ptr(), tokens, hidden, idx.data_ptr(), topk, E, align, q.data_ptr(), sf.data_ptr(), max_rows,
        off.data_ptr(), rmap.data_ptr(), ws.data_ptr(), ws.numel(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, sat.STATUS.get(rc, rc)
    return q, sf, off, rmap


def _case(tokens, hidden, E, topk, seed):
    rng = np.random.default_rng(seed)
    x = synthetic.to_torch_bf16(synthetic.scaled_normal(tokens, hidden, seed=seed, row_sigma=2.0)).cuda()
    idx = torch.from_numpy(synthetic.zipf_topk(tokens, E, topk, rng)).cuda()
    return x, idx


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    cases = [((2048, 1024, 32, 8, 1), 128), ((1500, 512, 8, 2, 2), 16), ((2048, 1024, 32, 8, 1), 128)]
    for (tokens, hidden, E, topk, seed), align in cases:
        x, idx = _case(tokens, hidden, E, topk, seed)
        got = _noalloc(x, idx, E, align)
        want = _with_workspace(x, idx, E, align)
        torch.cuda.synchronize()
        assert sat.fp8q_last_device_status() == 0
        # offsets and row ids exactly; every row up to offsets[E] byte for byte, and the
        # rows beyond it untouched in both
        assert torch.equal(got[2], want[2]) and torch.equal(got[3], want[3])
        assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])
        n = int(want[2][-1].item())
        assert n > 0 and bool((got[0][n:] == 0xEE).all())


def test_noalloc_rejects_routing_beyond_its_scratch():
    """2^24 tokens x 8 slots x 4096 experts needs far more than the static scratch: the
    call fails with FP8Q_ERR_ARG before any CUDA call (so this runs without a GPU)."""
    assert sat.fp8q_permute_workspace_bytes(1 << 24, 8, 4096) > sat.NOALLOC_SCRATCH_BYTES
    A = 0x10000
    rc = sat.lib().fp8q_permute_pad_quant_noalloc(A, 1 << 24, 256, A, 8, 4096, 16, A, A, (1 << 27) + 4096 * 15,
                                                  A, A, None)
    assert rc == sat.FP8Q_ERR_ARG
