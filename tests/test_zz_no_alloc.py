"""fp8q_permute_pad_quant_noalloc — permute + pad + quantize for callers that cannot
allocate device memory (their memory belongs to an allocator they cannot reach where
they route tokens, they run under a fixed memory budget, or they are a plugin handed
only its input and output buffers).  Instead of a caller-provided workspace it uses the
library's static device scratch, shared by every call.

These tests call it through the C ABI and hold its output to the CPU oracle's permute,
byte for byte, and to the allocating entry point's, over consecutive calls with
different routings; they check that a call leaves the device's free memory unchanged,
and run one routing whose scratch lies just under the array's size.

The file's name sorts last so that pytest collects it last: should it fail, a run that
stops at the first failure (-x) has already run every other test.  It depends on no
other test and passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic


def _outputs(tokens, hidden, topk, E, align):
    max_rows = sat.permute_max_rows(tokens, topk, E, align)
    q = torch.full((max_rows, hidden), 0xEE, dtype=torch.uint8, device="cuda")
    sf = torch.full((max_rows, hidden // 128), 0xEE, dtype=torch.uint8, device="cuda")
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    rmap = torch.full((tokens * topk,), -7, dtype=torch.int32, device="cuda")
    return max_rows, q, sf, off, rmap


def _call_noalloc(x, idx, E, align, outs):
    tokens, hidden = x.shape
    topk = idx.shape[1]
    max_rows, q, sf, off, rmap = outs
    return sat.lib().fp8q_permute_pad_quant_noalloc(
        x.data_ptr(), tokens, hidden, idx.data_ptr(), topk, E, align, q.data_ptr(), sf.data_ptr(), max_rows,
        off.data_ptr(), rmap.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _noalloc(x, idx, E, align):
    tokens, hidden = x.shape
    outs = _outputs(tokens, hidden, idx.shape[1], E, align)
    rc = _call_noalloc(x, idx, E, align, outs)
    assert rc == 0, sat.STATUS.get(rc, rc)
    return outs[1:]


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
    x_bits = synthetic.scaled_normal(tokens, hidden, seed=seed, row_sigma=2.0)
    idx = synthetic.zipf_topk(tokens, E, topk, rng)
    return x_bits, idx


def _host(t):
    return t.cpu().numpy()


def _check_against_oracle(got, x_bits, idx, E, align):
    """Offsets and row ids exactly; every row below offsets[E] byte for byte; the rows
    at or beyond it untouched (still the 0xEE fill)."""
    q, sf, off, rmap = got
    oq, osf, ooff, ormap = oracle.permute_pad_quant(x_bits, idx, E, align)
    np.testing.assert_array_equal(_host(off), ooff)
    np.testing.assert_array_equal(_host(rmap), ormap)
    n = int(ooff[-1])
    assert n > 0
    np.testing.assert_array_equal(_host(sf)[:n], osf[:n])
    np.testing.assert_array_equal(_host(q)[:n], oq[:n])
    assert bool((q[n:] == 0xEE).all()) and bool((sf[n:] == 0xEE).all())


@pytest.mark.gpu
def test_noalloc_matches_oracle_and_workspace_entry_point_on_consecutive_calls():
    cases = [((2048, 1024, 32, 8, 1), 128), ((1500, 512, 8, 2, 2), 16), ((2048, 1024, 32, 8, 1), 128)]
    for (tokens, hidden, E, topk, seed), align in cases:
        x_bits, idx_np = _case(tokens, hidden, E, topk, seed)
        x = synthetic.to_torch_bf16(x_bits).cuda()
        idx = torch.from_numpy(idx_np).cuda()
        got = _noalloc(x, idx, E, align)
        want = _with_workspace(x, idx, E, align)
        torch.cuda.synchronize()
        assert sat.fp8q_last_device_status() == 0
        _check_against_oracle(got, x_bits, idx_np, E, align)
        for a, b in zip(got, want):
            assert torch.equal(a, b)


@pytest.mark.gpu
def test_noalloc_call_allocates_no_device_memory():
    """After a first call (which may load the library's device code and its static
    array), a call changes neither torch's allocator nor the device's free memory."""
    x_bits, idx_np = _case(4096, 512, 64, 4, 7)
    x = synthetic.to_torch_bf16(x_bits).cuda()
    idx = torch.from_numpy(idx_np).cuda()
    outs = _outputs(4096, 512, 4, 64, 16)
    assert _call_noalloc(x, idx, 64, 16, outs) == 0
    torch.cuda.synchronize()
    free0, used0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        assert _call_noalloc(x, idx, 64, 16, outs) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == used0
    assert sat.fp8q_last_device_status() == 0
    _check_against_oracle(outs[1:], x_bits, idx_np, 64, 16)


@pytest.mark.gpu
def test_noalloc_routing_just_under_the_scratch_size():
    """256 experts, top-8: 262016 tokens need 4,193,296 bytes of routing scratch (the
    array holds 4,194,304) and are accepted; one token more is refused with ARG."""
    tokens, hidden, E, topk = 262016, 128, 256, 8
    assert sat.fp8q_permute_workspace_bytes(tokens, topk, E) <= sat.NOALLOC_SCRATCH_BYTES
    assert sat.fp8q_permute_workspace_bytes(tokens + 1, topk, E) > sat.NOALLOC_SCRATCH_BYTES
    x_bits, idx_np = _case(tokens, hidden, E, topk, 11)
    x = synthetic.to_torch_bf16(x_bits).cuda()
    idx = torch.from_numpy(idx_np).cuda()
    got = _noalloc(x, idx, E, 16)
    torch.cuda.synchronize()
    assert sat.fp8q_last_device_status() == 0
    _check_against_oracle(got, x_bits, idx_np, E, 16)
    x1 = torch.zeros((tokens + 1, hidden), dtype=torch.bfloat16, device="cuda")
    i1 = torch.zeros((tokens + 1, topk), dtype=torch.int32, device="cuda")
    assert _call_noalloc(x1, i1, E, 16, _outputs(tokens + 1, hidden, topk, E, 16)) == sat.FP8Q_ERR_ARG


def test_noalloc_rejects_routing_beyond_its_scratch():
    """2^24 tokens x 8 slots x 4096 experts needs far more than the static scratch: the
    call fails with FP8Q_ERR_ARG before any CUDA call (so this runs without a GPU)."""
    assert sat.fp8q_permute_workspace_bytes(1 << 24, 8, 4096) > sat.NOALLOC_SCRATCH_BYTES
    A = 0x10000
    rc = sat.lib().fp8q_permute_pad_quant_noalloc(A, 1 << 24, 256, A, 8, 4096, 16, A, A, (1 << 27) + 4096 * 15,
                                                  A, A, None)
    assert rc == sat.FP8Q_ERR_ARG


def test_noalloc_rejects_token_counts_whose_slots_overflow():
    """tokens * topk beyond int32 (here 2^58 x 64, which also wraps int64) is refused
    with FP8Q_ERR_SHAPE before anything multiplies it, by both permute entry points."""
    A = 0x10000
    big = 1 << 58
    L = sat.lib()
    assert L.fp8q_permute_pad_quant_noalloc(A, big, 256, A, 64, 256, 16, A, A, (1 << 31) - 1, A, A,
                                            None) == sat.FP8Q_ERR_SHAPE
    assert L.fp8q_permute_pad_quant(A, big, 256, A, 64, 256, 16, A, A, (1 << 31) - 1, A, A, A, 1 << 40,
                                    None) == sat.FP8Q_ERR_SHAPE
    assert sat.fp8q_permute_workspace_bytes(big, 64, 256) == 0
