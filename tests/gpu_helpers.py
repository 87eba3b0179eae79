"""Shared helpers for the GPU parity tests: move seeded numpy inputs to the device and
bring results back as numpy bytes."""
import numpy as np
import torch

import scaling_aware_transpose_b200 as sat


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy -> CUDA tensor with the same bytes (uint16 is carried as bf16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_bytes_equal(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got).reshape(want.shape)
    if np.array_equal(got, want):
        return
    bad = np.argwhere(got != want)
    first = [tuple(int(i) for i in b) for b in bad[:5]]
    vals = [(hex(int(got[tuple(b)])), hex(int(want[tuple(b)]))) for b in bad[:5]]
    raise AssertionError(f"{what}: {len(bad)} of {want.size} bytes differ; first at {first}: got/want {vals}")


def device_status_ok():
    st = sat.fp8q_last_device_status()
    assert st == 0, f"device status {sat.STATUS.get(st, st)}"
