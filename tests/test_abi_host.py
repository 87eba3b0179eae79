"""CPU-only checks of the C ABI: the library loads, exports every entry point the header
declares, and rejects bad arguments on the host before any CUDA call (no GPU needed:
the checks run before the library asks for a device)."""
import ctypes
import os
import re

import pytest

import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")
A = 0x10000   # a fake, 16-byte aligned "device" address; never dereferenced on these paths
MIS = 0x10008  # misaligned


@pytest.fixture(scope="module")
def L():
    lib_build.build()
    return sat.lib()


def declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8q_\w+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fp8q_quantize_rowwise", "fp8q_direct_transpose", "fp8q_naive_transpose", "fp8q_swiglu_quant",
              "fp8q_permute_pad_quant", "fp8q_last_device_status", "fp8q_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings_and_version(L):
    for code in range(8):
        assert sat.lib().fp8q_status_string(code)
    assert sat.fp8q_version() >= 10000


def test_quantize_host_errors(L):
    f = L.fp8q_quantize_rowwise
    assert f(A, 4, 100, A, A, None) == sat.FP8Q_ERR_SHAPE
    assert f(A, -1, 128, A, A, None) == sat.FP8Q_ERR_SHAPE
    assert f(None, 0, 128, None, None, None) == sat.FP8Q_OK          # empty: no-op
    assert f(None, 4, 128, A, A, None) == sat.FP8Q_ERR_NULL
    assert f(MIS, 4, 128, A, A, None) == sat.FP8Q_ERR_ALIGN
    assert f(A, 4, 128, MIS, A, None) == sat.FP8Q_ERR_ALIGN


@pytest.mark.parametrize("name", ["fp8q_direct_transpose", "fp8q_naive_transpose"])
def test_transpose_host_errors(L, name):
    fn = getattr(L, name)
    extra = (A, 1 << 30) if "naive" in name else ()

    def call(q, sf, rows, cols, off, G, qt, sft, *ex):
        return fn(q, sf, rows, cols, off, G, qt, sft, *(ex or extra), None)

    assert call(A, A, 100, 256, None, 1, A, A) == sat.FP8Q_ERR_SHAPE      # dense rows % 128
    assert call(A, A, 256, 200, None, 1, A, A) == sat.FP8Q_ERR_SHAPE      # cols % 128
    assert call(A, A, 256, 256, None, 2, A, A) == sat.FP8Q_ERR_ARG        # groups without offsets
    assert call(A, A, 256, 256, A, 0, A, A) == sat.FP8Q_ERR_ARG           # zero groups
    assert call(A, A, 256, 256, None, 1, None, A) == sat.FP8Q_ERR_NULL
    assert call(MIS, A, 256, 256, None, 1, A, A) == sat.FP8Q_ERR_ALIGN
    assert call(A, A, 256, 256, A + 2, 3, A, A) == sat.FP8Q_ERR_ALIGN     # offsets not int32-aligned
    assert call(A, A, 0, 256, None, 1, A, A) == sat.FP8Q_OK               # empty: no-op
    assert call(A, A, 1 << 31, 128, A, 1, A, A) == sat.FP8Q_ERR_SHAPE     # beyond int32 coordinates
    if "naive" in name:
        assert call(A, A, 256, 256, None, 1, A, A, A, 100) == sat.FP8Q_ERR_ARG    # workspace too small
        assert call(A, A, 256, 256, None, 1, A, A, None, 1 << 30) == sat.FP8Q_ERR_NULL
        assert call(A, A, 256, 256, None, 1, A, A, MIS, 1 << 30) == sat.FP8Q_ERR_ALIGN


def test_workspace_sizes(L):
    assert sat.fp8q_naive_workspace_bytes(8192, 7168) == 4 * 8192 * 7168
    assert sat.fp8q_naive_workspace_bytes(0, 128) == 0
    ws = sat.fp8q_permute_workspace_bytes(16384, 8, 32)
    assert ws >= 4 * (2 * 128 * 32 + 32)


def test_swiglu_host_errors(L):
    f = L.fp8q_swiglu_quant
    assert f(A, A, 256, 100, A, A, A, A, None) == sat.FP8Q_ERR_SHAPE
    assert f(A, A, 256, 256, A, A, A, None, None) == sat.FP8Q_ERR_ARG       # qt without sft
    assert f(A, A, 100, 256, A, A, A, A, None) == sat.FP8Q_ERR_SHAPE        # transposed needs rows % 128
    assert f(None, A, 256, 256, A, A, None, None, None) == sat.FP8Q_ERR_NULL
    assert f(A, MIS, 256, 256, A, A, None, None, None) == sat.FP8Q_ERR_ALIGN
    assert f(None, None, 0, 256, None, None, None, None, None) == sat.FP8Q_OK


def test_rowwise_colwise_host_errors(L):
    f = L.fp8q_quantize_rowwise_colwise
    Z, P = sat.ZERO_TILE_MIN_SCALE, sat.SF_PACKED_UE8M0
    assert f(A, 256, 100, 0, A, A, A, A, None) == sat.FP8Q_ERR_SHAPE        # cols % 128
    assert f(A, 100, 256, 0, A, A, A, A, None) == sat.FP8Q_ERR_SHAPE        # column-wise needs rows % 128
    assert f(A, 256, 256, 4, A, A, A, A, None) == sat.FP8Q_ERR_ARG          # unknown flag bit
    assert f(A, 256, 256, 0, A, A, A, None, None) == sat.FP8Q_ERR_ARG       # qt without sft
    assert f(A, 256, 256, 0, A, A, None, A, None) == sat.FP8Q_ERR_ARG       # sft without qt
    assert f(None, 256, 256, 0, A, A, None, None, None) == sat.FP8Q_ERR_NULL
    assert f(A, 256, 256, 0, A, None, A, A, None) == sat.FP8Q_ERR_NULL
    assert f(MIS, 256, 256, Z, A, A, A, A, None) == sat.FP8Q_ERR_ALIGN
    assert f(A, 256, 256, 0, A, A, MIS, A, None) == sat.FP8Q_ERR_ALIGN      # qt must be 16-byte aligned
    assert f(A, 256, 256, P, A, A + 2, A, A, None) == sat.FP8Q_ERR_ALIGN    # packed words: 4-byte aligned
    assert f(A, 256, 256, P, A, A, A, A + 1, None) == sat.FP8Q_ERR_ALIGN
    assert f(None, 0, 256, Z | P, None, None, None, None, None) == sat.FP8Q_OK  # empty: no-op
    assert f(A, 1 << 31, 128, 0, A, A, None, None, None) == sat.FP8Q_ERR_SHAPE


def test_packed_sf_bytes(L):
    assert sat.fp8q_packed_sf_bytes(8192, 7168) == 4 * 14 * 8192
    assert sat.fp8q_packed_sf_bytes(7168, 8192) == 4 * 16 * 7168
    assert sat.fp8q_packed_sf_bytes(3, 640) == 4 * 2 * 4      # K tiles 5 -> 2 words; mn 3 -> 4
    assert sat.fp8q_packed_sf_bytes(0, 128) == 0
    assert sat.packed_sf_shape(3, 640) == (2, 4)


def test_unpermute_host_errors(L):
    f = L.fp8q_unpermute_unpad

    def call(y=A, sf=None, rows=64, hidden=256, rmap=A, w=A, tokens=16, topk=2, out=A):
        return f(y, sf, rows, hidden, rmap, w, tokens, topk, out, None)

    assert call(hidden=200) == sat.FP8Q_ERR_SHAPE
    assert call(rows=-1) == sat.FP8Q_ERR_SHAPE
    assert call(topk=0) == sat.FP8Q_ERR_ARG
    assert call(topk=65) == sat.FP8Q_ERR_ARG
    assert call(y=None) == sat.FP8Q_ERR_NULL
    assert call(rmap=None) == sat.FP8Q_ERR_NULL
    assert call(out=None) == sat.FP8Q_ERR_NULL
    assert call(y=MIS) == sat.FP8Q_ERR_ALIGN
    assert call(out=MIS) == sat.FP8Q_ERR_ALIGN
    assert call(rmap=A + 2) == sat.FP8Q_ERR_ALIGN
    assert call(w=A + 1) == sat.FP8Q_ERR_ALIGN
    assert call(y=None, rmap=None, out=None, tokens=0) == sat.FP8Q_OK   # empty: no-op


def test_mx32_host_errors(L):
    fq, fd = L.fp8q_quantize_rowwise_mx32, L.fp8q_direct_transpose_mx32
    assert fq(A, 4, 48, A, A, None) == sat.FP8Q_ERR_SHAPE          # cols % 32
    assert fq(None, 4, 64, A, A, None) == sat.FP8Q_ERR_NULL
    assert fq(MIS, 4, 64, A, A, None) == sat.FP8Q_ERR_ALIGN
    assert fq(None, 0, 64, None, None, None) == sat.FP8Q_OK        # empty: no-op
    assert fd(A, A, 96, 128, A, A, None) == sat.FP8Q_ERR_SHAPE     # rows % 128 (this build's kernel)
    assert fd(A, A, 128, 160, A, A, None) == sat.FP8Q_ERR_SHAPE
    assert fd(A, A, 128, 128, None, A, None) == sat.FP8Q_ERR_NULL
    assert fd(A, A, 128, 128, MIS, A, None) == sat.FP8Q_ERR_ALIGN
    assert fd(A, A + 2, 128, 128, A, A, None) == sat.FP8Q_ERR_ALIGN      # scale words
    assert fd(A, A, 128, 128, A, A + 1, None) == sat.FP8Q_ERR_ALIGN
    assert fd(None, None, 0, 128, None, None, None) == sat.FP8Q_OK


def test_debug_hook_host_errors(L):
    assert L.fp8q_debug_e4m3_encode_range(0xFFFFFFF0, 32, A, None) == sat.FP8Q_ERR_ARG   # past 2^32
    assert L.fp8q_debug_e4m3_encode_range(0, 16, None, None) == sat.FP8Q_ERR_NULL
    assert L.fp8q_debug_exp_spec_range(0, 16, A + 2, None) == sat.FP8Q_ERR_ALIGN
    assert L.fp8q_debug_exp_spec_range(0, -1, A, None) == sat.FP8Q_ERR_ARG
    assert L.fp8q_debug_swiglu_spec(A, None, 16, A, None) == sat.FP8Q_ERR_NULL
    assert L.fp8q_debug_swiglu_spec(A, A, 16, A + 1, None) == sat.FP8Q_ERR_ALIGN
    assert L.fp8q_debug_swiglu_spec(None, None, 0, None, None) == sat.FP8Q_OK
    assert L.fp8q_debug_silu_bf16(A, 15, A, None) == sat.FP8Q_ERR_ARG      # n odd
    assert L.fp8q_debug_silu_bf16(A, -2, A, None) == sat.FP8Q_ERR_ARG
    assert L.fp8q_debug_silu_bf16(None, 16, A, None) == sat.FP8Q_ERR_NULL
    assert L.fp8q_debug_silu_bf16(A + 2, 16, A, None) == sat.FP8Q_ERR_ALIGN  # gate words
    assert L.fp8q_debug_silu_bf16(A, 16, A + 4, None) == sat.FP8Q_ERR_ALIGN  # float pairs
    assert L.fp8q_debug_silu_bf16(None, 0, None, None) == sat.FP8Q_OK


def test_permute_host_errors(L):
    f = L.fp8q_permute_pad_quant

    def call(tokens=16, hidden=256, topk=2, E=4, align=16, max_rows=None, ws=1 << 20, **kw):
        if max_rows is None:
            max_rows = tokens * topk + E * (align - 1)
        p = dict(x=A, idx=A, q=A, sf=A, off=A, rmap=A, wsp=A)
        p.update(kw)
        return f(p["x"], tokens, hidden, p["idx"], topk, E, align, p["q"], p["sf"], max_rows, p["off"], p["rmap"],
                 p["wsp"], ws, None)

    assert call(hidden=100) == sat.FP8Q_ERR_SHAPE
    assert call(topk=0) == sat.FP8Q_ERR_ARG
    assert call(topk=65) == sat.FP8Q_ERR_ARG
    assert call(E=5000) == sat.FP8Q_ERR_ARG
    assert call(align=0) == sat.FP8Q_ERR_ARG
    assert call(max_rows=10) == sat.FP8Q_ERR_ARG
    assert call(ws=4) == sat.FP8Q_ERR_ARG
    assert call(off=None) == sat.FP8Q_ERR_NULL
    assert call(idx=None) == sat.FP8Q_ERR_NULL
    assert call(x=None) == sat.FP8Q_ERR_NULL
    assert call(x=MIS) == sat.FP8Q_ERR_ALIGN
    assert call(rmap=A + 2) == sat.FP8Q_ERR_ALIGN


def test_permute_fp8_host_errors(L):
    f = L.fp8q_permute_pad_fp8

    def call(tokens=16, hidden=256, topk=2, E=4, align=16, max_rows=None, ws=1 << 20, **kw):
        if max_rows is None:
            max_rows = tokens * topk + E * (align - 1)
        p = dict(xq=A, xsf=A, idx=A, q=A, sf=A, off=A, rmap=A, wsp=A)
        p.update(kw)
        return f(p["xq"], p["xsf"], tokens, hidden, p["idx"], topk, E, align, p["q"], p["sf"], max_rows, p["off"],
                 p["rmap"], p["wsp"], ws, None)

    assert call(hidden=100) == sat.FP8Q_ERR_SHAPE
    assert call(topk=0) == sat.FP8Q_ERR_ARG
    assert call(max_rows=10) == sat.FP8Q_ERR_ARG
    assert call(ws=4) == sat.FP8Q_ERR_ARG
    assert call(xq=None) == sat.FP8Q_ERR_NULL
    assert call(xsf=None) == sat.FP8Q_ERR_NULL
    assert call(off=None) == sat.FP8Q_ERR_NULL
    assert call(xq=MIS) == sat.FP8Q_ERR_ALIGN
    assert call(q=MIS) == sat.FP8Q_ERR_ALIGN


def test_binding_rejects_host_tensors():
    import torch
    x = torch.zeros((4, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sat.fp8q_quantize_rowwise(x, 4, 128, x, x, 0)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(sat, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(sat, "_lib", None)
    with pytest.raises(RuntimeError, match="libfp8q.so is missing"):
        sat.lib()


def test_no_oracle_in_product_package():
    pkg = os.path.join(ROOT, "scaling_aware_transpose_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, fn), encoding="utf-8").read()
                assert "import oracle" not in txt and "from oracle" not in txt and "fp8q_oracle" not in txt, fn
