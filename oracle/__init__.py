"""CPU oracle for the FP8 quantize / scaling-aware direct transpose path.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``scaling_aware_transpose_b200``) never imports, links or calls it, and it shares no
code with it: the C source here is an independent, plain restatement of the method's
definitions (see the header of ``fp8q_oracle.c`` for the passages each function
follows).

Arrays are numpy: bf16 tensors travel as ``uint16`` bit patterns, FP8 codes and UE8M0
scale bytes as ``uint8``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _declare(L):
    V, I64, I32, D, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_float
    L.orc_e4m3_encode.argtypes, L.orc_e4m3_encode.restype = [D], ctypes.c_uint8
    L.orc_e4m3_decode.argtypes, L.orc_e4m3_decode.restype = [ctypes.c_uint8], D
    L.orc_scale_exponent.argtypes, L.orc_scale_exponent.restype = [D], ctypes.c_int
    L.orc_shift_code_value.argtypes = [ctypes.c_uint8, ctypes.c_int]
    L.orc_shift_code_value.restype = ctypes.c_uint8
    L.orc_shift_code_bytes.argtypes = [ctypes.c_uint8, ctypes.c_int]
    L.orc_shift_code_bytes.restype = ctypes.c_uint8
    for name, args in {
        "orc_e4m3_encode_array": [V, I64, V],
        "orc_e4m3_decode_array": [V, I64, V],
        "orc_scale_exponent_array": [V, I64, V],
        "orc_shift_codes": [V, I64, ctypes.c_int, ctypes.c_int, V],
        "orc_quantize_rowwise": [V, I64, I64, V, V],
        "orc_quantize_rowwise_f32": [V, I64, I64, V, V],
        "orc_exp_spec_constants": [V],
        "orc_exp_spec_array": [V, I64, V],
        "orc_swiglu_array": [V, V, I64, V],
        "orc_pack_ue8m0": [V, I64, I64, V],
        "orc_quantize_rowwise_opt": [V, I64, I64, ctypes.c_int, V, V],
    }.items():
        fn = getattr(L, name)
        fn.argtypes, fn.restype = args, None
    for name, args in {
        "orc_direct_transpose": [V, V, I64, I64, V, I32, V, V],
        "orc_naive_transpose": [V, V, I64, I64, V, I32, V, V],
        "orc_swiglu_quant": [V, V, I64, I64, V, V, V, V],
        "orc_permute_pad_quant": [V, I64, I64, V, I32, I32, I32, V, V, I64, V, V],
        "orc_quantize_rowwise_colwise": [V, I64, I64, ctypes.c_uint32, V, V, V, V],
        "orc_unpermute_unpad": [V, V, I64, I64, V, V, I64, I32, V],
        "orc_permute_pad_fp8": [V, V, I64, I64, V, I32, I32, I32, V, V, I64, V, V],
        "orc_quantize_rowwise_g": [V, I64, I64, I32, V, V],
        "orc_e4m3_encode_f32_range": [ctypes.c_uint32, I64, V],
        "orc_exp_spec_f32_range": [ctypes.c_uint32, I64, V],
        "orc_direct_transpose_g": [V, V, I64, I64, I32, V, V],
        "orc_ep_dispatch_pack": [V, V, I64, I64, V, I32, I32, I32, V, V, V, I64, V, V],
        "orc_ep_recv_permute": [V, V, V, I64, I64, I32, I32, I32, V, V, I64, V, V],
    }.items():
        fn = getattr(L, name)
        fn.argtypes, fn.restype = args, ctypes.c_int
    L.orc_exp_spec.argtypes, L.orc_exp_spec.restype = [F], F
    L.orc_num_threads.argtypes, L.orc_num_threads.restype = [], ctypes.c_int
    L.orc_set_num_threads.argtypes, L.orc_set_num_threads.restype = [ctypes.c_int], None


class OracleError(RuntimeError):
    pass


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- codec
def e4m3_encode(y) -> np.ndarray:
    y = _c(y, np.float64)
    out = np.empty(y.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(y), y.size, _p(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode_array(_p(c), c.size, _p(out))
    return out


def scale_exponent(amax) -> np.ndarray:
    a = _c(amax, np.float64)
    out = np.empty(a.shape, np.int32)
    lib().orc_scale_exponent_array(_p(a), a.size, _p(out))
    return out


def shift_codes(codes, k: int, rule: str = "value") -> np.ndarray:
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.uint8)
    lib().orc_shift_codes(_p(c), c.size, int(k), 1 if rule == "bytes" else 0, _p(out))
    return out


# ---------------------------------------------------------------- path steps
def quantize_rowwise(x_bf16_bits):
    x = _c(x_bf16_bits, np.uint16)
    rows, cols = x.shape
    if cols % 128:
        raise OracleError("cols must be a multiple of 128")
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // 128), np.uint8)
    lib().orc_quantize_rowwise(_p(x), rows, cols, _p(q), _p(sf))
    return q, sf


def quantize_rowwise_f32(y):
    y = _c(y, np.float32)
    rows, cols = y.shape
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // 128), np.uint8)
    lib().orc_quantize_rowwise_f32(_p(y), rows, cols, _p(q), _p(sf))
    return q, sf


ZERO_TILE_MIN_SCALE = 1  # flags of the single-pass quantizer (same meaning as the library's)
SF_PACKED_UE8M0 = 2


def packed_sf_shape(mn: int, ktiles: int) -> tuple[int, int]:
    """Shape (words) of the packed UE8M0 scales of an operand with mn rows and ktiles
    1x128 tiles along K."""
    return ((ktiles + 3) // 4, (mn + 3) // 4 * 4)


def pack_ue8m0(sf):
    """Unpacked scale bytes [mn, ktiles] -> packed words [ceil(ktiles/4), mn_pad] (uint32)."""
    sf = _c(sf, np.uint8)
    mn, kt = sf.shape
    out = np.empty(packed_sf_shape(mn, kt), np.uint32)
    lib().orc_pack_ue8m0(_p(sf), mn, kt, _p(out))
    return out


def quantize_rowwise_opt(x_bf16_bits, zero_tile_min: bool):
    x = _c(x_bf16_bits, np.uint16)
    rows, cols = x.shape
    if cols % 128:
        raise OracleError("cols must be a multiple of 128")
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // 128), np.uint8)
    lib().orc_quantize_rowwise_opt(_p(x), rows, cols, 1 if zero_tile_min else 0, _p(q), _p(sf))
    return q, sf


def quantize_rowwise_colwise(x_bf16_bits, flags: int = 0, colwise: bool = True):
    """Single-pass quantizer's definition: (Q, SF, Q^T, SF^T); Q^T/SF^T are None when
    colwise is False.  With SF_PACKED_UE8M0 the scales are packed uint32 words."""
    x = _c(x_bf16_bits, np.uint16)
    rows, cols = x.shape
    packed = bool(flags & SF_PACKED_UE8M0)
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty(packed_sf_shape(rows, cols // 128), np.uint32) if packed else np.empty((rows, cols // 128), np.uint8)
    qt = sft = None
    if colwise:
        qt = np.empty((cols, rows), np.uint8)
        sft = (np.empty(packed_sf_shape(cols, rows // 128), np.uint32) if packed
               else np.empty((cols, rows // 128), np.uint8))
    rc = lib().orc_quantize_rowwise_colwise(_p(x), rows, cols, int(flags), _p(q), _p(sf), _p(qt), _p(sft))
    if rc:
        raise OracleError(f"oracle single-pass quantizer rejected its arguments (code {rc})")
    return q, sf, qt, sft


def quantize_rowwise_g(x_bf16_bits, tile: int):
    """Row-wise quantization with 1 x tile scaling tiles (tile = 128, or 32 for MX)."""
    x = _c(x_bf16_bits, np.uint16)
    rows, cols = x.shape
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // tile), np.uint8)
    if lib().orc_quantize_rowwise_g(_p(x), rows, cols, tile, _p(q), _p(sf)):
        raise OracleError("cols must be a multiple of the tile")
    return q, sf


def direct_transpose_g(q, sf, tile: int):
    """Direct transpose with tile x tile blocks: (Q^T [cols, rows], SF^T [cols, rows/tile])."""
    q = _c(q, np.uint8)
    sf = _c(sf, np.uint8)
    rows, cols = q.shape
    qt = np.empty((cols, rows), np.uint8)
    sft = np.empty((cols, rows // tile), np.uint8)
    if lib().orc_direct_transpose_g(_p(q), _p(sf), rows, cols, tile, _p(qt), _p(sft)):
        raise OracleError("rows and cols must be multiples of the tile")
    return qt, sft


def _transpose_common(fn, q, sf, offsets):
    q = _c(q, np.uint8)
    sf = _c(sf, np.uint8)
    rows, cols = q.shape
    off = None if offsets is None else _c(offsets, np.int32)
    G = 1 if off is None else off.size - 1
    qt = np.zeros(rows * cols, np.uint8)
    sft = np.zeros(rows * cols // 128, np.uint8)
    rc = fn(_p(q), _p(sf), rows, cols, _p(off), G, _p(qt), _p(sft))
    if rc:
        raise OracleError(f"oracle transpose rejected its arguments (code {rc})")
    if off is None:
        return qt.reshape(cols, rows), sft.reshape(cols, rows // 128)
    return qt, sft  # flat: group g at cols*off[g], shape [cols, M_g]


def direct_transpose(q, sf, offsets=None):
    """Dense: returns (Q^T [cols, rows], SF^T [cols, rows/128]).  Grouped (offsets):
    returns the flat output buffers, group g at cols*off_g with shape [cols, M_g]."""
    return _transpose_common(lib().orc_direct_transpose, q, sf, offsets)


def naive_transpose(q, sf, offsets=None):
    return _transpose_common(lib().orc_naive_transpose, q, sf, offsets)


def exp_spec(a) -> np.ndarray:
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.float32)
    lib().orc_exp_spec_array(_p(a), a.size, _p(out))
    return out


def exp_spec_constants() -> np.ndarray:
    out = np.empty(11, np.float32)
    lib().orc_exp_spec_constants(_p(out))
    return out


def swiglu(g, u) -> np.ndarray:
    g = _c(g, np.float32)
    u = _c(u, np.float32)
    out = np.empty(g.shape, np.float32)
    lib().orc_swiglu_array(_p(g), _p(u), g.size, _p(out))
    return out


def swiglu_quant(gate_bits, up_bits, transposed: bool = True):
    g = _c(gate_bits, np.uint16)
    u = _c(up_bits, np.uint16)
    rows, cols = g.shape
    q = np.empty((rows, cols), np.uint8)
    sf = np.empty((rows, cols // 128), np.uint8)
    qt = np.empty((cols, rows), np.uint8) if transposed else None
    sft = np.empty((cols, rows // 128), np.uint8) if transposed else None
    rc = lib().orc_swiglu_quant(_p(g), _p(u), rows, cols, _p(q), _p(sf), _p(qt), _p(sft))
    if rc:
        raise OracleError(f"oracle swiglu_quant rejected its arguments (code {rc})")
    return q, sf, qt, sft


def permute_max_rows(tokens: int, topk: int, num_experts: int, align: int) -> int:
    return tokens * topk + num_experts * (align - 1)


def permute_pad_quant(x_bits, topk_idx, num_experts: int, align: int, max_rows: int | None = None,
                      fill: int = 0xEE):
    """Returns (Q [max_rows, H], SF [max_rows, H/128], offsets [E+1], row_id_map [T*K]).
    Rows at or beyond offsets[E] keep the `fill` byte (they are not written)."""
    x = _c(x_bits, np.uint16)
    idx = _c(topk_idx, np.int32)
    T, H = x.shape
    K = idx.shape[1] if idx.ndim == 2 else 1
    if max_rows is None:
        max_rows = permute_max_rows(T, K, num_experts, align)
    q = np.full((max_rows, H), fill, np.uint8)
    sf = np.full((max_rows, H // 128), fill, np.uint8)
    off = np.zeros(num_experts + 1, np.int32)
    rmap = np.zeros(T * K, np.int32)
    rc = lib().orc_permute_pad_quant(_p(x), T, H, _p(idx), K, num_experts, align, _p(q), _p(sf),
                                     max_rows, _p(off), _p(rmap))
    if rc:
        raise OracleError(f"oracle permute_pad_quant rejected its arguments (code {rc})")
    return q, sf, off, rmap


def permute_pad_fp8(q_bits, sf, topk_idx, num_experts: int, align: int, max_rows: int | None = None,
                    fill: int = 0xEE):
    """FP8-input permute + pad: the same outputs as permute_pad_quant, from row-wise codes
    q [T, H] and scales sf [T, H/128] instead of BF16 X."""
    xq = _c(q_bits, np.uint8)
    xsf = _c(sf, np.uint8)
    idx = _c(topk_idx, np.int32)
    T, H = xq.shape
    K = idx.shape[1] if idx.ndim == 2 else 1
    if max_rows is None:
        max_rows = permute_max_rows(T, K, num_experts, align)
    q = np.full((max_rows, H), fill, np.uint8)
    osf = np.full((max_rows, H // 128), fill, np.uint8)
    off = np.zeros(num_experts + 1, np.int32)
    rmap = np.zeros(T * K, np.int32)
    rc = lib().orc_permute_pad_fp8(_p(xq), _p(xsf), T, H, _p(idx), K, num_experts, align, _p(q), _p(osf), max_rows,
                                   _p(off), _p(rmap))
    if rc:
        raise OracleError(f"oracle FP8 permute rejected its arguments (code {rc})")
    return q, osf, off, rmap


def ep_dispatch_pack(q_bits, sf, topk_idx, num_ranks: int, experts_per_rank: int, fill: int = 0xEE):
    """Send side of one source rank of the expert-parallel FP8 dispatch: returns
    (send_q [S, H], send_sf [S, H/128], send_ids [S, K], send_offsets [W+1],
    send_map [T, W]) with S = send_offsets[W] (every token sent once to each rank that
    holds one of its experts, grouped by destination rank)."""
    xq = _c(q_bits, np.uint8)
    xsf = _c(sf, np.uint8)
    idx = _c(topk_idx, np.int32)
    T, H = xq.shape
    K = idx.shape[1]
    W = num_ranks
    cap = T * W
    sq = np.full((cap, H), fill, np.uint8)
    ssf = np.full((cap, H // 128), fill, np.uint8)
    sids = np.full((cap, K), -7, np.int32)
    soff = np.zeros(W + 1, np.int32)
    smap = np.zeros((T, W), np.int32)
    rc = lib().orc_ep_dispatch_pack(_p(xq), _p(xsf), T, H, _p(idx), K, W, experts_per_rank, _p(sq), _p(ssf),
                                    _p(sids), cap, _p(soff), _p(smap))
    if rc:
        raise OracleError(f"oracle EP dispatch pack rejected its arguments (code {rc})")
    S = int(soff[W])
    return sq[:S], ssf[:S], sids[:S], soff, smap


def ep_recv_permute(recv_q, recv_sf, recv_ids, experts_per_rank: int, align: int, max_rows: int | None = None,
                    fill: int = 0xEE):
    """Receive side of one destination rank: the rows received from every source rank
    (concatenated in source-rank order) -> (Q [max_rows, H], SF [max_rows, H/128],
    offsets [Eloc+1], row_id_map [R*K]); slots with id -1 (expert on another rank)
    get row id -1."""
    rq = _c(recv_q, np.uint8)
    rsf = _c(recv_sf, np.uint8)
    rids = _c(recv_ids, np.int32)
    R, H = rq.shape
    K = rids.shape[1] if rids.ndim == 2 else 1
    if max_rows is None:
        max_rows = permute_max_rows(R, K, experts_per_rank, align)
    q = np.full((max_rows, H), fill, np.uint8)
    osf = np.full((max_rows, H // 128), fill, np.uint8)
    off = np.zeros(experts_per_rank + 1, np.int32)
    rmap = np.zeros(R * K, np.int32)
    rc = lib().orc_ep_recv_permute(_p(rq), _p(rsf), _p(rids), R, H, K, experts_per_rank, align, _p(q), _p(osf),
                                   max_rows, _p(off), _p(rmap))
    if rc:
        raise OracleError(f"oracle EP receive permute rejected its arguments (code {rc})")
    return q, osf, off, rmap


def unpermute_unpad(y, row_id_map, topk: int, weights=None, y_sf=None):
    """Combine side: out bf16 bits [T, H] = sum_s w[t,s] * Y[row_id_map[t,s]] (fp32 fma
    chain in slot order, BF16 RNE).  y is bf16 bits [rows, H], or E4M3 codes [rows, H]
    with y_sf [rows, H/128].  row_id_map [T*topk] (or [T, topk]); weights fp32
    [T, topk] or None (all ones)."""
    rmap = _c(row_id_map, np.int32).reshape(-1, topk)
    T, K = rmap.shape
    if y_sf is None:
        yy = _c(y, np.uint16)
        sf = None
    else:
        yy = _c(y, np.uint8)
        sf = _c(y_sf, np.uint8)
    rows, H = yy.shape
    w = None if weights is None else _c(weights, np.float32)
    if w is not None and w.shape != (T, K):
        raise OracleError("weights must be [tokens, topk]")
    out = np.empty((T, H), np.uint16)
    rc = lib().orc_unpermute_unpad(_p(yy), _p(sf), rows, H, _p(rmap), _p(w), T, K, _p(out))
    if rc:
        raise OracleError(f"oracle unpermute rejected its arguments (code {rc})")
    return out


def e4m3_encode_f32_range(first: int, n: int) -> np.ndarray:
    """E4M3 codes of the fp32 values with bit patterns first..first+n-1 (0 for non-finite)."""
    out = np.empty(n, np.uint8)
    lib().orc_e4m3_encode_f32_range(first, n, _p(out))
    return out


def exp_spec_f32_range(first: int, n: int) -> np.ndarray:
    """The SwiGLU spec's exp of the fp32 values with bit patterns first..first+n-1 (0 for NaN)."""
    out = np.empty(n, np.float32)
    lib().orc_exp_spec_f32_range(first, n, _p(out))
    return out


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ---------------------------------------------------------------- error report
# Reported numbers, not parity: how far each column-wise result lands from the
# original tensor (the "double quantization error" of the FP8-Flow-MoE review,
# section 问题与动机), and DeepGEMM's calc_diff (DeepSeek FP8 与 DeepGEMM, §5.7).

def dequant_rowwise(q, sf) -> np.ndarray:
    vals = e4m3_decode(q)
    e = sf.astype(np.int64) - 127
    return vals * np.exp2(np.repeat(e, 128, axis=1).astype(np.float64))


def dequant_colwise(qt, sft) -> np.ndarray:
    """Dense Q^T [cols, rows] + SF^T [cols, rows/128] -> values [rows, cols]."""
    return dequant_rowwise(qt, sft).T


def naive_fp32_colwise(v: np.ndarray) -> np.ndarray:
    """Column requantization with non-power-of-two fp32 scales amax/448 (the SM90
    DeepGEMM convention, DeepSeek FP8 与 DeepGEMM §3): report-only reference for the
    genuine double-quantization case.  v: [rows, cols] float64, rows % 128 == 0.
    Returns the dequantized column-wise values [rows, cols]."""
    rows, cols = v.shape
    t = v.reshape(rows // 128, 128, cols)
    amax = np.abs(t).max(axis=1, keepdims=True).astype(np.float32)
    s = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0)).astype(np.float64)
    codes = e4m3_encode(t / s)
    return (e4m3_decode(codes) * s).reshape(rows, cols)


def rel_rms(approx: np.ndarray, exact: np.ndarray) -> float:
    exact = np.asarray(exact, np.float64)
    num = np.sqrt(np.sum((np.asarray(approx, np.float64) - exact) ** 2))
    den = np.sqrt(np.sum(exact ** 2))
    return float(num / den) if den > 0 else 0.0


def calc_diff(x: np.ndarray, y: np.ndarray) -> float:
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    den = np.sum(x * x + y * y)
    return float(1.0 - 2.0 * np.sum(x * y) / den) if den > 0 else 0.0
