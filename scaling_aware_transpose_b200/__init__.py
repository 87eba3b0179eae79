"""scaling_aware_transpose_b200 — Python binding of libfp8q (the C ABI in include/fp8q.h).

FP8-Flow-MoE's FP8 data-movement hot path on one B200: row-wise 1x128 E4M3
quantization with power-of-two scales, the scaling-aware direct transpose to the
column-wise layout, the naive three-pass baseline, fused SwiGLU+quantize and fused
permute+pad+quantize.  Every step runs in the library's CUDA kernels; this module only
marshals arguments (torch tensors -> device pointers, the current torch stream) and
turns non-zero status codes into exceptions.  There is no CPU fallback: if libfp8q.so
has not been built, every call raises.

The functions named ``fp8q_*`` mirror the C entry points argument for argument;
tensors stand in for pointers.  The lower-case helpers allocate outputs with torch.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8q.so")

STATUS = {
    0: "FP8Q_OK", 1: "FP8Q_ERR_NULL", 2: "FP8Q_ERR_SHAPE", 3: "FP8Q_ERR_ALIGN", 4: "FP8Q_ERR_ARG",
    5: "FP8Q_ERR_CUDA", 6: "FP8Q_ERR_TIMEOUT", 7: "FP8Q_ERR_DEVICE",
}
globals().update({name: code for code, name in STATUS.items()})


class Fp8qError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS.get(self.status, self.status)} ({_status_string(self.status)})")


class EpSource(ctypes.Structure):
    """fp8q_ep_source: one received segment (device pointers and its row count)."""
    _fields_ = [("q", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("ids", ctypes.c_void_p), ("rows", ctypes.c_int64)]


EP_MAX_RANKS = 64  # FP8Q_EP_MAX_RANKS

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libfp8q.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfp8q.so is missing ({LIB_PATH}); build it with "
                               "`python -m scaling_aware_transpose_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        sig = {
            "fp8q_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "fp8q_last_device_status": ([P], ctypes.c_int),
            "fp8q_quantize_rowwise": ([P, I64, I64, P, P, P], ctypes.c_int),
            "fp8q_direct_transpose": ([P, P, I64, I64, P, I32, P, P, P], ctypes.c_int),
            "fp8q_naive_workspace_bytes": ([I64, I64], SZ),
            "fp8q_naive_transpose": ([P, P, I64, I64, P, I32, P, P, P, SZ, P], ctypes.c_int),
            "fp8q_swiglu_quant": ([P, P, I64, I64, P, P, P, P, P], ctypes.c_int),
            "fp8q_packed_sf_bytes": ([I64, I64], SZ),
            "fp8q_quantize_rowwise_colwise": ([P, I64, I64, ctypes.c_uint32, P, P, P, P, P], ctypes.c_int),
            "fp8q_permute_workspace_bytes": ([I64, I32, I32], SZ),
            "fp8q_permute_pad_quant": ([P, I64, I64, P, I32, I32, I32, P, P, I64, P, P, P, SZ, P], ctypes.c_int),
            "fp8q_permute_pad_fp8": ([P, P, I64, I64, P, I32, I32, I32, P, P, I64, P, P, P, SZ, P], ctypes.c_int),
            "fp8q_permute_pad_quant_noalloc": ([P, I64, I64, P, I32, I32, I32, P, P, I64, P, P, P], ctypes.c_int),
            "fp8q_unpermute_unpad": ([P, P, I64, I64, P, P, I64, I32, P, P], ctypes.c_int),
            "fp8q_quantize_rowwise_mx32": ([P, I64, I64, P, P, P], ctypes.c_int),
            "fp8q_direct_transpose_mx32": ([P, P, I64, I64, P, P, P], ctypes.c_int),
            "fp8q_debug_expire_wait": ([ctypes.c_uint64, P], ctypes.c_int),
            "fp8q_debug_e4m3_encode_range": ([ctypes.c_uint32, I64, P, P], ctypes.c_int),
            "fp8q_debug_exp_spec_range": ([ctypes.c_uint32, I64, P, P], ctypes.c_int),
            "fp8q_debug_swiglu_spec": ([P, P, I64, P, P], ctypes.c_int),
            "fp8q_debug_silu_bf16": ([P, I64, P, P], ctypes.c_int),
            "fp8q_ep_pack_workspace_bytes": ([I64, I32], SZ),
            "fp8q_ep_dispatch_pack": ([P, P, I64, I64, P, I32, I32, I32, P, P, P, I64, P, P, P, SZ, P], ctypes.c_int),
            "fp8q_ep_recv_workspace_bytes": ([I64, I32, I32], SZ),
            "fp8q_ep_recv_permute_fp8": ([ctypes.POINTER(EpSource), I32, I64, I32, I32, I32, P, P, I64, P, P, P, SZ,
                                          P], ctypes.c_int),
            "fp8q_version": ([], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes, fn.restype = args, res
        _lib = L
    return _lib


def _status_string(code: int) -> str:
    try:
        return lib().fp8q_status_string(int(code)).decode()
    except Exception:  # pragma: no cover - only while reporting another error
        return "?"


# ---------------------------------------------------------------- marshalling
def _ptr(t):
    """Device pointer of a CUDA tensor (must be contiguous); ints pass through; None -> NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libfp8q takes device tensors; got a tensor on " + str(t.device))
    if not t.is_contiguous():
        raise ValueError("libfp8q takes contiguous tensors")
    return t.data_ptr() if t.numel() else None


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise Fp8qError(rc, where)


# ---------------------------------------------------------------- C entry points
def fp8q_last_device_status(stream=None) -> int:
    return int(lib().fp8q_last_device_status(_stream(stream)))


def fp8q_quantize_rowwise(x, rows: int, cols: int, q, sf, stream=None) -> None:
    _check(lib().fp8q_quantize_rowwise(_ptr(x), rows, cols, _ptr(q), _ptr(sf), _stream(stream)),
           "fp8q_quantize_rowwise")


def fp8q_direct_transpose(q, sf, rows: int, cols: int, group_offsets, num_groups: int, qt, sft,
                          stream=None) -> None:
    _check(lib().fp8q_direct_transpose(_ptr(q), _ptr(sf), rows, cols, _ptr(group_offsets), num_groups,
                                       _ptr(qt), _ptr(sft), _stream(stream)), "fp8q_direct_transpose")


def fp8q_naive_workspace_bytes(rows: int, cols: int) -> int:
    return int(lib().fp8q_naive_workspace_bytes(rows, cols))


def fp8q_naive_transpose(q, sf, rows: int, cols: int, group_offsets, num_groups: int, qt, sft, workspace,
                         workspace_bytes: int, stream=None) -> None:
    _check(lib().fp8q_naive_transpose(_ptr(q), _ptr(sf), rows, cols, _ptr(group_offsets), num_groups,
                                      _ptr(qt), _ptr(sft), _ptr(workspace), workspace_bytes,
                                      _stream(stream)), "fp8q_naive_transpose")


def fp8q_swiglu_quant(gate, up, rows: int, cols: int, q, sf, qt, sft, stream=None) -> None:
    _check(lib().fp8q_swiglu_quant(_ptr(gate), _ptr(up), rows, cols, _ptr(q), _ptr(sf), _ptr(qt), _ptr(sft),
                                   _stream(stream)), "fp8q_swiglu_quant")


ZERO_TILE_MIN_SCALE = 0x1  # FP8Q_ZERO_TILE_MIN_SCALE
SF_PACKED_UE8M0 = 0x2      # FP8Q_SF_PACKED_UE8M0


def fp8q_packed_sf_bytes(mn: int, k: int) -> int:
    return int(lib().fp8q_packed_sf_bytes(mn, k))


def fp8q_quantize_rowwise_colwise(x, rows: int, cols: int, flags: int, q, sf, qt, sft, stream=None) -> None:
    _check(lib().fp8q_quantize_rowwise_colwise(_ptr(x), rows, cols, int(flags), _ptr(q), _ptr(sf), _ptr(qt),
                                               _ptr(sft), _stream(stream)), "fp8q_quantize_rowwise_colwise")


def fp8q_permute_workspace_bytes(tokens: int, topk: int, num_experts: int) -> int:
    return int(lib().fp8q_permute_workspace_bytes(tokens, topk, num_experts))


def fp8q_permute_pad_fp8(xq, xsf, tokens: int, hidden: int, topk_idx, topk: int, num_experts: int, align: int,
                         q, sf, max_out_rows: int, expert_offsets, row_id_map, workspace, workspace_bytes: int,
                         stream=None) -> None:
    _check(lib().fp8q_permute_pad_fp8(_ptr(xq), _ptr(xsf), tokens, hidden, _ptr(topk_idx), topk, num_experts, align,
                                      _ptr(q), _ptr(sf), max_out_rows, _ptr(expert_offsets), _ptr(row_id_map),
                                      _ptr(workspace), workspace_bytes, _stream(stream)), "fp8q_permute_pad_fp8")


def fp8q_permute_pad_quant(x, tokens: int, hidden: int, topk_idx, topk: int, num_experts: int, align: int,
                           q, sf, max_out_rows: int, expert_offsets, row_id_map, workspace,
                           workspace_bytes: int, stream=None) -> None:
    _check(lib().fp8q_permute_pad_quant(_ptr(x), tokens, hidden, _ptr(topk_idx), topk, num_experts, align,
                                        _ptr(q), _ptr(sf), max_out_rows, _ptr(expert_offsets),
                                        _ptr(row_id_map), _ptr(workspace), workspace_bytes,
                                        _stream(stream)), "fp8q_permute_pad_quant")


NOALLOC_SCRATCH_BYTES = 4 << 20  # FP8Q_NOALLOC_SCRATCH_BYTES


def fp8q_permute_pad_quant_noalloc(x, tokens: int, hidden: int, topk_idx, topk: int, num_experts: int,
                                   align: int, q, sf, max_out_rows: int, expert_offsets, row_id_map,
                                   stream=None) -> None:
    """fp8q_permute_pad_quant without a workspace argument: the routing scratch lives in the
    library's static device array (for callers that cannot allocate device memory)."""
    _check(lib().fp8q_permute_pad_quant_noalloc(_ptr(x), tokens, hidden, _ptr(topk_idx), topk, num_experts,
                                                align, _ptr(q), _ptr(sf), max_out_rows, _ptr(expert_offsets),
                                                _ptr(row_id_map), _stream(stream)),
           "fp8q_permute_pad_quant_noalloc")


def fp8q_unpermute_unpad(y, y_sf, rows: int, hidden: int, row_id_map, weights, tokens: int, topk: int, out,
                         stream=None) -> None:
    _check(lib().fp8q_unpermute_unpad(_ptr(y), _ptr(y_sf), rows, hidden, _ptr(row_id_map), _ptr(weights), tokens,
                                      topk, _ptr(out), _stream(stream)), "fp8q_unpermute_unpad")


def fp8q_quantize_rowwise_mx32(x, rows: int, cols: int, q, sf, stream=None) -> None:
    _check(lib().fp8q_quantize_rowwise_mx32(_ptr(x), rows, cols, _ptr(q), _ptr(sf), _stream(stream)),
           "fp8q_quantize_rowwise_mx32")


def fp8q_direct_transpose_mx32(q, sf, rows: int, cols: int, qt, sft, stream=None) -> None:
    _check(lib().fp8q_direct_transpose_mx32(_ptr(q), _ptr(sf), rows, cols, _ptr(qt), _ptr(sft), _stream(stream)),
           "fp8q_direct_transpose_mx32")


def fp8q_debug_expire_wait(timeout_ns: int, stream=None) -> None:
    _check(lib().fp8q_debug_expire_wait(int(timeout_ns), _stream(stream)), "fp8q_debug_expire_wait")


def fp8q_debug_e4m3_encode_range(first_bits: int, n: int, out, stream=None) -> None:
    _check(lib().fp8q_debug_e4m3_encode_range(first_bits, n, _ptr(out), _stream(stream)),
           "fp8q_debug_e4m3_encode_range")


def fp8q_debug_exp_spec_range(first_bits: int, n: int, out, stream=None) -> None:
    _check(lib().fp8q_debug_exp_spec_range(first_bits, n, _ptr(out), _stream(stream)), "fp8q_debug_exp_spec_range")


def fp8q_debug_swiglu_spec(gate, up, n: int, y, stream=None) -> None:
    _check(lib().fp8q_debug_swiglu_spec(_ptr(gate), _ptr(up), n, _ptr(y), _stream(stream)), "fp8q_debug_swiglu_spec")


def fp8q_debug_silu_bf16(gate, n: int, y, stream=None) -> None:
    _check(lib().fp8q_debug_silu_bf16(_ptr(gate), n, _ptr(y), _stream(stream)), "fp8q_debug_silu_bf16")


def fp8q_version() -> int:
    return int(lib().fp8q_version())


# ---------------------------------------------------------------- allocating helpers
def _empty(shape, dtype, like):
    import torch
    return torch.empty(shape, dtype=dtype, device=like.device)


def quantize_rowwise(x, stream=None):
    """x: bf16 [rows, cols] on the GPU -> (q u8 [rows, cols], sf u8 [rows, cols/128])."""
    import torch
    rows, cols = x.shape
    q = _empty((rows, cols), torch.uint8, x)
    sf = _empty((rows, cols // 128), torch.uint8, x)
    fp8q_quantize_rowwise(x, rows, cols, q, sf, stream)
    return q, sf


def direct_transpose(q, sf, group_offsets=None, stream=None):
    """Dense: (Q^T [cols, rows], SF^T [cols, rows/128]).  Grouped (device int32 offsets):
    flat buffers of rows*cols and rows*cols/128 bytes, group g at cols*off[g]."""
    import torch
    rows, cols = q.shape
    G = 1 if group_offsets is None else group_offsets.numel() - 1
    if group_offsets is None:
        qt = _empty((cols, rows), torch.uint8, q)
        sft = _empty((cols, rows // 128), torch.uint8, q)
    else:
        qt = _empty((rows * cols,), torch.uint8, q)
        sft = _empty((rows * cols // 128,), torch.uint8, q)
    fp8q_direct_transpose(q, sf, rows, cols, group_offsets, G, qt, sft, stream)
    return qt, sft


def naive_transpose(q, sf, group_offsets=None, workspace=None, stream=None):
    import torch
    rows, cols = q.shape
    G = 1 if group_offsets is None else group_offsets.numel() - 1
    need = fp8q_naive_workspace_bytes(rows, cols)
    if workspace is None:
        workspace = _empty((max(need, 16),), torch.uint8, q)
    if group_offsets is None:
        qt = _empty((cols, rows), torch.uint8, q)
        sft = _empty((cols, rows // 128), torch.uint8, q)
    else:
        qt = _empty((rows * cols,), torch.uint8, q)
        sft = _empty((rows * cols // 128,), torch.uint8, q)
    fp8q_naive_transpose(q, sf, rows, cols, group_offsets, G, qt, sft, workspace, workspace.numel(), stream)
    return qt, sft


def swiglu_quant(gate, up, transposed: bool = True, stream=None):
    import torch
    rows, cols = gate.shape
    q = _empty((rows, cols), torch.uint8, gate)
    sf = _empty((rows, cols // 128), torch.uint8, gate)
    qt = _empty((cols, rows), torch.uint8, gate) if transposed else None
    sft = _empty((cols, rows // 128), torch.uint8, gate) if transposed else None
    fp8q_swiglu_quant(gate, up, rows, cols, q, sf, qt, sft, stream)
    return q, sf, qt, sft


def packed_sf_shape(mn: int, k: int) -> tuple[int, int]:
    """Shape (int32 words) of packed UE8M0 scales for an operand [mn, k]."""
    return ((k // 128 + 3) // 4, (mn + 3) // 4 * 4)


def quantize_rowwise_colwise(x, flags: int = 0, colwise: bool = True, stream=None):
    """One read of x -> (Q, SF, Q^T, SF^T); Q^T/SF^T are None when colwise is False.
    With SF_PACKED_UE8M0 the scales are int32 tensors of packed UE8M0 words."""
    import torch
    rows, cols = x.shape
    packed = bool(flags & SF_PACKED_UE8M0)
    q = _empty((rows, cols), torch.uint8, x)
    sf = (_empty(packed_sf_shape(rows, cols), torch.int32, x) if packed
          else _empty((rows, cols // 128), torch.uint8, x))
    qt = sft = None
    if colwise:
        qt = _empty((cols, rows), torch.uint8, x)
        sft = (_empty(packed_sf_shape(cols, rows), torch.int32, x) if packed
               else _empty((cols, rows // 128), torch.uint8, x))
    fp8q_quantize_rowwise_colwise(x, rows, cols, flags, q, sf, qt, sft, stream)
    return q, sf, qt, sft


def permute_max_rows(tokens: int, topk: int, num_experts: int, align: int) -> int:
    return tokens * topk + num_experts * (align - 1)


def permute_pad_quant(x, topk_idx, num_experts: int, align: int, max_out_rows: int | None = None, stream=None):
    """Returns (q [max_out_rows, H], sf [max_out_rows, H/128], expert_offsets [E+1],
    row_id_map [T*K]); rows at or beyond expert_offsets[E] are left unwritten."""
    import torch
    tokens, hidden = x.shape
    topk = topk_idx.shape[1]
    if max_out_rows is None:
        max_out_rows = permute_max_rows(tokens, topk, num_experts, align)
    q = _empty((max_out_rows, hidden), torch.uint8, x)
    sf = _empty((max_out_rows, hidden // 128), torch.uint8, x)
    off = _empty((num_experts + 1,), torch.int32, x)
    rmap = _empty((tokens * topk,), torch.int32, x)
    ws_bytes = fp8q_permute_workspace_bytes(tokens, topk, num_experts)
    ws = _empty((max(ws_bytes, 16),), torch.uint8, x)
    fp8q_permute_pad_quant(x, tokens, hidden, topk_idx, topk, num_experts, align, q, sf, max_out_rows, off,
                           rmap, ws, ws.numel(), stream)
    return q, sf, off, rmap


def permute_pad_fp8(xq, xsf, topk_idx, num_experts: int, align: int, max_out_rows: int | None = None, stream=None):
    """FP8-input permute: same outputs as permute_pad_quant, from row-wise codes xq
    [T, H] and scale bytes xsf [T, H/128]."""
    import torch
    tokens, hidden = xq.shape
    topk = topk_idx.shape[1]
    if max_out_rows is None:
        max_out_rows = permute_max_rows(tokens, topk, num_experts, align)
    q = _empty((max_out_rows, hidden), torch.uint8, xq)
    sf = _empty((max_out_rows, hidden // 128), torch.uint8, xq)
    off = _empty((num_experts + 1,), torch.int32, xq)
    rmap = _empty((tokens * topk,), torch.int32, xq)
    ws_bytes = fp8q_permute_workspace_bytes(tokens, topk, num_experts)
    ws = _empty((max(ws_bytes, 16),), torch.uint8, xq)
    fp8q_permute_pad_fp8(xq, xsf, tokens, hidden, topk_idx, topk, num_experts, align, q, sf, max_out_rows, off, rmap,
                         ws, ws.numel(), stream)
    return q, sf, off, rmap


def unpermute_unpad(y, row_id_map, topk: int, weights=None, y_sf=None, stream=None):
    """Combine side of the permute: BF16 [tokens, hidden] from the expert-ordered rows y
    (BF16, or E4M3 codes with row-wise scales y_sf) gathered by row_id_map [tokens*topk]
    and summed with weights [tokens, topk] (None: all ones)."""
    import torch
    rows, hidden = y.shape
    tokens = row_id_map.numel() // topk
    out = _empty((tokens, hidden), torch.bfloat16, y)
    fp8q_unpermute_unpad(y, y_sf, rows, hidden, row_id_map, weights, tokens, topk, out, stream)
    return out


def quantize_rowwise_mx32(x, stream=None):
    """1x32 tiles: (q [rows, cols], sf [rows, cols/32])."""
    import torch
    rows, cols = x.shape
    q = _empty((rows, cols), torch.uint8, x)
    sf = _empty((rows, cols // 32), torch.uint8, x)
    fp8q_quantize_rowwise_mx32(x, rows, cols, q, sf, stream)
    return q, sf


def direct_transpose_mx32(q, sf, stream=None):
    """32x32 blocks: (qt [cols, rows], sft [cols, rows/32])."""
    import torch
    rows, cols = q.shape
    qt = _empty((cols, rows), torch.uint8, q)
    sft = _empty((cols, rows // 32), torch.uint8, q)
    fp8q_direct_transpose_mx32(q, sf, rows, cols, qt, sft, stream)
    return qt, sft


# ---------------------------------------------------------------- expert-parallel dispatch
def fp8q_ep_pack_workspace_bytes(tokens: int, num_ranks: int) -> int:
    return int(lib().fp8q_ep_pack_workspace_bytes(tokens, num_ranks))


def fp8q_ep_recv_workspace_bytes(rows: int, topk: int, experts_per_rank: int) -> int:
    return int(lib().fp8q_ep_recv_workspace_bytes(rows, topk, experts_per_rank))


def fp8q_ep_dispatch_pack(xq, xsf, tokens: int, hidden: int, topk_idx, topk: int, num_ranks: int,
                          experts_per_rank: int, send_q, send_sf, send_ids, max_send_rows: int, send_offsets,
                          send_map, workspace, workspace_bytes: int, stream=None) -> None:
    _check(lib().fp8q_ep_dispatch_pack(_ptr(xq), _ptr(xsf), tokens, hidden, _ptr(topk_idx), topk, num_ranks,
                                       experts_per_rank, _ptr(send_q), _ptr(send_sf), _ptr(send_ids), max_send_rows,
                                       _ptr(send_offsets), _ptr(send_map), _ptr(workspace), workspace_bytes,
                                       _stream(stream)), "fp8q_ep_dispatch_pack")


def fp8q_ep_recv_permute_fp8(segments, hidden: int, topk: int, experts_per_rank: int, align: int, q, sf,
                             max_out_rows: int, expert_offsets, row_id_map, workspace, workspace_bytes: int,
                             stream=None) -> None:
    """segments: sequence of (q, sf, ids, rows) with q/sf/ids device tensors (or raw
    device addresses as ints) of the received rows of one source rank each."""
    arr = (EpSource * len(segments))()
    for i, (sq, ssf, sids, rows) in enumerate(segments):
        arr[i] = EpSource(_ptr(sq), _ptr(ssf), _ptr(sids), int(rows))
    _check(lib().fp8q_ep_recv_permute_fp8(arr, len(segments), hidden, topk, experts_per_rank, align, _ptr(q), _ptr(sf),
                                          max_out_rows, _ptr(expert_offsets), _ptr(row_id_map), _ptr(workspace),
                                          workspace_bytes, _stream(stream)), "fp8q_ep_recv_permute_fp8")


def ep_dispatch_pack(xq, xsf, topk_idx, num_ranks: int, experts_per_rank: int, stream=None):
    """Send side of one rank: (send_q [cap, H], send_sf [cap, H/128], send_ids [cap, K],
    send_offsets [W+1], send_map [T, W]); rows send_offsets[W] and beyond are unused."""
    import torch
    tokens, hidden = xq.shape
    topk = topk_idx.shape[1]
    cap = max(tokens * min(num_ranks, topk), 1)
    send_q = _empty((cap, hidden), torch.uint8, xq)
    send_sf = _empty((cap, hidden // 128), torch.uint8, xq)
    send_ids = _empty((cap, topk), torch.int32, xq)
    send_off = _empty((num_ranks + 1,), torch.int32, xq)
    send_map = _empty((tokens, num_ranks), torch.int32, xq)
    ws_bytes = fp8q_ep_pack_workspace_bytes(tokens, num_ranks)
    ws = _empty((max(ws_bytes, 16),), torch.uint8, xq)
    fp8q_ep_dispatch_pack(xq, xsf, tokens, hidden, topk_idx, topk, num_ranks, experts_per_rank, send_q, send_sf,
                          send_ids, cap, send_off, send_map, ws, ws.numel(), stream)
    return send_q, send_sf, send_ids, send_off, send_map


def ep_recv_permute(segments, experts_per_rank: int, align: int, max_out_rows: int | None = None, stream=None):
    """Receive side of one rank from per-source segments (q [n, H], sf [n, H/128],
    ids [n, K]) -> (q [max_out_rows, H], sf, expert_offsets [Eloc+1], row_id_map [R*K])."""
    import torch
    ref = next(s[0] for s in segments)
    hidden = ref.shape[1]
    topk = next(s[2] for s in segments).shape[1]
    rows = sum(int(s[0].shape[0]) for s in segments)
    if max_out_rows is None:
        max_out_rows = permute_max_rows(rows, topk, experts_per_rank, align)
    q = _empty((max(max_out_rows, 1), hidden), torch.uint8, ref)
    sf = _empty((max(max_out_rows, 1), hidden // 128), torch.uint8, ref)
    off = _empty((experts_per_rank + 1,), torch.int32, ref)
    rmap = _empty((max(rows * topk, 1),), torch.int32, ref)
    ws_bytes = fp8q_ep_recv_workspace_bytes(rows, topk, experts_per_rank)
    ws = _empty((max(ws_bytes, 16),), torch.uint8, ref)
    fp8q_ep_recv_permute_fp8([(a, b, c, a.shape[0]) for a, b, c in segments], hidden, topk, experts_per_rank, align,
                             q, sf, max_out_rows, off, rmap, ws, ws.numel(), stream)
    return q, sf, off, rmap[:rows * topk]
