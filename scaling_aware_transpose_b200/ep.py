"""Expert-parallel FP8 dispatch across ranks: one process per GPU, torch.distributed.

FP8-Flow-MoE review, 核心方法 and Table 1: the dispatch all-to-all carries row-wise FP8
codes with their UE8M0 scale bytes, not BF16 rows; DeepSeek FP8 §5.6: on the receiving
rank each local expert reads its rows as one contiguous, aligned group.

One call, on every rank of the group:
  1. pack (device): fp8q_ep_dispatch_pack groups this rank's tokens by destination rank,
     each token once per rank that holds one of its experts, with its slot ids
     re-expressed for that rank;
  2. exchange: the per-rank row counts, then the codes, scale bytes and slot ids, with
     all_to_all_single (over NCCL: grouped send/receive of device buffers, no host copy);
  3. receive-side permute (device): fp8q_ep_recv_permute_fp8 reads each source rank's
     segment of the receive buffers in place and writes the local experts'
     expert-grouped, padded layout.
Only the split sizes go through the host (they size the receive buffers).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass
class Dispatched:
    q: object                 # u8 [rows >= expert_offsets[-1], H]: local experts' rows, grouped, padded
    sf: object                # u8 [.., H/128] scale bytes
    expert_offsets: object    # int32 [experts_per_rank + 1]
    row_id_map: object        # int32 [R * K]: row of received slot (r, k), -1 for other ranks' experts
    recv_counts: list         # rows received from each source rank
    send_counts: list         # rows sent to each destination rank
    send_map: object          # int32 [T, W]: send row of (token, rank), -1 where not sent


class DeviceKernels:
    """The library's CUDA entry points for the two device steps."""

    @staticmethod
    def pack(xq, xsf, topk_idx, num_ranks, experts_per_rank):
        from . import ep_dispatch_pack
        return ep_dispatch_pack(xq, xsf, topk_idx, num_ranks, experts_per_rank)

    @staticmethod
    def recv_permute(segments, experts_per_rank, align):
        from . import ep_recv_permute
        return ep_recv_permute(segments, experts_per_rank, align)


def _prefix(counts):
    out, acc = [0], 0
    for c in counts:
        acc += c
        out.append(acc)
    return out


def dispatch(xq, xsf, topk_idx, experts_per_rank: int, align: int, group=None, kernels=None) -> Dispatched:
    """Dispatch this rank's row-wise FP8 tokens (xq [T, H], xsf [T, H/128]) routed by
    topk_idx [T, K] (global expert ids, expert e on rank e // experts_per_rank) to the
    ranks of `group`, and permute what arrives here into the local experts' layout.

    kernels: the two device steps; DeviceKernels (the CUDA library) unless given.  Tests
    of the exchange logic on CPU ranks pass implementations backed by the oracle."""
    import torch
    import torch.distributed as dist
    kern = kernels or DeviceKernels
    W = dist.get_world_size(group)
    T, H = xq.shape
    K = topk_idx.shape[1]
    send_q, send_sf, send_ids, send_off, send_map = kern.pack(xq, xsf, topk_idx, W, experts_per_rank)
    send_counts_t = (send_off[1:] - send_off[:-1]).to(torch.int64)
    recv_counts_t = torch.empty_like(send_counts_t)
    dist.all_to_all_single(recv_counts_t, send_counts_t, group=group)
    sc = [int(v) for v in send_counts_t.tolist()]
    rc = [int(v) for v in recv_counts_t.tolist()]
    S, R = sum(sc), sum(rc)
    recv_q = torch.empty((R, H), dtype=torch.uint8, device=xq.device)
    recv_sf = torch.empty((R, H // 128), dtype=torch.uint8, device=xq.device)
    recv_ids = torch.empty((R, K), dtype=torch.int32, device=xq.device)
    for out, inp in ((recv_q, send_q[:S]), (recv_sf, send_sf[:S]), (recv_ids, send_ids[:S])):
        dist.all_to_all_single(out, inp.contiguous(), output_split_sizes=rc, input_split_sizes=sc, group=group)
    bounds = _prefix(rc)
    segments = [(recv_q[bounds[s]:bounds[s + 1]], recv_sf[bounds[s]:bounds[s + 1]], recv_ids[bounds[s]:bounds[s + 1]])
                for s in range(W)]
    q, sf, off, rmap = kern.recv_permute(segments, experts_per_rank, align)
    return Dispatched(q, sf, off, rmap, rc, sc, send_map)
