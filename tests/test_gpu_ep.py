"""GPU parity of the expert-parallel FP8 dispatch against the CPU oracle, byte for byte.

W ranks are simulated on one GPU: each source rank's tokens are packed by
fp8q_ep_dispatch_pack; each destination rank's receive permute (fp8q_ep_recv_permute_fp8)
is then given, as its segments, the slices of the source ranks' send buffers that an
all-to-all would deliver to it - read in place, as they would be read from a receive
buffer.  The exchange itself runs through NCCL on a one-rank group (all this machine
offers); its multi-rank logic is covered on gloo ranks in test_ep_host.py.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import assert_bytes_equal, dev, device_status_ok, host

pytestmark = pytest.mark.gpu


def _sources(W, T, H, K, Eloc, seed, row_sigma=1.0):
    rng = np.random.default_rng(seed)
    xs, idx = [], []
    for s in range(W):
        q, sf = oracle.quantize_rowwise(synthetic.scaled_normal(T, H, seed=seed + s, row_sigma=row_sigma))
        xs.append((q, sf))
        idx.append(synthetic.zipf_topk(T, W * Eloc, K, rng) if T else np.zeros((0, K), np.int32))
    return xs, idx


def _check_pack(got, want, T):
    sq, ssf, sids, soff, smap = got
    oq, osf, oids, ooff, omap = want
    assert_bytes_equal(host(soff), ooff, "send offsets")
    assert_bytes_equal(host(smap), omap, "send map")
    S = int(ooff[-1])
    assert_bytes_equal(host(sids)[:S], oids, "send ids")
    assert_bytes_equal(host(ssf)[:S], osf, "send SF")
    assert_bytes_equal(host(sq)[:S], oq, "send Q")


def run_ep(W, T, H, K, Eloc, align, seed=0):
    """Pack on every simulated source rank, receive-permute on every destination rank;
    compare each step with the oracle and the result with the global FP8 permute."""
    xs, idx = _sources(W, T, H, K, Eloc, seed)
    packs_d, packs_o = [], []
    for s in range(W):
        got = sat.ep_dispatch_pack(dev(xs[s][0]), dev(xs[s][1]), dev(idx[s]), W, Eloc)
        device_status_ok()
        want = oracle.ep_dispatch_pack(xs[s][0], xs[s][1], idx[s], W, Eloc)
        _check_pack(got, want, T)
        packs_d.append(got)
        packs_o.append(want)
    gq, gsf, goff, _ = oracle.permute_pad_fp8(np.concatenate([x[0] for x in xs]), np.concatenate([x[1] for x in xs]),
                                              np.concatenate(idx), W * Eloc, align)
    for d in range(W):
        segs = []
        for s in range(W):
            a, b = int(packs_o[s][3][d]), int(packs_o[s][3][d + 1])
            sq, ssf, sids = packs_d[s][0], packs_d[s][1], packs_d[s][2]
            segs.append((sq[a:b], ssf[a:b], sids[a:b]))
        q, sf, off, rmap = sat.ep_recv_permute(segs, Eloc, align)
        device_status_ok()
        rq = np.concatenate([p[0][p[3][d]:p[3][d + 1]] for p in packs_o])
        rsf = np.concatenate([p[1][p[3][d]:p[3][d + 1]] for p in packs_o])
        rids = np.concatenate([p[2][p[3][d]:p[3][d + 1]] for p in packs_o])
        oq, osf, ooff, ormap = oracle.ep_recv_permute(rq, rsf, rids, Eloc, align)
        assert_bytes_equal(host(off), ooff, f"rank {d} expert offsets")
        assert_bytes_equal(host(rmap), ormap, f"rank {d} row_id_map")
        n = int(ooff[-1])
        assert_bytes_equal(host(sf)[:n], osf[:n], f"rank {d} SF")
        assert_bytes_equal(host(q)[:n], oq[:n], f"rank {d} Q")
        base = int(goff[d * Eloc])
        assert np.array_equal(oq[:n], gq[base:base + n])


@pytest.mark.parametrize("W,T,H,K,Eloc,align", [(2, 300, 256, 4, 4, 16), (4, 512, 384, 8, 8, 128),
                                                 (8, 200, 128, 2, 1, 1), (3, 1000, 512, 6, 5, 64),
                                                 (1, 700, 256, 3, 7, 16), (5, 0, 256, 2, 2, 16)])
def test_ep_dispatch_simulated_ranks(W, T, H, K, Eloc, align):
    run_ep(W, T, H, K, Eloc, align, seed=W * 7 + T)


def test_ep_dispatch_moe_workload():
    """The MoE workload split over 4 expert-parallel ranks: 4 x 4096 tokens of hidden 7168,
    top-8 of 32 Zipf(1.1) experts, 8 experts per rank, 128-row alignment."""
    run_ep(4, 4096, 7168, 8, 8, 128, seed=0)


def test_ep_many_ranks_and_empty_segments():
    """64 ranks (the maximum), one expert each, few tokens: many empty segments."""
    run_ep(64, 20, 128, 2, 1, 16, seed=3)


def test_ep_pack_large_routing_takes_the_unfused_rank_path():
    """64 ranks x 4096 tokens: 262144 destination pairs, too many chunks for the fused rank
    kernel, so the pack runs the routing's separate scan and rank launches."""
    W, T, H, K, Eloc = 64, 4096, 128, 2, 1
    xs, idx = _sources(1, T, H, K, W * Eloc, seed=6)
    rng = np.random.default_rng(6)
    idx = synthetic.zipf_topk(T, W * Eloc, K, rng)
    got = sat.ep_dispatch_pack(dev(xs[0][0]), dev(xs[0][1]), dev(idx), W, Eloc)
    device_status_ok()
    _check_pack(got, oracle.ep_dispatch_pack(xs[0][0], xs[0][1], idx, W, Eloc), T)


def test_ep_duplicate_experts_and_one_hot_rank():
    """Routing the Zipf sampler never draws: two slots of a token on the same expert (one
    send row, two slot ids, two expert rows), and every token routed to rank 2's experts
    only (ranks 0, 1, 3 receive nothing)."""
    W, T, H, K, Eloc, align = 4, 300, 256, 3, 4, 16
    rng = np.random.default_rng(12)
    xs = [oracle.quantize_rowwise(synthetic.scaled_normal(T, H, seed=40 + s)) for s in range(W)]
    for mode in ("dup", "one_rank"):
        idx = []
        for s in range(W):
            if mode == "dup":
                a = rng.integers(0, W * Eloc, (T, K)).astype(np.int32)
                a[:, 1] = a[:, 0]
            else:
                a = (2 * Eloc + rng.integers(0, Eloc, (T, K))).astype(np.int32)
            idx.append(np.ascontiguousarray(a))
        packs_d = [sat.ep_dispatch_pack(dev(xs[s][0]), dev(xs[s][1]), dev(idx[s]), W, Eloc) for s in range(W)]
        device_status_ok()
        packs_o = [oracle.ep_dispatch_pack(xs[s][0], xs[s][1], idx[s], W, Eloc) for s in range(W)]
        for s in range(W):
            _check_pack(packs_d[s], packs_o[s], T)
        for d in range(W):
            segs = [(p[0][int(o[3][d]):int(o[3][d + 1])], p[1][int(o[3][d]):int(o[3][d + 1])],
                     p[2][int(o[3][d]):int(o[3][d + 1])]) for p, o in zip(packs_d, packs_o)]
            q, sf, off, rmap = sat.ep_recv_permute(segs, Eloc, align)
            device_status_ok()
            rq = np.concatenate([p[0][p[3][d]:p[3][d + 1]] for p in packs_o])
            rsf = np.concatenate([p[1][p[3][d]:p[3][d + 1]] for p in packs_o])
            rids = np.concatenate([p[2][p[3][d]:p[3][d + 1]] for p in packs_o])
            oq, osf, ooff, ormap = oracle.ep_recv_permute(rq, rsf, rids, Eloc, align)
            assert_bytes_equal(host(off), ooff, f"{mode} rank {d} offsets")
            n = int(ooff[-1])
            if rq.shape[0]:
                assert_bytes_equal(host(rmap), ormap, f"{mode} rank {d} row_id_map")
            assert_bytes_equal(host(q)[:n], oq[:n], f"{mode} rank {d} Q")
            assert_bytes_equal(host(sf)[:n], osf[:n], f"{mode} rank {d} SF")


def test_ep_back_to_back_calls_share_one_workspace():
    """Two different routings, packed (and then receive-permuted) alternately on one stream
    through ONE workspace, with no synchronisation between the calls.  The kernels of a
    call may be placed before the previous call's kernels end (dependent launches), so a
    kernel that read routing data written inside its own call before waiting for it would
    see the other routing's stale values here.  Every result must still be the oracle's."""
    W, T, H, K, Eloc, align = 4, 4096, 256, 8, 8, 128
    xs, idx_a = _sources(W, T, H, K, Eloc, seed=21)
    _, idx_b = _sources(W, T, H, K, Eloc, seed=77)
    q0, sf0 = dev(xs[0][0]), dev(xs[0][1])
    routings = [dev(idx_a[0]), dev(idx_b[0])]
    cap = T * min(W, K)
    ws = torch.empty(sat.fp8q_ep_pack_workspace_bytes(T, W), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in routings:
        outs.append((torch.empty((cap, H), dtype=torch.uint8, device="cuda"),
                     torch.empty((cap, H // 128), dtype=torch.uint8, device="cuda"),
                     torch.empty((cap, K), dtype=torch.int32, device="cuda"),
                     torch.empty((W + 1,), dtype=torch.int32, device="cuda"),
                     torch.empty((T, W), dtype=torch.int32, device="cuda")))
    for rep in range(6):
        for r, idx in enumerate(routings):
            o = outs[r]
            sat.fp8q_ep_dispatch_pack(q0, sf0, T, H, idx, K, W, Eloc, o[0], o[1], o[2], cap, o[3], o[4], ws,
                                      ws.numel())
    device_status_ok()
    wants = [oracle.ep_dispatch_pack(xs[0][0], xs[0][1], i, W, Eloc) for i in (idx_a[0], idx_b[0])]
    for r in range(2):
        _check_pack(outs[r], wants[r], T)
    # the receive side: rank 0's segment of each routing's pack, alternately
    segs = []
    for r in range(2):
        a, b = int(wants[r][3][0]), int(wants[r][3][1])
        segs.append([(outs[r][0][a:b], outs[r][1][a:b], outs[r][2][a:b], b - a)])
    rows = [sg[0][3] for sg in segs]
    rws = torch.empty(max(sat.fp8q_ep_recv_workspace_bytes(n, K, Eloc) for n in rows), dtype=torch.uint8,
                      device="cuda")
    rout = []
    for n in rows:
        m = sat.permute_max_rows(n, K, Eloc, align)
        rout.append((torch.empty((m, H), dtype=torch.uint8, device="cuda"),
                     torch.empty((m, H // 128), dtype=torch.uint8, device="cuda"),
                     torch.empty((Eloc + 1,), dtype=torch.int32, device="cuda"),
                     torch.empty((max(n * K, 1),), dtype=torch.int32, device="cuda"), m))
    for rep in range(6):
        for r in range(2):
            o = rout[r]
            sat.fp8q_ep_recv_permute_fp8(segs[r], H, K, Eloc, align, o[0], o[1], o[4], o[2], o[3], rws, rws.numel())
    device_status_ok()
    for r in range(2):
        a, b = int(wants[r][3][0]), int(wants[r][3][1])
        oq, osf, ooff, ormap = oracle.ep_recv_permute(wants[r][0][a:b], wants[r][1][a:b], wants[r][2][a:b], Eloc,
                                                      align)
        assert_bytes_equal(host(rout[r][2]), ooff, f"routing {r} offsets")
        n = int(ooff[-1])
        assert_bytes_equal(host(rout[r][3])[:rows[r] * K], ormap, f"routing {r} row_id_map")
        assert_bytes_equal(host(rout[r][0])[:n], oq[:n], f"routing {r} Q")
        assert_bytes_equal(host(rout[r][1])[:n], osf[:n], f"routing {r} SF")


def test_ep_bad_ids_set_device_status():
    q = torch.zeros((4, 128), dtype=torch.uint8, device="cuda")
    sf = torch.full((4, 1), 127, dtype=torch.uint8, device="cuda")
    idx = torch.tensor([[0], [1], [9], [2]], dtype=torch.int32, device="cuda")
    sat.ep_dispatch_pack(q, sf, idx, 2, 4)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE
    ids = torch.tensor([[0], [-2], [1], [2]], dtype=torch.int32, device="cuda")
    sat.ep_recv_permute([(q, sf, ids)], 4, 16)
    assert sat.fp8q_last_device_status() == sat.FP8Q_ERR_DEVICE


def test_ep_dispatch_through_nccl_one_rank():
    """ep.dispatch end to end over a one-rank NCCL group: all_to_all_single of device
    buffers, then the receive permute; with one rank the result is the FP8 permute's."""
    import torch.distributed as dist
    from scaling_aware_transpose_b200 import ep
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=datetime.timedelta(seconds=60))
    try:
        xs, idx = _sources(1, 2048, 1024, 8, 16, seed=5)
        res = ep.dispatch(dev(xs[0][0]), dev(xs[0][1]), dev(idx[0]), 16, 128)
        device_status_ok()
        oq, osf, ooff, ormap = oracle.permute_pad_fp8(xs[0][0], xs[0][1], idx[0], 16, 128)
        assert_bytes_equal(host(res.expert_offsets), ooff, "offsets")
        assert_bytes_equal(host(res.row_id_map), ormap, "row_id_map")
        n = int(ooff[-1])
        assert_bytes_equal(host(res.q)[:n], oq[:n], "Q")
        assert_bytes_equal(host(res.sf)[:n], osf[:n], "SF")
        assert res.recv_counts == res.send_counts == [2048]
    finally:
        dist.destroy_process_group()
