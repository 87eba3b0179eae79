"""Host side of the expert-parallel FP8 dispatch, without a GPU: the exchange logic of
ep.dispatch on 2 and 3 gloo ranks (CPU processes), with the two device steps stood in
for by the oracle, checked against the single-device oracle permute; and the C entry
points' argument checks, which return before any CUDA call."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

import scaling_aware_transpose_b200 as sat


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _OracleKernels:
    """The pack and the receive permute computed by the oracle on CPU tensors (test
    stand-ins for the CUDA entry points; the exchange between them is the product's)."""

    @staticmethod
    def pack(xq, xsf, topk_idx, num_ranks, experts_per_rank):
        import torch
        import oracle
        sq, ssf, sids, soff, smap = oracle.ep_dispatch_pack(xq.numpy(), xsf.numpy(), topk_idx.numpy(), num_ranks,
                                                            experts_per_rank)
        return tuple(torch.from_numpy(np.ascontiguousarray(a)) for a in (sq, ssf, sids, soff, smap))

    @staticmethod
    def recv_permute(segments, experts_per_rank, align):
        import torch
        import oracle
        rq = np.concatenate([s[0].numpy() for s in segments])
        rsf = np.concatenate([s[1].numpy() for s in segments])
        rids = np.concatenate([s[2].numpy() for s in segments])
        out = oracle.ep_recv_permute(rq, rsf, rids, experts_per_rank, align)
        return tuple(torch.from_numpy(np.ascontiguousarray(a)) for a in out)


def _inputs(W, T, H, K, Eloc, seed):
    """Every rank's tokens and routing, from one seed (each rank takes its own)."""
    import oracle
    from scaling_aware_transpose_b200 import synthetic
    rng = np.random.default_rng(seed)
    xs, idx = [], []
    for s in range(W):
        q, sf = oracle.quantize_rowwise(synthetic.scaled_normal(T, H, seed=seed + s, row_sigma=1.0))
        xs.append((q, sf))
        idx.append(synthetic.zipf_topk(T, W * Eloc, K, rng))
    return xs, idx


def _rank_main(rank, world, port, cfg, out_q):
    import torch
    import torch.distributed as dist
    import oracle
    from scaling_aware_transpose_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, H, K, Eloc, align, seed = cfg
        xs, idx = _inputs(world, T, H, K, Eloc, seed)
        res = ep.dispatch(torch.from_numpy(xs[rank][0]), torch.from_numpy(xs[rank][1]), torch.from_numpy(idx[rank]),
                          Eloc, align, kernels=_OracleKernels)
        gq, gsf, goff, _ = oracle.permute_pad_fp8(np.concatenate([x[0] for x in xs]),
                                                  np.concatenate([x[1] for x in xs]), np.concatenate(idx),
                                                  world * Eloc, align)
        base = int(goff[rank * Eloc])
        off = res.expert_offsets.numpy()
        n = int(off[-1])
        ok = (np.array_equal(off, goff[rank * Eloc:(rank + 1) * Eloc + 1] - base)
              and np.array_equal(res.q.numpy()[:n], gq[base:base + n])
              and np.array_equal(res.sf.numpy()[:n], gsf[base:base + n]))
        dist.barrier()
        out_q.put((rank, ok, res.recv_counts, res.send_counts))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cfg", [(2, (96, 256, 4, 3, 16, 1)), (3, (50, 128, 2, 2, 128, 7))])
def test_dispatch_exchange_on_gloo_ranks(world, cfg):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, cfg, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs)
    res = {r: (ok, rc, sc) for r, ok, rc, sc in (q.get(timeout=5) for _ in range(world))}
    assert all(v[0] for v in res.values())
    # what rank s sent to rank d is what rank d received from rank s
    for s in range(world):
        for d in range(world):
            assert res[s][2][d] == res[d][1][s]


# ------------------------------------------------------------------ C entry points: host-side checks
def test_ep_workspace_sizes():
    L = sat.lib()
    assert L.fp8q_ep_pack_workspace_bytes(4096, 8) >= 4096 * 8 * 4
    assert L.fp8q_ep_pack_workspace_bytes(-1, 8) == 0 and L.fp8q_ep_pack_workspace_bytes(10, 65) == 0
    assert L.fp8q_ep_recv_workspace_bytes(1000, 8, 8) >= 1000 * 8 * 4
    assert L.fp8q_ep_recv_workspace_bytes(1 << 40, 8, 8) == 0


def test_ep_pack_host_errors():
    f = sat.lib().fp8q_ep_dispatch_pack
    A = 0x10000
    ws = sat.fp8q_ep_pack_workspace_bytes(64, 4)
    ok = dict(xq=A, xsf=A, tokens=64, hidden=256, idx=A, topk=2, W=4, Eloc=2, sq=A, ssf=A, sids=A, cap=128,
              soff=A, smap=A, ws=A, wsb=ws)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["xq"], a["xsf"], a["tokens"], a["hidden"], a["idx"], a["topk"], a["W"], a["Eloc"], a["sq"],
                 a["ssf"], a["sids"], a["cap"], a["soff"], a["smap"], a["ws"], a["wsb"], None)

    assert call(hidden=200) == sat.FP8Q_ERR_SHAPE
    assert call(W=0) == sat.FP8Q_ERR_ARG and call(W=65) == sat.FP8Q_ERR_ARG and call(topk=65) == sat.FP8Q_ERR_ARG
    assert call(cap=127) == sat.FP8Q_ERR_ARG
    assert call(soff=None) == sat.FP8Q_ERR_NULL
    assert call(smap=None) == sat.FP8Q_ERR_NULL and call(xq=None) == sat.FP8Q_ERR_NULL
    assert call(xq=A + 4) == sat.FP8Q_ERR_ALIGN and call(ws=A + 8) == sat.FP8Q_ERR_ALIGN
    assert call(wsb=ws - 1) == sat.FP8Q_ERR_ARG
    assert call(tokens=1 << 40) == sat.FP8Q_ERR_SHAPE


def test_ep_recv_host_errors():
    f = sat.lib().fp8q_ep_recv_permute_fp8
    A = 0x10000
    segs = (sat.EpSource * 2)(sat.EpSource(A, A, A, 10), sat.EpSource(A, A, A, 6))
    R, K, Eloc, align = 16, 2, 4, 16
    ws = sat.fp8q_ep_recv_workspace_bytes(R, K, Eloc)
    need = R * K + Eloc * (align - 1)

    def call(segs=segs, n=2, hidden=256, topk=K, Eloc=Eloc, align=align, q=A, sf=A, cap=need, off=A, rmap=A,
             wsp=A, wsb=ws):
        return f(segs, n, hidden, topk, Eloc, align, q, sf, cap, off, rmap, wsp, wsb, None)

    assert call(hidden=100) == sat.FP8Q_ERR_SHAPE
    assert call(n=0) == sat.FP8Q_ERR_ARG and call(n=65) == sat.FP8Q_ERR_ARG and call(align=0) == sat.FP8Q_ERR_ARG
    assert call(segs=None) == sat.FP8Q_ERR_NULL
    assert call(cap=need - 1) == sat.FP8Q_ERR_ARG
    assert call(off=None) == sat.FP8Q_ERR_NULL and call(rmap=None) == sat.FP8Q_ERR_NULL
    assert call(wsb=ws - 1) == sat.FP8Q_ERR_ARG and call(wsp=A + 4) == sat.FP8Q_ERR_ALIGN
    bad = (sat.EpSource * 2)(sat.EpSource(A + 8, A, A, 10), sat.EpSource(A, A, A, 6))
    assert call(segs=bad) == sat.FP8Q_ERR_ALIGN
    nul = (sat.EpSource * 2)(sat.EpSource(A, A, None, 10), sat.EpSource(None, None, None, 0))
    assert call(segs=nul) == sat.FP8Q_ERR_NULL
    neg = (sat.EpSource * 2)(sat.EpSource(A, A, A, -1), sat.EpSource(A, A, A, 6))
    assert call(segs=neg) == sat.FP8Q_ERR_SHAPE
    huge = (sat.EpSource * 2)(sat.EpSource(A, A, A, 1 << 30), sat.EpSource(A, A, A, 1 << 30))
    assert call(segs=huge, cap=(1 << 31) - 1) == sat.FP8Q_ERR_SHAPE
