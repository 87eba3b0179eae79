"""Pins of the oracle's expert-parallel FP8 dispatch (send-side pack, receive-side
permute), independent of the functions themselves.

FP8-Flow-MoE review, 核心方法 and Table 1: the dispatch moves row-wise FP8 codes with
their scale metadata; DeepSeek FP8 §5.6: each rank's experts read contiguous row
groups.  The strongest pin is a composition identity: exchanging the packed rows among
W simulated ranks and permuting on receive must give, on rank d, exactly the slice of
the single-device FP8 permute (itself pinned in test_oracle_swiglu_permute.py) that
covers rank d's experts - rows, padding, offsets and row ids.
"""
import numpy as np
import pytest

import oracle
from scaling_aware_transpose_b200 import synthetic


def _tokens(T, H, seed):
    q, sf = oracle.quantize_rowwise(synthetic.scaled_normal(T, H, seed=seed, row_sigma=1.5))
    return q, sf


def _exchange(packs, W):
    """What the all-to-all delivers to each rank: rank d receives, from every source s
    in rank order, the rows source s packed for d."""
    recv = []
    for d in range(W):
        parts = [(p[0][p[3][d]:p[3][d + 1]], p[1][p[3][d]:p[3][d + 1]], p[2][p[3][d]:p[3][d + 1]]) for p in packs]
        recv.append(tuple(np.concatenate([x[i] for x in parts]) for i in range(3)))
    return recv


def test_pack_brute_force_tiny():
    T, H, K, W, Eloc = 9, 128, 2, 3, 2
    rng = np.random.default_rng(4)
    idx = rng.integers(0, W * Eloc, (T, K)).astype(np.int32)
    idx[3] = [1, 1]          # duplicate expert within a token: one row, two slots
    q, sf = _tokens(T, H, 2)
    sq, ssf, sids, soff, smap = oracle.ep_dispatch_pack(q, sf, idx, W, Eloc)
    row = 0
    for d in range(W):
        assert soff[d] == row
        for t in range(T):
            dests = {int(e) // Eloc for e in idx[t]}
            if d not in dests:
                assert smap[t, d] == -1
                continue
            assert smap[t, d] == row
            assert np.array_equal(sq[row], q[t]) and np.array_equal(ssf[row], sf[t])
            want = [int(e) - d * Eloc if int(e) // Eloc == d else -1 for e in idx[t]]
            assert sids[row].tolist() == want
            row += 1
    assert soff[W] == row == sq.shape[0]


@pytest.mark.parametrize("W,T,H,K,Eloc,align", [(4, 64, 256, 3, 3, 16), (2, 100, 128, 8, 16, 128),
                                                 (8, 40, 384, 4, 1, 1), (3, 0, 128, 2, 2, 16)])
def test_exchange_then_receive_permute_is_the_global_permute_slice(W, T, H, K, Eloc, align):
    rng = np.random.default_rng(W * 100 + T)
    E = W * Eloc
    src = [_tokens(T, H, seed=s + 10) for s in range(W)]
    idx = [synthetic.zipf_topk(T, E, min(K, E), rng) if T else np.zeros((0, min(K, E)), np.int32) for _ in range(W)]
    K = idx[0].shape[1]
    packs = [oracle.ep_dispatch_pack(src[s][0], src[s][1], idx[s], W, Eloc) for s in range(W)]
    recv = _exchange(packs, W)
    gq, gsf, goff, grmap = oracle.permute_pad_fp8(np.concatenate([s[0] for s in src]),
                                                  np.concatenate([s[1] for s in src]),
                                                  np.concatenate(idx), E, align)
    grmap = grmap.reshape(W, T, K)
    for d in range(W):
        rq, rsf, rids = recv[d]
        q, sf, off, rmap = oracle.ep_recv_permute(rq, rsf, rids, Eloc, align)
        base = int(goff[d * Eloc])
        assert np.array_equal(off, goff[d * Eloc:(d + 1) * Eloc + 1] - base)
        n = int(off[-1])
        assert np.array_equal(q[:n], gq[base:base + n]) and np.array_equal(sf[:n], gsf[base:base + n])
        # row ids: received row -> (source, token) through the source's send map
        rmap = rmap.reshape(-1, K)
        r = 0
        for s in range(W):
            toks = np.nonzero(packs[s][4][:, d] >= 0)[0]
            for t in toks:
                for k in range(K):
                    if rids[r, k] < 0:
                        assert rmap[r, k] == -1
                    else:
                        assert rmap[r, k] + base == grmap[s, t, k]
                r += 1
        assert r == rq.shape[0]


def test_one_rank_is_the_fp8_permute():
    T, H, K, E, align = 200, 256, 4, 8, 16
    rng = np.random.default_rng(1)
    idx = synthetic.zipf_topk(T, E, K, rng)
    q, sf = _tokens(T, H, 5)
    sq, ssf, sids, soff, smap = oracle.ep_dispatch_pack(q, sf, idx, 1, E)
    assert np.array_equal(sq, q) and np.array_equal(sids, idx) and np.array_equal(smap[:, 0], np.arange(T))
    a = oracle.ep_recv_permute(sq, ssf, sids, E, align)
    b = oracle.permute_pad_fp8(q, sf, idx, E, align)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_every_slot_is_delivered_exactly_once():
    W, T, H, K, Eloc = 4, 300, 128, 6, 5
    rng = np.random.default_rng(9)
    idx = synthetic.zipf_topk(T, W * Eloc, K, rng)
    q, sf = _tokens(T, H, 3)
    sq, ssf, sids, soff, smap = oracle.ep_dispatch_pack(q, sf, idx, W, Eloc)
    assert np.all(np.diff(soff) >= 0)
    assert soff[-1] == sum(len({int(e) // Eloc for e in idx[t]}) for t in range(T))
    assert int((sids >= 0).sum()) == T * K
    for d in range(W):
        seg = sids[soff[d]:soff[d + 1]]
        assert np.all((seg == -1) | ((seg >= 0) & (seg < Eloc)))
        assert np.all((seg >= 0).any(axis=1))   # every sent row has a slot for its rank


def test_invalid_ids_are_rejected():
    q, sf = _tokens(4, 128, 0)
    with pytest.raises(oracle.OracleError):
        oracle.ep_dispatch_pack(q, sf, np.array([[0], [1], [8], [2]], np.int32), 2, 4)
    with pytest.raises(oracle.OracleError):
        oracle.ep_recv_permute(q, sf, np.array([[0], [-2], [1], [2]], np.int32), 4, 16)
