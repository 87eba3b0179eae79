"""The library under CUDA graph capture: every entry point takes caller-owned buffers and
a stream and neither allocates nor synchronizes, so a whole MoE data-movement step -
quantize, direct transpose, permute+pad+quantize (workspace allocated up front), grouped
direct transpose, unpermute+unpad - can be captured once and replayed.  Replays on new input
bytes must give exactly what eager calls give."""
import numpy as np
import pytest
import torch

import scaling_aware_transpose_b200 as sat
from scaling_aware_transpose_b200 import synthetic
from gpu_helpers import dev, device_status_ok

pytestmark = pytest.mark.gpu

T, H, E, K, ALIGN = 512, 1024, 8, 4, 128


def make_buffers():
    max_rows = sat.permute_max_rows(T, K, E, ALIGN)
    b = {
        "x": torch.empty((T, H), dtype=torch.bfloat16, device="cuda"),
        "idx": torch.empty((T, K), dtype=torch.int32, device="cuda"),
        "w": torch.empty((T, K), dtype=torch.float32, device="cuda"),
        "q": torch.empty((T, H), dtype=torch.uint8, device="cuda"),
        "sf": torch.empty((T, H // 128), dtype=torch.uint8, device="cuda"),
        "qt": torch.empty((H, T), dtype=torch.uint8, device="cuda"),
        "sft": torch.empty((H, T // 128), dtype=torch.uint8, device="cuda"),
        "pq": torch.zeros((max_rows, H), dtype=torch.uint8, device="cuda"),
        "psf": torch.zeros((max_rows, H // 128), dtype=torch.uint8, device="cuda"),
        "off": torch.empty((E + 1,), dtype=torch.int32, device="cuda"),
        "rmap": torch.empty((T * K,), dtype=torch.int32, device="cuda"),
        "gqt": torch.zeros((max_rows * H,), dtype=torch.uint8, device="cuda"),
        "gsft": torch.zeros((max_rows * H // 128,), dtype=torch.uint8, device="cuda"),
        "comb": torch.empty((T, H), dtype=torch.bfloat16, device="cuda"),
        "ws": torch.empty((sat.fp8q_permute_workspace_bytes(T, K, E),), dtype=torch.uint8, device="cuda"),
    }
    return max_rows, b


def step(max_rows, b, stream):
    sp = stream.cuda_stream
    sat.fp8q_quantize_rowwise(b["x"], T, H, b["q"], b["sf"], sp)
    sat.fp8q_direct_transpose(b["q"], b["sf"], T, H, None, 1, b["qt"], b["sft"], sp)
    sat.fp8q_permute_pad_quant(b["x"], T, H, b["idx"], K, E, ALIGN, b["pq"], b["psf"], max_rows, b["off"], b["rmap"],
                               b["ws"], b["ws"].numel(), sp)
    sat.fp8q_direct_transpose(b["pq"], b["psf"], max_rows, H, b["off"], E, b["gqt"], b["gsft"], sp)
    sat.fp8q_unpermute_unpad(b["pq"], b["psf"], max_rows, H, b["rmap"], b["w"], T, K, b["comb"], sp)


def load_inputs(b, seed):
    d = synthetic.moe(tokens=T, hidden=H, num_experts=E, topk=K, seed=seed)
    w = np.random.default_rng(seed).dirichlet(np.ones(K), size=T).astype(np.float32)
    b["x"].copy_(dev(d["x"]))
    b["idx"].copy_(dev(d["topk_idx"]))
    b["w"].copy_(torch.from_numpy(w).cuda())


def snapshot(b, max_rows):
    n = int(b["off"][-1].item())
    return [b["q"].clone(), b["sf"].clone(), b["qt"].clone(), b["sft"].clone(), b["off"].clone(), b["rmap"].clone(),
            b["pq"][:n].clone(), b["psf"][:n].clone(), b["gqt"][: H * n].clone(), b["gsft"][: H * n // 128].clone(),
            b["comb"].clone()]


def test_graph_replay_matches_eager():
    max_rows, b = make_buffers()
    s = torch.cuda.Stream()
    load_inputs(b, seed=0)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        step(max_rows, b, s)  # warm-up outside capture: per-device set-up happens here
    s.synchronize()
    device_status_ok()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(max_rows, b, s)
    for seed in (1, 2, 3):
        load_inputs(b, seed)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        got = snapshot(b, max_rows)
        device_status_ok()
        with torch.cuda.stream(s):
            step(max_rows, b, s)  # eager, same buffers
        s.synchronize()
        want = snapshot(b, max_rows)
        for i, (a, c) in enumerate(zip(got, want)):
            assert torch.equal(a, c), f"replay output {i} differs from eager (seed {seed})"
    del g
