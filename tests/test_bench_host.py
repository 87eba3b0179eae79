"""Host logic of bench.py without a GPU: byte accounting, roofline arithmetic, the
traffic lookup, the max-over-ranks reduction on a 2-rank gloo group, and the reference
arm's JSON line."""
import json
import multiprocessing as mp
import os
import re
import socket

import pytest

import bench


def test_algorithmic_bytes_match_the_definition():
    n = 8192 * 7168
    assert bench.BYTES_QUANT == 176_619_520 == 3 * n + n // 128
    assert bench.BYTES_DIRECT == 118_358_016 == 2 * n + 2 * (n // 128)


def test_roofline_fields():
    r = bench.roofline(bench.BYTES_QUANT, 30e-6, 6555.5, "measured", None)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] is None
    assert abs(r["achieved"] - bench.BYTES_QUANT / 30e-6 / 1e9) < 0.1
    assert abs(r["frac"] - r["achieved"] / 6555.5) < 1e-3


def test_traffic_requires_matching_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    csrc = tmp_path / "scaling_aware_transpose_b200" / "csrc"
    os.makedirs(csrc)
    (csrc / "quantize_rowwise.cu").write_text("a")
    (csrc / "common.cuh").write_text("b")
    digest = bench.source_digest(bench.kernel_sources("quantize"))
    p = tmp_path / "profiles" / "quantize_rowwise_dense_8192x7168.md"
    p.write_text(f"- dram_bytes_per_launch: 12345\n- source_sha256: {digest}\n")
    assert bench.profiled_traffic("quantize") == 12345
    (csrc / "quantize_rowwise.cu").write_text("changed")
    assert bench.profiled_traffic("quantize") is None


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        v = bench.reduce_max(float(rank * 10 + 1), dist, "cpu")
        dist.barrier()
        q.put((rank, v))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 11.0, 1: 11.0}


def test_reduce_max_without_group_is_identity():
    assert bench.reduce_max(3.5) == 3.5


def test_reference_arm_line(capsys):
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-rows", "256"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["metric"] == bench.METRIC


def test_reference_arm_other_ranks_do_nothing(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1"]) == 0
    assert capsys.readouterr().out == ""


def test_every_profile_choice_names_existing_sources():
    """The --profile kind in each summary's command maps to kernel sources that exist, so
    the summary's source hash can always be recomputed."""
    d = os.path.join(bench.ROOT, "profiles")
    kinds = set()
    for name in sorted(os.listdir(d)):
        if name.startswith("launches_"):
            continue
        m = re.search(r"--profile (\w+)", open(os.path.join(d, name)).read())
        assert m, name
        kinds.add(m.group(1))
    assert {"permute_e512", "permute_e4096", "unpermute_fp8_k", "ep_pack", "ep_recv"} <= kinds
    for kind in kinds:
        paths = bench.kernel_sources(kind)
        assert paths and all(os.path.exists(p) for p in paths), kind
    assert bench.kernel_sources("unpermute_fp8") == bench.kernel_sources("unpermute")


def test_profile_summaries_carry_command_and_hash():
    """Every committed ncu summary names the command that made it and a source hash."""
    d = os.path.join(bench.ROOT, "profiles")
    for name in sorted(os.listdir(d)):
        txt = open(os.path.join(d, name)).read()
        assert "--clock-control none" in txt, name
        if name.startswith("launches_"):
            continue
        assert "source_sha256:" in txt and "dram_bytes_per_launch:" in txt, name
