"""Exhaustive cross-checks of the device arithmetic every kernel relies on, against the
CPU oracle, over every fp32 bit pattern (non-finite inputs excluded): the fp32 -> E4M3
conversion (round to nearest even, saturating at 448) and the SwiGLU spec's exp; plus
the SwiGLU spec itself (y = silu(g) * u, before quantization) on a large random sample
of finite fp32 pairs and on special values; and silu of every finite BF16 value through
the fused kernel's own table path.  Inputs are generated from bit indices on
each side, so nothing computed by one side feeds the other."""
import numpy as np
import pytest
import torch

import oracle
import scaling_aware_transpose_b200 as sat

pytestmark = pytest.mark.gpu

CHUNK = 1 << 28


def finite_count(chunk: int) -> int:
    """Chunk c covers bit patterns c*2^28 .. ; exponent field 0xFF (Inf/NaN) occurs only
    where bits 28..30 are all ones (chunks 7 and 15), in the chunk's last 2^23 patterns."""
    return CHUNK - (1 << 23) if (chunk & 7) == 7 else CHUNK


def test_encoder_matches_oracle_on_every_finite_fp32():
    out = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
    for c in range(16):
        sat.fp8q_debug_e4m3_encode_range(c << 28, CHUNK, out)
        n = finite_count(c)
        got = out[:n].cpu().numpy()
        want = oracle.e4m3_encode_f32_range(c << 28, n)
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (f"chunk {c}: {bad.size} codes differ, first bits "
                               f"{hex((c << 28) + int(bad[0]))}: got {hex(got[bad[0]])} want {hex(want[bad[0]])}")


def test_exp_spec_matches_oracle_on_every_finite_fp32():
    out = torch.empty(CHUNK, dtype=torch.float32, device="cuda")
    for c in range(16):
        sat.fp8q_debug_exp_spec_range(c << 28, CHUNK, out)
        n = finite_count(c)
        got = out[:n].cpu().numpy().view(np.uint32)
        want = oracle.exp_spec_f32_range(c << 28, n).view(np.uint32)
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (f"chunk {c}: {bad.size} values differ, first bits {hex((c << 28) + int(bad[0]))}: "
                               f"got {hex(got[bad[0]])} want {hex(want[bad[0]])}")


def test_swiglu_spec_matches_oracle_on_random_and_special_pairs():
    rng = np.random.default_rng(2024)
    n = 1 << 26
    gb = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    gb[(gb & 0x7F800000) == 0x7F800000] &= 0xBFFFFFFF  # keep every pattern finite
    g = gb.view(np.float32)
    g[: n // 2] = rng.standard_normal(n // 2).astype(np.float32) * 8     # the range activations live in
    u = rng.standard_normal(n).astype(np.float32) * np.exp2(rng.integers(-20, 20, size=n)).astype(np.float32)
    specials = np.array([0.0, -0.0, 88.0, 89.0, 89.0001, 103.9, 104.0, 104.1, -88.0, -89.0, -89.0001, -103.9, -104.0,
                         -104.1, 1e-30, -1e-30, 3.4e38, -3.4e38, 1.4e-45, -1.4e-45], np.float32)
    g[: specials.size] = specials
    u[: specials.size] = 1.0
    y = torch.empty(n, dtype=torch.float32, device="cuda")
    sat.fp8q_debug_swiglu_spec(torch.from_numpy(g).cuda(), torch.from_numpy(u).cuda(), n, y)
    got = y.cpu().numpy().view(np.uint32)
    want = oracle.swiglu(g, u).view(np.uint32)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (f"{bad.size} of {n} differ; first g={g[bad[0]]!r} u={u[bad[0]]!r}: "
                           f"got {hex(got[bad[0]])} want {hex(want[bad[0]])}")


@pytest.mark.parametrize("order", ["sorted", "shuffled", "ragged"])
def test_silu_table_path_matches_oracle_on_every_finite_bf16(order):
    """The fused SwiGLU kernel tabulates silu for BF16 inputs and uses closed forms outside
    the table's range; every finite BF16 gate value must give the spec's fp32 silu(g).
    Sorted, the range edges fall inside warps; shuffled, most warps that see an input
    outside the range see only one; ragged leaves the last warp partly empty.  The hook
    fills its table the way the fused kernel does: the first call on the device evaluates
    it and publishes it, later calls copy the published one; two calls cover both."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    bits = bits[(bits & 0x7F80) != 0x7F80].astype(np.uint16)  # finite only
    if order == "shuffled":
        bits = np.random.default_rng(7).permutation(bits)
    if order == "ragged":
        bits = bits[: 2 * 1000 + 2 * 17]
    g = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    gf = (bits.astype(np.uint32) << 16).view(np.float32)
    want = oracle.swiglu(gf, np.ones_like(gf)).view(np.uint32)   # silu(g) * 1
    for call in range(2):
        y = torch.full((bits.size,), float("nan"), dtype=torch.float32, device="cuda")
        sat.fp8q_debug_silu_bf16(g, bits.size, y)
        got = y.cpu().numpy().view(np.uint32)
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (f"call {call}: {bad.size} of {bits.size} differ; first g bits "
                               f"{hex(int(bits[bad[0]]))}: got {hex(got[bad[0]])} want {hex(want[bad[0]])}")
