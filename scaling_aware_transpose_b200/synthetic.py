"""Seeded synthetic inputs for the FP8 quantize / direct-transpose path.

This module is the single source of input bytes for both the CUDA library and the
CPU oracle, so that the two see identical data.  It holds none of the method's
arithmetic: it only draws random numbers and rounds them to BF16.

Draws come from numpy's PCG64 (``default_rng(seed)``) in float32, in the order
written below; BF16 rounding is round-to-nearest-even (``torch.Tensor.to``).  Arrays
are returned as ``uint16`` BF16 bit patterns (use :func:`to_torch_bf16` for a torch
view).

The workloads stand in for the "DeepSeek V2-lite/V2/V3 representative shapes" of the
FP8-Flow-MoE review (section 实验与结果, micro-benchmarks), whose exact shapes the
pages do not print.
"""
from __future__ import annotations

import numpy as np
import torch


def _bf16_bits(a_f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_torch_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def scaled_normal(rows: int, cols: int, seed: int = 0, row_sigma: float = 1.0) -> np.ndarray:
    """x = z * f_t, z ~ N(0,1) [rows, cols], f_t ~ lognormal(0, row_sigma) per row."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((rows, cols), dtype=np.float32)
    f = rng.lognormal(0.0, row_sigma, size=rows).astype(np.float32)
    z *= f[:, None]
    return _bf16_bits(z)


def tiny(seed: int = 0, rows: int = 256, cols: int = 512) -> dict:
    """X bf16 [256, 512], x ~ N(0,1) times a lognormal(0, 2) factor per row."""
    return {"x": scaled_normal(rows, cols, seed, 2.0)}


def dense(seed: int = 0, rows: int = 8192, cols: int = 7168, outlier_frac: float = 0.001,
          outlier_gain: float = 100.0) -> dict:
    """X bf16 [8192, 7168]: N(0,1) times a lognormal(0, 1.5) factor per row; then
    round(0.001*cols) channels, drawn without replacement, scaled by 100."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((rows, cols), dtype=np.float32)
    f = rng.lognormal(0.0, 1.5, size=rows).astype(np.float32)
    n_out = int(round(outlier_frac * cols))
    ch = rng.choice(cols, size=n_out, replace=False) if n_out else np.zeros(0, np.int64)
    z *= f[:, None]
    z[:, ch] *= np.float32(outlier_gain)
    return {"x": _bf16_bits(z), "outlier_channels": np.sort(ch)}


def zipf_topk(tokens: int, num_experts: int, topk: int, rng: np.random.Generator,
              alpha: float = 1.1) -> np.ndarray:
    """Top-k routing with Zipf(alpha) expert popularity: p_i ~ i^-alpha (i = 1..E);
    each token takes k distinct experts by Gumbel-top-k on log p_i, highest score
    first."""
    logp = -alpha * np.log(np.arange(1, num_experts + 1, dtype=np.float64))
    scores = logp[None, :] + rng.gumbel(size=(tokens, num_experts))
    idx = np.argsort(-scores, axis=1, kind="stable")[:, :topk]
    return np.ascontiguousarray(idx.astype(np.int32))


def moe(seed: int = 0, tokens: int = 16384, hidden: int = 7168, num_experts: int = 32,
        topk: int = 8) -> dict:
    """MoE expert input: X bf16 [16384, 7168] ~ N(0,1) and top-8 routing over 32
    experts with Zipf(1.1) popularity."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((tokens, hidden), dtype=np.float32)
    idx = zipf_topk(tokens, num_experts, topk, rng)
    return {"x": _bf16_bits(x), "topk_idx": idx, "num_experts": num_experts}


def moe_combine(seed: int = 0, tokens: int = 16384, hidden: int = 7168, rows: int = 133120,
                topk: int = 8) -> dict:
    """Combine-side inputs of the MoE workload: expert outputs Y bf16 [rows, hidden] ~
    N(0,1) (the permuted, padded buffer after the expert GEMMs) and routing weights
    fp32 [tokens, topk] drawn from a flat Dirichlet (positive, each token's weights sum
    to 1, like normalised router probabilities)."""
    rng = np.random.default_rng(seed + 1000)
    y = rng.standard_normal((rows, hidden), dtype=np.float32)
    w = rng.dirichlet(np.ones(topk), size=tokens).astype(np.float32)
    return {"y": _bf16_bits(y), "weights": np.ascontiguousarray(w)}


def swiglu(seed: int = 0, rows: int = 32768, cols: int = 2048) -> dict:
    """gate, up bf16 [32768, 2048], independent N(0,1), both multiplied by one
    lognormal(0, 1) factor per row (reading: "N(0,1) times per-row lognormal(0,1)"
    is taken as one factor per row shared by gate and up)."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((rows, cols), dtype=np.float32)
    u = rng.standard_normal((rows, cols), dtype=np.float32)
    f = rng.lognormal(0.0, 1.0, size=rows).astype(np.float32)
    g *= f[:, None]
    u *= f[:, None]
    return {"gate": _bf16_bits(g), "up": _bf16_bits(u)}



def swiglu_wide(seed: int = 0, rows: int = 4096, cols: int = 2048) -> dict:
    """Gate values over every BF16 binade that keeps y finite: each 1x128 gate tile draws a
    binade B uniform in [-134, 118], each element B + {0, 1, 2} (clipped below at -133;
    binades below -126 are BF16 subnormals), a uniform 7-bit mantissa and a random sign;
    up ~ N(0, 1), so |y| < 2^121 * 8.  This covers tiny, table-range and huge gates in the
    same tensor, one scale per tile."""
    rng = np.random.default_rng(seed)
    e = rng.integers(-134, 119, size=(rows, cols // 128, 1)) + rng.integers(0, 3, size=(rows, cols // 128, 128))
    e = np.maximum(e, -133)
    mant = rng.integers(0, 128, size=e.shape)
    bits = np.where(e >= -126, ((e + 127) << 7) | mant, mant >> np.clip(-126 - e, 0, 7)).astype(np.uint16)
    bits |= (rng.integers(0, 2, size=e.shape) << 15).astype(np.uint16)
    u = rng.standard_normal((rows, cols), dtype=np.float32)
    return {"gate": bits.reshape(rows, cols), "up": _bf16_bits(u)}

def stress(seed: int = 0, rows: int = 65536, cols: int = 7168, lo: float = -20.0, hi: float = 12.0,
           zero_frac: float = 0.01) -> dict:
    """Range stress: each 1x128 tile is z / max|z| * 2^u with u ~ U(lo, hi) per tile
    (so the tile amax is 2^u before BF16 rounding), and a Bernoulli(zero_frac) share
    of tiles set to +0."""
    rng = np.random.default_rng(seed)
    nt = cols // 128
    u = rng.uniform(lo, hi, size=(rows, nt)).astype(np.float32)
    zero = rng.random(size=(rows, nt)) < zero_frac
    out = np.empty((rows, cols), np.uint16)
    chunk = 4096
    for r0 in range(0, rows, chunk):  # chunked to bound the float32 working set
        r1 = min(rows, r0 + chunk)
        z = rng.standard_normal((r1 - r0, nt, 128), dtype=np.float32)
        z /= np.abs(z).max(axis=2, keepdims=True)
        z *= np.exp2(u[r0:r1]).astype(np.float32)[:, :, None]
        z[zero[r0:r1]] = 0.0
        out[r0:r1] = _bf16_bits(z.reshape(r1 - r0, cols))
    return {"x": out, "zero_tiles": zero}


CONFIGS = {
    "tiny": tiny,
    "dense": dense,
    "moe": moe,
    "swiglu": swiglu,
    "stress": stress,
}


def device_normal(rows: int, cols: int, seed: int, device, row_sigma: float = 1.0):
    """Large inputs made on the device (too big to draw on the host in a test): a seeded
    torch generator gives z ~ N(0,1) times a lognormal(0, row_sigma) factor per row, as
    BF16.  Both sides use the same bytes: the GPU reads the tensor, the oracle its rows
    copied back."""
    import torch
    g = torch.Generator(device=device).manual_seed(seed)
    z = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    f = torch.exp(row_sigma * torch.randn((rows, 1), generator=g, device=device, dtype=torch.float32))
    return (z * f).to(torch.bfloat16)
