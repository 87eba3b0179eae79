// quantize_rowwise.cu — row-wise 1x128 E4M3 quantization with power-of-two scales.
//
// DeepSeek FP8 与 DeepGEMM §3: activations are scaled per token per 128 channels from
// the tile's online amax; FP8-Flow-MoE review 关键观察 2 / DeepSeek FP8 §8: the scale is
// restricted to a power of two, S = 2^ceil(log2(amax/448)), stored as a UE8M0 byte.
//
// HBM-bound streaming kernel (3 bytes moved per element plus 1 per 128).  Layout: a
// row-major [rows, cols] tensor with cols % 128 == 0 is a flat sequence of 128-element
// tiles, so the kernel runs over tiles: 8 lanes per tile, 16 bf16 (two 16-byte loads)
// per lane, four tiles per warp per slot, two slots per thread with every load issued
// before any use.  Instruction budget matters here (the integer ALU pipe is the first
// to saturate): the amax uses packed bf16x2 max-of-magnitudes, three shuffles, an
// exponent read straight off the BF16 bits, and packed f32x2 multiplies.
#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr int kQThreads = 256;
constexpr int kQUnroll = 2;        // tile slots per thread, all loads issued first
constexpr int kTilesPerWarp = 4;   // 8 lanes per tile, 16 elements per lane

// limit_rows (optional, device): only the first limit_rows[0] * tiles_per_row tiles are
// processed (the valid rows of a grouped buffer, known only on the device).
// Lane l of a warp serves tile 4*slot + l/8; its 16 elements are 8 from each half of
// the tile (16-byte chunk l%8 of bytes 0..127 and of bytes 128..255), so each load
// instruction reads whole 128-byte lines and each store writes 64 contiguous bytes.
__global__ void __launch_bounds__(kQThreads) quantize_tiles_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
                                                                    uint8_t* __restrict__ sf, int64_t n_tiles,
                                                                    const int32_t* __restrict__ limit_rows,
                                                                    int64_t tiles_per_row) {
  pdl_wait_for(x, limit_rows);
  pdl_trigger();
  if (limit_rows != nullptr) {
    const int64_t lim = (int64_t)ld_g(limit_rows);
    n_tiles = lim <= 0 ? 0 : min(n_tiles, lim * tiles_per_row);
  }
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const int64_t warp = ((int64_t)blockIdx.x * kQThreads + threadIdx.x) >> 5;
  int64_t tile[kQUnroll];
  uint4 v0[kQUnroll], v1[kQUnroll];
#pragma unroll
  for (int u = 0; u < kQUnroll; ++u) {
    tile[u] = (warp * kQUnroll + u) * kTilesPerWarp + (lane >> 3);
    if (tile[u] < n_tiles) {
      v0[u] = ld_stream(x + tile[u] * 16 + sub);
      v1[u] = ld_stream(x + tile[u] * 16 + 8 + sub);
    } else {
      v0[u] = v1[u] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int u = 0; u < kQUnroll; ++u) {
    uint32_t m = maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(v0[u].x, v0[u].y), maxabs_bf16x2(v0[u].z, v0[u].w)),
                               maxabs_bf16x2(maxabs_bf16x2(v1[u].x, v1[u].y), maxabs_bf16x2(v1[u].z, v1[u].w)));
    m = maxabs_bf16x2(m, __byte_perm(m, 0u, 0x1032)) & 0x7FFFu;
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int e = bf16_tile_exponent(m);
    const float s = exp2_neg(e);
    if (tile[u] < n_tiles) {
      q[tile[u] * 16 + sub] = make_uint2(encode4(v0[u].x, v0[u].y, s), encode4(v0[u].z, v0[u].w, s));
      q[tile[u] * 16 + 8 + sub] = make_uint2(encode4(v1[u].x, v1[u].y, s), encode4(v1[u].z, v1[u].w, s));
      if (sub == 0) sf[tile[u]] = (uint8_t)(e + 127);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_tiles(const void* x, int64_t n_tiles, uint8_t* q, uint8_t* sf, cudaStream_t stream,
                                  const int32_t* limit_rows, int64_t tiles_per_row) {
  if (n_tiles <= 0) return cudaSuccess;
  const int64_t tiles_per_block = (kQThreads / 32) * kQUnroll * kTilesPerWarp;
  const int64_t blocks = (n_tiles + tiles_per_block - 1) / tiles_per_block;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  return launch_after(quantize_tiles_kernel, dim3((unsigned)blocks), kQThreads, 0, stream,
                      static_cast<const uint4*>(x), reinterpret_cast<uint2*>(q), sf, n_tiles, limit_rows,
                      tiles_per_row);
}

}  // namespace fp8q
