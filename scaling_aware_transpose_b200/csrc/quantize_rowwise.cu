// quantize_rowwise.cu — row-wise 1x128 E4M3 quantization with power-of-two scales.
//
// DeepSeek FP8 与 DeepGEMM §3: activations are scaled per token per 128 channels from
// the tile's online amax; FP8-Flow-MoE review 关键观察 2 / DeepSeek FP8 §8: the scale is
// restricted to a power of two, S = 2^ceil(log2(amax/448)), stored as a UE8M0 byte.
//
// HBM-bound streaming kernel (3 bytes moved per element plus 1 per 128).  Layout: a
// row-major [rows, cols] tensor with cols % 128 == 0 is a flat sequence of 128-element
// tiles, so the kernel runs over tiles: 16 lanes per tile, 8 bf16 (one 16-byte load)
// per lane, two tiles per warp per slot, UNROLL slots per thread with every load issued
// before any use.  Loads are coalesced 512-byte warp segments, stores 256-byte ones.
#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr int kQThreads = 256;
constexpr int kQUnroll = 4;

// Max of the 8 bf16 magnitudes in `v`, as the fp32 bit pattern (non-negative floats
// order like their bit patterns, so an unsigned 16-bit max is a float max).
__device__ __forceinline__ uint32_t absmax8_bits(const uint4& v) {
  const uint32_t m0 = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  const uint32_t m1 = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
  const uint32_t m = __vmaxu2(m0, m1);
  return max(m & 0xFFFFu, m >> 16) << 16;
}

__device__ __forceinline__ uint32_t encode4(uint32_t a, uint32_t b, float s) {
  // a, b: two bf16x2 words (elements 0,1 and 2,3) -> 4 codes, element 0 in the low byte
  const float f0 = __uint_as_float(a << 16) * s, f1 = __uint_as_float(a & 0xFFFF0000u) * s;
  const float f2 = __uint_as_float(b << 16) * s, f3 = __uint_as_float(b & 0xFFFF0000u) * s;
  return cvt_e4m3x2_f32(f0, f1) | (cvt_e4m3x2_f32(f2, f3) << 16);
}

// limit_rows (optional, device): only the first limit_rows[0] * tiles_per_row tiles are
// processed (the valid rows of a grouped buffer, known only on the device).
__global__ void __launch_bounds__(kQThreads) quantize_tiles_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
                                                                    uint8_t* __restrict__ sf, int64_t n_tiles,
                                                                    const int32_t* __restrict__ limit_rows,
                                                                    int64_t tiles_per_row) {
  if (limit_rows != nullptr) {
    const int64_t lim = (int64_t)__ldg(limit_rows);
    n_tiles = lim <= 0 ? 0 : min(n_tiles, lim * tiles_per_row);
  }
  const int lane = threadIdx.x & 31;
  const int sub = lane & 15;  // 16-byte chunk within the tile
  const int64_t warp = ((int64_t)blockIdx.x * kQThreads + threadIdx.x) >> 5;
  int64_t tile[kQUnroll];
  uint4 v[kQUnroll];
#pragma unroll
  for (int u = 0; u < kQUnroll; ++u) {
    tile[u] = (warp * kQUnroll + u) * 2 + (lane >> 4);
    v[u] = tile[u] < n_tiles ? ld_stream(x + tile[u] * 16 + sub) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < kQUnroll; ++u) {
    uint32_t m = absmax8_bits(v[u]);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int e = tile_exponent(__uint_as_float(m));
    const float s = exp2_neg(e);  // x * 2^-e is exact (or rounds to +-0 in E4M3 anyway)
    if (tile[u] < n_tiles) {
      uint2 out;
      out.x = encode4(v[u].x, v[u].y, s);
      out.y = encode4(v[u].z, v[u].w, s);
      q[tile[u] * 16 + sub] = out;
      if (sub == 0) sf[tile[u]] = (uint8_t)(e + 127);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_tiles(const void* x, int64_t n_tiles, uint8_t* q, uint8_t* sf, cudaStream_t stream,
                                  const int32_t* limit_rows, int64_t tiles_per_row) {
  if (n_tiles <= 0) return cudaSuccess;
  const int64_t tiles_per_block = (kQThreads / 32) * kQUnroll * 2;
  const int64_t blocks = (n_tiles + tiles_per_block - 1) / tiles_per_block;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  quantize_tiles_kernel<<<(unsigned)blocks, kQThreads, 0, stream>>>(static_cast<const uint4*>(x),
                                                                      reinterpret_cast<uint2*>(q), sf, n_tiles,
                                                                      limit_rows, tiles_per_row);
  return cudaGetLastError();
}

}  // namespace fp8q
