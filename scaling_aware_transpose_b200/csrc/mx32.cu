// mx32.cu — the path at MX granularity: 1x32 scaling tiles and the scaling-aware direct
// transpose on 32x32 blocks.
//
// Low-precision format table: MXFP8 keeps E4M3 elements with one power-of-two (E8M0)
// scale per 32 elements.  FP8-Flow-MoE review, 局限与 Future Work 2: the scaling-aware
// layout conversion carried over to MX formats.  The scale rule is the path's own
// (S = 2^ceil(log2(amax/448)), S = 1 for a zero tile); only the tile shrinks to 32.
//
// quantize_mx32_kernel: X [rows, cols] (cols % 32 == 0) is a flat sequence of 64-byte
// tiles.  A warp covers 16 consecutive tiles (1 KB of X) per slot: lane l loads 16-byte
// chunk l of the first and of the second 512 bytes, so each load instruction reads 512
// contiguous bytes; a tile's four chunks sit in four consecutive lanes, whose amax is
// reduced with two shuffles.  Each lane encodes its two chunks with their tiles' scales
// and stores 8 codes per chunk (256 contiguous bytes per store instruction).
//
// direct_transpose_mx32_kernel: the 128x128 block-per-CTA direct transpose with 16 MX
// blocks per CTA tile.  Each row's four scale bytes (one per 32-column group) move as one
// 32-bit word.  The four warps that load the scale words each reduce their own row group
// (one single-instruction warp max per column group, __reduce_max_sync) and publish one
// packed word before the kernel's one barrier; every thread then assembles the two words
// of maxima it needs with byte permutes.  The shift of a 16-byte row chunk uses its own
// 32x32 block's k; staging and the byte transpose (8 tokens x 8 channels per lane) are
// those of the 128 kernel.  A 2-D grid (column blocks x row blocks); the shift's form is chosen
// once per warp (shift_row16_warp).
#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr int kQThreads = 256;
constexpr int kQUnroll = 2;

// One 16-byte chunk (8 bf16) -> its maxabs as bf16 bits (sign clear).
__device__ __forceinline__ uint32_t chunk_maxabs(const uint4& v) {
  uint32_t m = maxabs_bf16x2(maxabs_bf16x2(v.x, v.y), maxabs_bf16x2(v.z, v.w));
  return maxabs_bf16x2(m, __byte_perm(m, 0u, 0x1032)) & 0x7FFFu;
}

__global__ void __launch_bounds__(kQThreads) quantize_mx32_kernel(const uint4* __restrict__ x, uint2* __restrict__ q,
                                                                   uint8_t* __restrict__ sf, int64_t n_tiles) {
  pdl_wait_for(x);
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * kQThreads + threadIdx.x) >> 5;
  uint4 v[kQUnroll][2];
  int64_t tile[kQUnroll][2];
#pragma unroll
  for (int u = 0; u < kQUnroll; ++u) {
    const int64_t base = (warp * kQUnroll + u) * 16;  // first tile of this slot
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tile[u][h] = base + 8 * h + (lane >> 2);
      v[u][h] = tile[u][h] < n_tiles ? ld_stream(x + base * 4 + 32 * h + lane) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int u = 0; u < kQUnroll; ++u) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t m = chunk_maxabs(v[u][h]);
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      if (tile[u][h] >= n_tiles) continue;
      const int e = bf16_tile_exponent(m);
      const float s = exp2_neg(e);
      const int64_t base = (warp * kQUnroll + u) * 16;
      q[base * 4 + 32 * h + lane] = make_uint2(encode4(v[u][h].x, v[u][h].y, s), encode4(v[u][h].z, v[u][h].w, s));
      if ((lane & 3) == 0) sf[tile[u][h]] = (uint8_t)(e + 127);
    }
  }
}

constexpr int kThreads = 256;
constexpr int kPasses = 4;

__device__ __forceinline__ int chunk_pos(int r, int c) { return c ^ ((r >> 3) & 7); }
__device__ __forceinline__ int byte_of(uint32_t w, int i) { return (int)((w >> (8 * i)) & 0xFFu); }

__global__ void __launch_bounds__(kThreads, 6) direct_transpose_mx32_kernel(const uint8_t* __restrict__ q,
                                                                          const uint8_t* __restrict__ sf, int64_t rows,
                                                                          int cols, uint8_t* __restrict__ qt,
                                                                          uint8_t* __restrict__ sft) {
  __shared__ __align__(16) uint8_t tile[128 * 128];
  __shared__ uint32_t e_row[128];  // 4 scale bytes of the row: column groups 0..3 of this tile
  __shared__ __align__(16) uint32_t smax_rg[4];  // row group rg: Smax byte of column groups 0..3
  pdl_wait_for(q, sf);
  pdl_trigger();
  const int tid = threadIdx.x;
  const int ncb = cols >> 7;
  const int ngr = cols >> 5;  // scale bytes per row
  const int64_t b = blockIdx.y;  // 2-D grid: column blocks x row blocks
  const int j = blockIdx.x;
  const int64_t r0 = b * 128;
  const int c0 = j * 128;
  const int sub = tid & 7, rsub = tid >> 3;
  const uint8_t* qb = q + r0 * cols + c0;
  uint4 v[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) v[p] = ld_g(reinterpret_cast<const uint4*>(qb + (p * 32 + rsub) * cols) + sub);
  // The row's 4 scale bytes (4-byte aligned: rows of cols/32 bytes, cols % 128 == 0).
  // Warp rg < 4 loads the 32 rows of row group rg and reduces their Smax per column group
  // with single-instruction warp reductions, one packed word per row group.
  if (tid < 128) {
    const uint32_t w = ld_g(reinterpret_cast<const uint32_t*>(sf + (r0 + tid) * ngr + (c0 >> 5)));
    e_row[tid] = w;
    uint32_t m = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) m |= __reduce_max_sync(0xFFFFFFFFu, (w >> (8 * c)) & 0xFFu) << (8 * c);
    if ((tid & 31) == 0) smax_rg[tid >> 5] = m;
  }
  __syncthreads();
  // The two words this thread needs, byte rg = Smax of (row group rg, column group): its
  // own chunks' column group, and the column group of SF^T channel c0 + tid.
  const int cg = sub >> 1;            // 32-column group of this thread's 16-byte chunks
  const int cg_t = (tid >> 5) & 3;    // column group of channel c0 + tid (SF^T word)
  const uint4 sm = *reinterpret_cast<const uint4*>(smax_rg);
  const uint32_t sel = (uint32_t)cg | (uint32_t)(cg + 4) << 4, sel_t = (uint32_t)cg_t | (uint32_t)(cg_t + 4) << 4;
  const uint32_t smax_mine = __byte_perm(__byte_perm(sm.x, sm.y, sel), __byte_perm(sm.z, sm.w, sel), 0x5410);
  const uint32_t smax_sft = __byte_perm(__byte_perm(sm.x, sm.y, sel_t), __byte_perm(sm.z, sm.w, sel_t), 0x5410);
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int rl = p * 32 + rsub;  // row group p
    uint32_t w[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
    shift_row16_warp(w, byte_of(smax_mine, p) - byte_of(e_row[rl], cg));
    *reinterpret_cast<uint4*>(tile + rl * 128 + 16 * chunk_pos(rl, sub)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();
  const int lane = tid & 31, wi = tid >> 5;
  const int t = lane >> 1, g = lane & 1;  // 8 tokens x 8 channels per lane
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rl = 8 * t + i;
    const uint2 w = *reinterpret_cast<const uint2*>(tile + rl * 128 + 16 * chunk_pos(rl, wi) + 8 * g);
    lo[i] = w.x;
    hi[i] = w.y;
  }
  uint32_t a[4][2], c[4][2];
#pragma unroll
  for (int qd = 0; qd < 2; ++qd) {
    transpose4x4(lo[4 * qd], lo[4 * qd + 1], lo[4 * qd + 2], lo[4 * qd + 3], a[0][qd], a[1][qd], a[2][qd], a[3][qd]);
    transpose4x4(hi[4 * qd], hi[4 * qd + 1], hi[4 * qd + 2], hi[4 * qd + 3], c[0][qd], c[1][qd], c[2][qd], c[3][qd]);
  }
  uint8_t* out = qt + (int64_t)(c0 + 16 * wi + 8 * g) * rows + r0 + 8 * t;
#pragma unroll
  for (int k = 0; k < 4; ++k, out += rows) *reinterpret_cast<uint2*>(out) = make_uint2(a[k][0], a[k][1]);
#pragma unroll
  for (int k = 0; k < 4; ++k, out += rows) *reinterpret_cast<uint2*>(out) = make_uint2(c[k][0], c[k][1]);
  if (tid < 128)  // SF^T [cols, rows/32]: channel c0 + tid, token groups 4b..4b+3, one word
    *reinterpret_cast<uint32_t*>(sft + (int64_t)(c0 + tid) * (rows >> 5) + (r0 >> 5)) = smax_sft;
}

}  // namespace

fp8q_status launch_quantize_mx32(const void* x, int64_t rows, int64_t cols, uint8_t* q, uint8_t* sf,
                                 cudaStream_t stream) {
  const int64_t n_tiles = rows * (cols / 32);
  if (n_tiles == 0) return FP8Q_OK;
  const int64_t tiles_per_block = (kQThreads / 32) * kQUnroll * 16;
  const int64_t blocks = (n_tiles + tiles_per_block - 1) / tiles_per_block;
  if (blocks > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  return launch_after(quantize_mx32_kernel, dim3((unsigned)blocks), kQThreads, 0, stream,
                      static_cast<const uint4*>(x), reinterpret_cast<uint2*>(q), sf, n_tiles) == cudaSuccess
             ? FP8Q_OK
             : FP8Q_ERR_CUDA;
}

fp8q_status launch_direct_transpose_mx32(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t cols, uint8_t* qt,
                                         uint8_t* sft, cudaStream_t stream) {
  const int64_t nblk = (rows / 128) * (cols / 128);
  if (nblk == 0) return FP8Q_OK;
  if (nblk > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  if (rows / 128 > 65535) return FP8Q_ERR_SHAPE;  // grid y limit (rows up to 8,388,480)
  return launch_after(direct_transpose_mx32_kernel, dim3((unsigned)(cols / 128), (unsigned)(rows / 128)), kThreads, 0,
                      stream, q, sf, rows, (int)cols, qt, sft) == cudaSuccess
             ? FP8Q_OK
             : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
