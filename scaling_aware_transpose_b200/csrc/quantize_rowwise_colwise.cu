// quantize_rowwise_colwise.cu — single-pass quantization of a BF16 tensor into both FP8
// layouts: the row-wise (Q, SF) that Fprop/Dgrad consume and the column-wise (Q^T, SF^T)
// that Wgrad consumes (DeepSeek FP8 与 DeepGEMM §1, §3).
//
// The column-wise result is, by definition, the scaling-aware direct transpose of the
// row-wise one (FP8-Flow-MoE review, 核心方法): per 128x128 block, Smax = the largest
// row-tile scale, and each row's codes are shifted by k = log2(Smax / S_row) with
// round-to-nearest-even.  Computing both from one read of X saves the direct transpose's
// re-read of Q: 4 bytes per element move instead of 5.
//
// One CTA per 128x128 block (column blocks fastest), 256 threads, four CTAs per SM:
//   1. every thread loads its share of the block (16 bf16 of one row tile per pass, four
//      passes) before using any of it, reduces the tile amax over 8 lanes and derives the
//      row exponent e;
//   2. once the block's 128 exponents are in shared memory each warp reduces Smax, then
//      encodes the row-wise codes, stores them with their scale, shifts them by the row's
//      k (uniform over a thread's 16 codes) and stages them in a swizzled 16 KB tile;
//   3. each lane gathers 8 tokens x 8 channels from the tile, transposes them with byte
//      permutes and writes eight 8-byte runs of Q^T (each warp store fills 128 bytes of
//      two channel rows).
// Options: an all-zero tile may take e = -127 instead of 0 (it then never raises Smax);
// scales may be written as packed UE8M0 words (four K-consecutive scale bytes per
// 32-bit word, MN-major: word (g, m) at g * mn_pad + m), the layout the SM100 GEMM reads
// (DeepSeek FP8 §8).
#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
constexpr int kPasses = 4;  // 4 passes x 32 rows; 8 lanes per 1x128 row tile

// 16-byte chunk position of chunk `c` of tile row `r`.  Phase 3 reads 8 bytes from rows
// 8t + i (t = 0..7 in each half-warp) of the same chunk: the (r >> 3) term spreads those
// over 8 distinct chunks.  Phase 2 writes 8-byte pieces of 4 consecutive rows, served
// per half-warp (two rows each): the (r & 1) term puts the two rows of a half-warp into
// opposite bank halves, so each 256-byte warp store takes the minimum two wavefronts.
__device__ __forceinline__ int tile_chunk(int r, int c) { return c ^ ((r >> 3) & 7) ^ ((r & 1) << 2); }

// Byte `i` (0..3) of packed scale word `word` := v; bytes are the K order of the tiles.
__device__ __forceinline__ void put_packed(uint8_t* packed, int64_t word, int i, uint8_t v) { packed[word * 4 + i] = v; }

template <bool kColwise, bool kPacked>
__global__ void __launch_bounds__(kThreads, 4)
    quantize_rowwise_colwise_kernel(const uint16_t* __restrict__ x, int64_t rows, int cols, int zero_e,
                                    uint8_t* __restrict__ q, uint8_t* __restrict__ sf, uint8_t* __restrict__ qt,
                                    uint8_t* __restrict__ sft) {
  __shared__ __align__(16) uint8_t tile[128 * 128];
  __shared__ __align__(16) uint8_t e_row[128];
  pdl_wait_for(x);
  pdl_trigger();
  const int tid = threadIdx.x;
  const int ncb = cols >> 7;
  const int64_t b = (int64_t)blockIdx.x / ncb;             // row block
  const int j = (int)((int64_t)blockIdx.x - b * ncb);     // column block, fastest: concurrent CTAs
  const int64_t r0 = b * 128;                              // cover whole rows of X
  const int c0 = j * 128;
  const int sub = tid & 7;                      // 8-element chunk in each half of the row tile
  const int rsub = tid >> 3;                    // row within a pass
  const int64_t mn_pad = (rows + 3) & ~int64_t(3);
  const uint16_t* xb = x + r0 * cols + c0;      // this block; offsets inside it fit in 32 bits
  uint8_t* qb = q + r0 * cols + c0;

  // ---- 1. loads and row exponents
  uint4 v0[kPasses], v1[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int rl = p * 32 + rsub;
    if (kColwise || r0 + rl < rows) {
      const uint4* src = reinterpret_cast<const uint4*>(xb + rl * cols);
      v0[p] = ld_g(src + sub);
      v1[p] = ld_g(src + 8 + sub);
    } else {
      v0[p] = v1[p] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  int e[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    uint32_t m = maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(v0[p].x, v0[p].y), maxabs_bf16x2(v0[p].z, v0[p].w)),
                               maxabs_bf16x2(maxabs_bf16x2(v1[p].x, v1[p].y), maxabs_bf16x2(v1[p].z, v1[p].w)));
    m = maxabs_bf16x2(m, __byte_perm(m, 0u, 0x1032)) & 0x7FFFu;
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    e[p] = bf16_tile_exponent(m, zero_e);
    if (kColwise && sub == 0) e_row[p * 32 + rsub] = (uint8_t)(e[p] + 127);
  }
  int emax = 0;
  if (kColwise) {
    __syncthreads();
    const uint32_t w = reinterpret_cast<const uint32_t*>(e_row)[tid & 31];
    int m = (int)max(max(w & 0xFFu, (w >> 8) & 0xFFu), max((w >> 16) & 0xFFu, w >> 24));
    m = (int)__reduce_max_sync(0xFFFFFFFFu, (unsigned)m);
    emax = m - 127;
  }

  // ---- 2. row-wise codes and scales; shifted codes into the tile
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int rl = p * 32 + rsub;
    const int64_t r = r0 + rl;
    const float s = exp2_neg(e[p]);
    uint32_t w[4] = {encode4(v0[p].x, v0[p].y, s), encode4(v0[p].z, v0[p].w, s), encode4(v1[p].x, v1[p].y, s),
                     encode4(v1[p].z, v1[p].w, s)};
    if (kColwise || r < rows) {
      uint8_t* dst = qb + rl * cols;
      *reinterpret_cast<uint2*>(dst + 8 * sub) = make_uint2(w[0], w[1]);
      *reinterpret_cast<uint2*>(dst + 64 + 8 * sub) = make_uint2(w[2], w[3]);
    }
    if (sub == 0) {
      if (!kPacked) {
        if (kColwise || r < rows) sf[r * ncb + j] = (uint8_t)(e[p] + 127);
      } else if (r < mn_pad) {  // rows past the end (padding of the packed layout) get zero words
        const int64_t word = (int64_t)(j >> 2) * mn_pad + r;
        put_packed(sf, word, j & 3, r < rows ? (uint8_t)(e[p] + 127) : (uint8_t)0);
        if (j == ncb - 1)
          for (int i = (j & 3) + 1; i < 4; ++i) put_packed(sf, word, i, 0);
      }
    }
    if (kColwise) {
      shift_row16_warp(w, emax - e[p]);
      uint8_t* row = tile + rl * 128 + 8 * (sub & 1);
      *reinterpret_cast<uint2*>(row + 16 * tile_chunk(rl, sub >> 1)) = make_uint2(w[0], w[1]);
      *reinterpret_cast<uint2*>(row + 16 * tile_chunk(rl, 4 + (sub >> 1))) = make_uint2(w[2], w[3]);
    }
  }
  if (!kColwise) return;

  // ---- 3. transpose: warp wi owns channels 16wi..16wi+15, lane (t, g) tokens 8t.. x 8 channels
  __syncthreads();
  const int lane = tid & 31, wi = tid >> 5;
  const int t = lane >> 1, g = lane & 1;
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rl = 8 * t + i;
    const uint2 w = *reinterpret_cast<const uint2*>(tile + rl * 128 + 16 * tile_chunk(rl, wi) + 8 * g);
    lo[i] = w.x;
    hi[i] = w.y;
  }
  uint32_t a[4][2], c[4][2];  // [channel][token quad]: channels 0..3 from lo, 4..7 from hi
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

  if (tid < 128) {
    const int64_t h = c0 + tid;
    const int64_t nb = rows >> 7;
    const uint8_t byte = (uint8_t)(emax + 127);
    if (!kPacked) {
      sft[h * nb + b] = byte;
    } else {
      const int64_t word = (b >> 2) * (int64_t)cols + h;
      put_packed(sft, word, (int)(b & 3), byte);
      if (b == nb - 1)
        for (int i = (int)(b & 3) + 1; i < 4; ++i) put_packed(sft, word, i, 0);
    }
  }
}

}  // namespace

fp8q_status launch_quantize_rowwise_colwise(const DeviceInfo& dev, const void* x, int64_t rows, int64_t cols,
                                            uint32_t flags, uint8_t* q, void* sf, uint8_t* qt, void* sft,
                                            cudaStream_t stream) {
  (void)dev;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  const int64_t gx = (rows + 127) / 128;
  if (gx * (cols / 128) > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const int zero_e = (flags & FP8Q_ZERO_TILE_MIN_SCALE) ? -127 : 0;
  const bool packed = (flags & FP8Q_SF_PACKED_UE8M0) != 0;
  const dim3 grid((unsigned)(gx * (cols / 128)));
  auto kernel = qt ? (packed ? quantize_rowwise_colwise_kernel<true, true> : quantize_rowwise_colwise_kernel<true, false>)
                   : (packed ? quantize_rowwise_colwise_kernel<false, true> : quantize_rowwise_colwise_kernel<false, false>);
  return launch_after(kernel, grid, kThreads, 0, stream, static_cast<const uint16_t*>(x), rows, (int)cols, zero_e, q,
                      static_cast<uint8_t*>(sf), qt, static_cast<uint8_t*>(sft)) == cudaSuccess
             ? FP8Q_OK
             : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
