// direct_transpose.cu — FP8-Flow-MoE's scaling-aware direct transpose on sm_100a.
//
// FP8-Flow-MoE review, 核心方法: with power-of-two scales the row-wise -> column-wise
// conversion needs no dequant/requant: inside each 128x128 block take the largest row
// scale Smax and shift every code of row t by k_t = log2(Smax) - log2(S_t) binades,
// re-forming the mantissa only where the result turns subnormal (设计取舍 2: an O(1)
// exponent operation).  DeepSeek FP8 §1: wgrad reduces over tokens, so it consumes the
// transposed (1x128 along tokens) layout; §5.6: expert groups are contiguous row ranges.
//
// One CTA per 128x128 block, eight CTAs per SM (32 registers, 16.5 KB of shared memory
// each; six in grouped mode), so many small independent CTAs keep enough loads in flight
// without a pipeline.  256 threads:
//   1. each thread loads four 16-byte row chunks (one per 32-row pass) and, for the first
//      128 threads, one scale byte; every warp reduces Smax from shared memory;
//   2. each row chunk is shifted by its row's k (uniform over the chunk: the SWAR
//      exponent subtract when exact for all 16 bytes of every lane of the warp, else the
//      f16 route, see shift_row16_warp) and stored to a 16 KB tile whose 16-byte chunks
//      are XOR-swizzled by row;
//   3. each lane gathers 8 tokens x 8 channels with 8-byte shared loads (conflict-free per
//      half-warp), transposes them with byte permutes (four 4x4 transposes) and writes
//      eight 8-byte runs of Q^T (each warp store fills 128 bytes of two channel rows).
// Dense mode: a 2-D grid (column blocks x row blocks); the Q loads are marked evict-first
// and the Q^T stores streaming (each byte is touched once), which measured 4-6% faster
// than default caching when such launches run back to back.  Grouped mode (expert
// offsets on the device): a 1-D grid over the buffer's capacity in row-major block order
// with default caching (both measured faster there); each CTA finds its group by binary
// search, CTAs past the last group exit, and every inconsistency is recorded in the
// status word instead of producing an address.
#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
constexpr int kPasses = 4;

// Chunk c of tile row r sits at chunk position c ^ ((r >> 3) & 7): the phase-3 reads of
// rows 8t + i (t = 0..7 in each half-warp) hit 8 distinct chunk positions.
__device__ __forceinline__ int chunk_pos(int r, int c) { return c ^ ((r >> 3) & 7); }

template <bool kGrouped>
__global__ void __launch_bounds__(kThreads, kGrouped ? 6 : 8) direct_transpose_kernel(const uint8_t* __restrict__ q,
                                                                     const uint8_t* __restrict__ sf, int64_t rows,
                                                                     int cols, const int32_t* __restrict__ off,
                                                                     int G, uint8_t* __restrict__ qt,
                                                                     uint8_t* __restrict__ sft, int* status) {
  __shared__ __align__(16) uint8_t tile[128 * 128];
  __shared__ __align__(16) uint8_t e_row[128];
  const int tid = threadIdx.x;
  const int ncb = cols >> 7;
  int64_t b;
  int j;
  if (kGrouped || gridDim.y == 1) {  // 1-D grid, row-major blocks
    const unsigned bq = blockIdx.x / (unsigned)ncb;
    b = bq;
    j = (int)(blockIdx.x - bq * (unsigned)ncb);
  } else {
    b = blockIdx.y;
    j = blockIdx.x;
  }
  const int64_t r0 = b * 128;
  const int c0 = j * 128;
  int64_t o = 0, M = rows;
  if (kGrouped) {
    if (blockIdx.x == 0) validate_groups_cta(off, G, status);
    const int64_t limit = grouped_rows(off, G, rows, blockIdx.x == 0 ? status : nullptr);
    if (r0 >= limit) return;
    if (!find_group(off, G, r0, limit, o, M)) {
      if (tid == 0) record_status(status, FP8Q_ERR_SHAPE);
      return;
    }
  }
  const int sub = tid & 7, rsub = tid >> 3;    // 16-byte chunk, row within a 32-row pass
  // ---- 1. loads
  const uint8_t* qb = q + r0 * cols + c0;
  uint4 v[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const uint4* src = reinterpret_cast<const uint4*>(qb + (p * 32 + rsub) * cols) + sub;
    v[p] = kGrouped ? __ldg(src) : ld_stream(src);
  }
  if (tid < 128) e_row[tid] = __ldg(sf + (r0 + tid) * ncb + j);
  __syncthreads();
  const uint32_t ew = reinterpret_cast<const uint32_t*>(e_row)[tid & 31];
  int m = (int)max(max(ew & 0xFFu, (ew >> 8) & 0xFFu), max((ew >> 16) & 0xFFu, ew >> 24));
  m = (int)__reduce_max_sync(0xFFFFFFFFu, (unsigned)m);
  const int emax = m;
  // ---- 2. shift and stage
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int rl = p * 32 + rsub;
    uint32_t w[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
    shift_row16_warp(w, emax - (int)e_row[rl]);
    *reinterpret_cast<uint4*>(tile + rl * 128 + 16 * chunk_pos(rl, sub)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();
  // ---- 3. transpose (8 tokens x 8 channels per lane)
  const int lane = tid & 31, wi = tid >> 5;
  const int t = lane >> 1, g = lane & 1;
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rl = 8 * t + i;
    const uint2 w = *reinterpret_cast<const uint2*>(tile + rl * 128 + 16 * chunk_pos(rl, wi) + 8 * g);
    lo[i] = w.x;
    hi[i] = w.y;
  }
  uint32_t a[4][2], c[4][2];  // channel c (0..3 from lo, 4..7 from hi) x token quad
#pragma unroll
  for (int qd = 0; qd < 2; ++qd) {
    transpose4x4(lo[4 * qd], lo[4 * qd + 1], lo[4 * qd + 2], lo[4 * qd + 3], a[0][qd], a[1][qd], a[2][qd], a[3][qd]);
    transpose4x4(hi[4 * qd], hi[4 * qd + 1], hi[4 * qd + 2], hi[4 * qd + 3], c[0][qd], c[1][qd], c[2][qd], c[3][qd]);
  }
  uint8_t* out = qt + cols * o + (int64_t)(c0 + 16 * wi + 8 * g) * M + (r0 - o) + 8 * t;
#pragma unroll
  for (int k = 0; k < 8; ++k, out += M) {
    const uint2 val = k < 4 ? make_uint2(a[k][0], a[k][1]) : make_uint2(c[k - 4][0], c[k - 4][1]);
    if (kGrouped) *reinterpret_cast<uint2*>(out) = val; else st_stream8(out, val);
  }
  if (tid < 128) sft[cols * o / 128 + (int64_t)(c0 + tid) * (M >> 7) + ((r0 - o) >> 7)] = (uint8_t)emax;
}

}  // namespace

fp8q_status launch_direct_transpose(const DeviceInfo& dev, const uint8_t* q, const uint8_t* sf, int64_t rows,
                                    int64_t cols, const int32_t* offsets, int32_t num_groups, uint8_t* qt,
                                    uint8_t* sft, cudaStream_t stream) {
  const int64_t nblk = (rows / 128) * (cols / 128);
  if (nblk == 0) return FP8Q_OK;
  if (nblk > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const int64_t nrb = rows / 128;
  if (offsets)
    direct_transpose_kernel<true><<<(unsigned)nblk, kThreads, 0, stream>>>(q, sf, rows, (int)cols, offsets, num_groups,
                                                                           qt, sft, dev.status);
  else if (nrb > 1 && nrb <= 65535)  // 2-D grid: column blocks x row blocks
    direct_transpose_kernel<false><<<dim3((unsigned)(cols / 128), (unsigned)nrb), kThreads, 0, stream>>>(
        q, sf, rows, (int)cols, nullptr, 1, qt, sft, dev.status);
  else  // 1-D grid (gridDim.y == 1 selects the row-major mapping in the kernel)
    direct_transpose_kernel<false><<<(unsigned)nblk, kThreads, 0, stream>>>(q, sf, rows, (int)cols, nullptr, 1, qt,
                                                                            sft, dev.status);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
