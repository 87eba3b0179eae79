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
// than default caching when such launches run back to back.
// Large dense inputs (at least eight waves of 256x128 tiles) take direct_transpose_2x1:
// one CTA per two row blocks of one column block (32 KB), five CTAs per SM.  Its 16-byte
// row chunks land in the swizzled shared tile by cp.async, without passing through
// registers; each thread then shifts the chunks it landed in place, and phase 3 gives
// each lane 16 tokens x 8 channels, so every warp store writes 256 contiguous bytes of
// two Q^T rows.  The longer runs lift the stress-size transpose by 3-4%; at the headline
// size its 2.4 waves leave a partly empty last wave and it is slower, hence the switch.  Grouped mode (expert
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
  pdl_wait_for(q, sf, off);
  pdl_trigger();
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
    v[p] = kGrouped ? ld_g(src) : ld_stream(src);
  }
  if (tid < 128) e_row[tid] = ld_g(sf + (r0 + tid) * ncb + j);
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

// ---- 2 row blocks x 1 column block per CTA (dense mode, large inputs)
// Tile: 256 rows x 128 bytes, 16-byte chunk c of row r at c ^ ((r >> 4) & 7): phase 3's
// lanes t = 0..7 (and 8..15) of a half-warp read rows 16t + i at 8 distinct positions.
// Lane mapping of phase 3: t = lane & 15 (tokens 16t..16t+15), g = ((lane >> 3) ^
// (lane >> 4)) & 1 (channels 8g..8g+7 of the warp's 16), so each half-warp's 8-byte
// reads cover 16 distinct bank pairs and each warp store two 256-byte row runs.
constexpr int kMinBlocks2x1 = 5;
__device__ __forceinline__ int chunk_pos2(int r, int c) { return c ^ ((r >> 4) & 7); }
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}

__global__ void __launch_bounds__(kThreads, kMinBlocks2x1) direct_transpose_2x1(const uint8_t* __restrict__ q,
                                                                               const uint8_t* __restrict__ sf,
                                                                               int64_t rows, int cols,
                                                                               uint8_t* __restrict__ qt,
                                                                               uint8_t* __restrict__ sft) {
  __shared__ __align__(128) uint8_t tile[256 * 128];
  __shared__ __align__(16) uint8_t e_row[256];
  __shared__ int emax_w[8];
  pdl_wait_for(q, sf);
  pdl_trigger();
  const int tid = threadIdx.x;
  const int ncb = cols >> 7;
  const unsigned bq = blockIdx.x / (unsigned)ncb;
  const int64_t b0 = 2 * (int64_t)bq;  // first of the two row blocks
  const int j = (int)(blockIdx.x - bq * (unsigned)ncb);
  const int64_t r0 = b0 * 128;
  const int c0 = j * 128;
  // ---- 1. chunk L = i*256 + tid: row L >> 3, chunk L & 7 (a warp covers 4 whole rows)
  const uint8_t* qb = q + r0 * cols + c0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int L = i * 256 + tid;
    const int row = L >> 3, c = L & 7;
    cp_async16(tile + row * 128 + 16 * chunk_pos2(row, c), qb + (int64_t)row * cols + 16 * c);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  const int e = ld_g(sf + (r0 + tid) * ncb + j);  // scale byte of row tid
  e_row[tid] = (uint8_t)e;
  const int lane = tid & 31, wi = tid >> 5;  // warp wi holds rows 32wi..32wi+31: row block wi >> 2
  const unsigned wm = __reduce_max_sync(0xFFFFFFFFu, (unsigned)e);
  if (lane == 0) emax_w[wi] = (int)wm;
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  const int em0 = max(max(emax_w[0], emax_w[1]), max(emax_w[2], emax_w[3]));
  const int em1 = max(max(emax_w[4], emax_w[5]), max(emax_w[6], emax_w[7]));
  // ---- 2. each thread shifts the chunks it landed, in place
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int L = i * 256 + tid;
    const int row = L >> 3, c = L & 7;
    uint4* p = reinterpret_cast<uint4*>(tile + row * 128 + 16 * chunk_pos2(row, c));
    const uint4 v = *p;
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
    shift_row16_warp(w, (row < 128 ? em0 : em1) - (int)e_row[row]);
    *p = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();
  // ---- 3. transpose: 16 tokens x 8 channels per lane, 16-byte stores
  const int t = lane & 15, g = ((lane >> 3) ^ (lane >> 4)) & 1;
  uint32_t lo[16], hi[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int row = 16 * t + i;
    const uint2 w = *reinterpret_cast<const uint2*>(tile + row * 128 + 16 * chunk_pos2(row, wi) + 8 * g);
    lo[i] = w.x;
    hi[i] = w.y;
  }
  uint32_t a[4][4], c[4][4];  // channel (0..3 from lo, 4..7 from hi) x token quad
#pragma unroll
  for (int qd = 0; qd < 4; ++qd) {
    transpose4x4(lo[4 * qd], lo[4 * qd + 1], lo[4 * qd + 2], lo[4 * qd + 3], a[0][qd], a[1][qd], a[2][qd], a[3][qd]);
    transpose4x4(hi[4 * qd], hi[4 * qd + 1], hi[4 * qd + 2], hi[4 * qd + 3], c[0][qd], c[1][qd], c[2][qd], c[3][qd]);
  }
  uint8_t* out = qt + (int64_t)(c0 + 16 * wi + 8 * g) * rows + r0 + 16 * t;
#pragma unroll
  for (int k = 0; k < 8; ++k, out += rows)
    *reinterpret_cast<uint4*>(out) = k < 4 ? make_uint4(a[k][0], a[k][1], a[k][2], a[k][3])
                                           : make_uint4(c[k - 4][0], c[k - 4][1], c[k - 4][2], c[k - 4][3]);
  // SF^T [cols, rows/128]: channel c0 + tid, row blocks b0 and b0 + 1 (one 16-bit store)
  if (tid < 128)
    *reinterpret_cast<uint16_t*>(sft + (int64_t)(c0 + tid) * (rows >> 7) + b0) = (uint16_t)(em0 | (em1 << 8));
}

}  // namespace

fp8q_status launch_direct_transpose(const DeviceInfo& dev, const uint8_t* q, const uint8_t* sf, int64_t rows,
                                    int64_t cols, const int32_t* offsets, int32_t num_groups, uint8_t* qt,
                                    uint8_t* sft, cudaStream_t stream) {
  const int64_t nblk = (rows / 128) * (cols / 128);
  if (nblk == 0) return FP8Q_OK;
  if (nblk > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const int64_t nrb = rows / 128;
  const int64_t tiles2 = (rows / 256) * (cols / 128);
  if (!offsets && rows % 256 == 0 && tiles2 >= 8LL * kMinBlocks2x1 * dev.num_sms) {
    return launch_after(direct_transpose_2x1, dim3((unsigned)tiles2), kThreads, 0, stream, q, sf, rows, (int)cols,
                        qt, sft) == cudaSuccess
               ? FP8Q_OK
               : FP8Q_ERR_CUDA;
  }
  const int32_t* no_offsets = nullptr;
  cudaError_t rc;
  if (offsets)
    rc = launch_after(direct_transpose_kernel<true>, dim3((unsigned)nblk), kThreads, 0, stream, q, sf, rows, (int)cols,
                      offsets, (int)num_groups, qt, sft, dev.status);
  else if (nrb > 1 && nrb <= 65535)  // 2-D grid: column blocks x row blocks
    rc = launch_after(direct_transpose_kernel<false>, dim3((unsigned)(cols / 128), (unsigned)nrb), kThreads, 0, stream,
                      q, sf, rows, (int)cols, no_offsets, 1, qt, sft, dev.status);
  else  // 1-D grid (gridDim.y == 1 selects the row-major mapping in the kernel)
    rc = launch_after(direct_transpose_kernel<false>, dim3((unsigned)nblk), kThreads, 0, stream, q, sf, rows, (int)cols,
                      no_offsets, 1, qt, sft, dev.status);
  return rc == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
