// direct_transpose.cu — FP8-Flow-MoE's scaling-aware direct transpose on sm_100a.
//
// FP8-Flow-MoE review, 核心方法: with power-of-two scales the row-wise -> column-wise
// conversion needs no dequant/requant: inside each 128x128 block take the largest row
// scale Smax and shift every code of row t by k_t = log2(Smax) - log2(S_t) binades,
// re-forming the mantissa only where the result turns subnormal (设计取舍 2: an O(1)
// exponent operation).  DeepSeek FP8 §1: wgrad reduces over tokens, so it consumes the
// transposed (1x128 along tokens) layout; §5.6: expert groups are contiguous row ranges.
//
// Design (HBM-bound: 2 bytes moved per element):
//  * Persistent grid, one CTA per SM, 12 independent warps per CTA (3 per scheduler, so
//    that one warp's shift/transpose latency hides behind the others).  The work unit is
//    128 rows x 64 columns of a 128x128 block.  Each warp owns a contiguous range of units
//    (the two column halves of a block back to back, then the next column block, so
//    scale rows are reused from L1) and a private ring of two 8 KB shared buffers fed
//    by 2-D TMA loads (box 64 B x 128 rows, no multicast), one mbarrier per stage, every
//    wait bounded.
//  * Lane (a, c) handles the 16x16 byte sub-tile rows 16a..16a+15 x bytes 16c..16c+15 of
//    the unit: 16 conflict-free 16-byte shared loads, the exact row shift in registers
//    (hardware E4M3<->f16 conversions around an f16 multiply by 2^-k), a 16x16 byte
//    transpose with byte permutes, and 16 16-byte global stores.  The 8 lanes sharing c
//    cover all 128 tokens of an output row, so every store instruction writes four whole
//    128-byte lines (output rows written as partial lines cost the L1 store path one
//    wavefront per lane).
//  * Once per block each warp reads the block's 128 scale bytes (prefetched one block
//    ahead), reduces e_max with warp shuffles and stages each row's f16x2 shift scale
//    {2^-k, 2^-k} in a 512-byte per-warp buffer.
#include "common.cuh"
#include "launch.h"

#include <cudaTypedefs.h>

namespace fp8q {
namespace {

constexpr int kWarps = 12;                 // independent warps per CTA (one CTA per SM)
constexpr int kStages = 2;                 // TMA stages per warp
constexpr int kUnitCols = 64;              // a unit is 128 rows x 64 columns of a block
constexpr int kUnitBytes = 128 * kUnitCols;
constexpr int kMaxCachedOffsets = 1024;    // group offsets kept in shared memory

struct __align__(1024) DtShared {
  uint8_t unit[kWarps][kStages][kUnitBytes];
  uint32_t scale[kWarps][128];  // per row of the current block: f16x2 {2^-k, 2^-k}
  uint64_t full[kWarps][kStages];
  int32_t offsets[kMaxCachedOffsets + 1];
};

__device__ __forceinline__ uint32_t load_sf4(const uint8_t* __restrict__ sf, int64_t b, int j, int ncb, int lane) {
  // scale bytes of rows 128b + lane + 32m (m = 0..3) in column block j, packed m-th byte
  const uint8_t* p = sf + (b * 128 + lane) * (int64_t)ncb + j;
  const int64_t st = 32 * (int64_t)ncb;
  return (uint32_t)__ldg(p) | ((uint32_t)__ldg(p + st) << 8) | ((uint32_t)__ldg(p + 2 * st) << 16) |
         ((uint32_t)__ldg(p + 3 * st) << 24);
}

// One 16x16 byte sub-tile of the staged unit: rows 16a..16a+15, bytes 16c..16c+15.
// Odd row groups (s = 1) read their rows in pair-swapped order (row i^1 at step i), so
// that the 8 lanes of a shared-load phase (row groups 2p and 2p+1, chunks 0..3) hit
// rows of opposite parity: 8 distinct 16-byte bank groups of the unswizzled 64-byte
// rows.  The swap is undone by the byte-permute selectors of the transpose.
// `sc` holds the 16 rows' f16x2 shift scales {2^-k, 2^-k} in row order.  Every word goes
// through the general (exact) shift: on activation data a quarter of the 16-byte row
// chunks hold a code that needs re-rounding, so a per-lane branch would make nearly
// every warp take both paths; rows with k == 0 in every lane are skipped (warp-uniform).
__device__ __forceinline__ void process_subtile(const uint8_t* stage, int a, int s, int c, const uint4 (&sc)[4],
                                                uint8_t* __restrict__ out, int64_t ld) {
  constexpr uint32_t kOne = 0x3C003C00u;  // f16x2 {1, 1}: k == 0
  uint32_t w[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(stage + (16 * a + (i ^ s)) * kUnitCols + 16 * c);
    w[i][0] = v.x;
    w[i][1] = v.y;
    w[i][2] = v.z;
    w[i][3] = v.w;
  }
  const uint32_t sv[16] = {sc[0].x, sc[0].y, sc[0].z, sc[0].w, sc[1].x, sc[1].y, sc[1].z, sc[1].w,
                           sc[2].x, sc[2].y, sc[2].z, sc[2].w, sc[3].x, sc[3].y, sc[3].z, sc[3].w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t s2 = s ? sv[i ^ 1] : sv[i];  // scale of the row held in w[i]
    if (!__all_sync(0xFFFFFFFFu, s2 == kOne)) {
#pragma unroll
      for (int x = 0; x < 4; ++x) w[i][x] = shift_word_general(w[i][x], s2);
    }
  }
  // 16x16 transpose: output channel 4q+cc (q: word in the 16-byte chunk), token word v.
  // First-stage selectors interleave rows 0/1 (and 2/3) of each quad, accounting for the
  // pair swap of odd row groups.
  const uint32_t selA = s ? 0x1504u : 0x5140u, selC = s ? 0x3726u : 0x7362u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t o[4][4];  // [cc][v]
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint32_t r0 = w[4 * v][q], r1 = w[4 * v + 1][q], r2 = w[4 * v + 2][q], r3 = w[4 * v + 3][q];
      const uint32_t ab = __byte_perm(r0, r1, selA), cd = __byte_perm(r2, r3, selA);
      const uint32_t ef = __byte_perm(r0, r1, selC), gh = __byte_perm(r2, r3, selC);
      o[0][v] = __byte_perm(ab, cd, 0x5410);
      o[1][v] = __byte_perm(ab, cd, 0x7632);
      o[2][v] = __byte_perm(ef, gh, 0x5410);
      o[3][v] = __byte_perm(ef, gh, 0x7632);
    }
    // the 8 lanes with the same c write one whole 128-byte line of each channel row
#pragma unroll
    for (int cc = 0; cc < 4; ++cc)
      *reinterpret_cast<uint4*>(out + (int64_t)(16 * c + 4 * q + cc) * ld) = make_uint4(o[cc][0], o[cc][1], o[cc][2], o[cc][3]);
  }
}

__global__ void __launch_bounds__(kWarps * 32, 1)
    direct_transpose_kernel(const __grid_constant__ CUtensorMap tmap_q, const uint8_t* __restrict__ sf, int64_t rows,
                            int cols, const int32_t* __restrict__ offsets, int num_groups, uint8_t* __restrict__ qt,
                            uint8_t* __restrict__ sft, int* status) {
  extern __shared__ uint8_t smem_raw[];
  DtShared& sh = *reinterpret_cast<DtShared*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncb = cols >> 7;

  // ---- groups: validate the global shape once, cache the offsets
  int64_t valid_rows = rows;
  const bool cached = offsets != nullptr && num_groups <= kMaxCachedOffsets;
  if (offsets != nullptr) {
    valid_rows = grouped_rows(offsets, num_groups, rows, threadIdx.x == 0 ? status : nullptr);
    if (cached)
      for (int g = threadIdx.x; g <= num_groups; g += blockDim.x) sh.offsets[g] = __ldg(offsets + g);
  }
  __syncthreads();
  const int32_t* off = cached ? sh.offsets : offsets;
  if (offsets != nullptr && blockIdx.x == 0) validate_groups_cta(off, num_groups, status);

  // units: (row block b, column block j, column half h), h fastest; each warp a
  // contiguous range
  const int64_t nunits = (valid_rows >> 7) * ncb * 2;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + warp, GW = (int64_t)gridDim.x * kWarps;
  const int64_t u_begin = gw * nunits / GW, u_end = (gw + 1) * nunits / GW;
  if (u_begin >= u_end) return;

  uint8_t(*ring)[kUnitBytes] = sh.unit[warp];
  uint64_t* full = sh.full[warp];
  uint32_t* scale = sh.scale[warp];
  if (lane == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue = [&](int st, int64_t u) {
    const int64_t blk = u >> 1;
    const int64_t b = blk / ncb;
    const int j = (int)(blk - b * ncb);
    mbar_arrive_expect_tx(&full[st], kUnitBytes);
    tma_load_2d(ring[st], &tmap_q, &full[st], j * 128 + (int)(u & 1) * kUnitCols, (int)(b * 128));
  };
  if (lane == 0)
    for (int st = 0; st < kStages && u_begin + st < u_end; ++st) issue(st, u_begin + st);

  const int sw = (lane >> 2) & 1, a = 2 * (lane >> 3) + sw, c = lane & 3;
  int64_t blk_cur = -1;
  int emax = 0;
  int64_t o_g = 0, M = rows;
  bool valid = true;
  int64_t blk_next = u_begin >> 1;
  uint32_t sf_next = load_sf4(sf, blk_next / ncb, (int)(blk_next % ncb), ncb, lane);

  for (int64_t u = u_begin, i = 0; u < u_end; ++u, ++i) {
    const int st = (int)(i % kStages);
    const uint32_t parity = (uint32_t)((i / kStages) & 1);
    const int64_t blk = u >> 1;
    const int64_t b = blk / ncb;
    const int j = (int)(blk - b * ncb);
    if (blk != blk_cur) {
      // new 128x128 block: e_max over its 128 row exponents; stage each row's scale
      const uint32_t sf_cur = sf_next;
      blk_cur = blk;
      const int64_t nb = blk + 1;
      if ((nb << 1) < u_end) sf_next = load_sf4(sf, nb / ncb, (int)(nb % ncb), ncb, lane);
      int m = (int)max(max(sf_cur & 0xFFu, (sf_cur >> 8) & 0xFFu), max((sf_cur >> 16) & 0xFFu, sf_cur >> 24));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      emax = m;
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q) scale[lane + 32 * q] = f16x2_pow2_neg(emax - (int)((sf_cur >> (8 * q)) & 0xFFu));
      __syncwarp();
      o_g = 0;
      M = rows;
      valid = true;
      if (offsets != nullptr) valid = find_group(off, num_groups, b * 128, valid_rows, o_g, M);
      if (!valid && lane == 0) record_status(status, FP8Q_ERR_SHAPE);
    }
    const int h = (int)(u & 1);
    uint4 sc[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) sc[x] = *reinterpret_cast<const uint4*>(&scale[16 * a + 4 * x]);

    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[st], parity, kWaitTimeoutNs));
    if (!ok) {
      if (lane == 0) {
        record_status(status, FP8Q_ERR_TIMEOUT);
        // let the loads still in flight land before the CTA's shared memory is released
        for (int64_t v = u + 1; v < u_end && v < u + kStages; ++v) {
          const int64_t iv = i + (v - u);
          mbar_wait_bounded(&full[iv % kStages], (uint32_t)((iv / kStages) & 1), 10000000ull);
        }
      }
      __syncwarp();
      return;
    }
    if (valid) {
      const int64_t tok = b * 128 - o_g;  // first token of the block inside its group
      const int64_t ch0 = (int64_t)j * 128 + h * kUnitCols;
      uint8_t* out = qt + (int64_t)cols * o_g + ch0 * M + tok + 16 * a;
      process_subtile(ring[st], a, sw, c, sc, out, M);
      uint8_t* so = sft + (int64_t)cols * o_g / 128 + ch0 * (M >> 7) + (tok >> 7);
#pragma unroll
      for (int q = 0; q < 2; ++q) so[(int64_t)(lane + 32 * q) * (M >> 7)] = (uint8_t)emax;
    }
    __syncwarp();  // every lane has consumed stage st (its registers depend on the loads)
    if (lane == 0 && u + kStages < u_end) {
      fence_proxy_async_smem();
      issue(st, u + kStages);
    }
  }
}

}  // namespace

fp8q_status launch_direct_transpose(const DeviceInfo& dev, const uint8_t* q, const uint8_t* sf, int64_t rows,
                                    int64_t cols, const int32_t* offsets, int32_t num_groups, uint8_t* qt,
                                    uint8_t* sft, cudaStream_t stream) {
  const int64_t nunits_max = (rows / 128) * (cols / 128) * 2;
  if (nunits_max == 0) return FP8Q_OK;
  auto encode = tensor_map_encoder();
  if (!encode) return FP8Q_ERR_CUDA;
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {(cuuint32_t)kUnitCols, 128};
  cuuint32_t estr[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return FP8Q_ERR_CUDA;
  const size_t smem = sizeof(DtShared) + 1024;
  static int configured_device = -1;
  if (configured_device != dev.device) {
    if (cudaFuncSetAttribute(direct_transpose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return FP8Q_ERR_CUDA;
    configured_device = dev.device;
  }
  const int grid = (int)std::min<int64_t>(dev.num_sms, (nunits_max + kWarps - 1) / kWarps);
  direct_transpose_kernel<<<grid, kWarps * 32, smem, stream>>>(map, sf, rows, (int)cols, offsets, num_groups, qt, sft,
                                                               dev.status);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
