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
//  * Persistent grid, one CTA per SM, WARPS independent warps per CTA.  Each warp owns
//    a contiguous range of 128x128 tiles (column block fastest, so consecutive tiles
//    share their scale rows in L1) and a private ring of STAGES shared-memory buffers
//    fed by 2-D TMA loads (16 KB box, 128B swizzle, no multicast), one mbarrier per
//    stage, every wait bounded.
//  * Lane (a = lane/8, c = lane%8) handles the 16x16 byte sub-tiles (rows 16a.., 64+16a..)
//    x (bytes 16c..): 16 conflict-free 16-byte shared loads per sub-tile (the 8 lanes of
//    a load phase read the 8 distinct chunks of one row), the row shift in registers
//    (SWAR fast path), a 16x16 byte transpose with byte permutes, and 16 coalesced
//    16-byte global stores (each output row gets 64 contiguous bytes per warp).
//  * Each warp reads the tile's 128 scale bytes itself (prefetched one tile ahead),
//    reduces e_max with warp shuffles and stages the row exponents in a 128-byte
//    per-warp buffer.
#include "common.cuh"
#include "launch.h"

#include <cudaTypedefs.h>

namespace fp8q {
namespace {

constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr int kTileBytes = 128 * 128;
constexpr int kMaxCachedOffsets = 1024;  // group offsets kept in shared memory

struct __align__(1024) DtShared {
  uint8_t tile[kWarps][kStages][kTileBytes];
  uint8_t e_row[kWarps][128];
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

// One 16x16 byte sub-tile: rows r0..r0+15 of the staged tile, bytes 16c..16c+15.
// `er` holds the 16 row exponent bytes (e + 127) of those rows.
__device__ __forceinline__ void process_subtile(const uint8_t* stage, int r0, int c, uint4 er, int emax,
                                                uint8_t* __restrict__ out, int64_t ld) {
  uint32_t w[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = r0 + i;
    const uint4 v = *reinterpret_cast<const uint4*>(stage + r * 128 + ((c ^ (r & 7)) << 4));  // 128B swizzle
    w[i][0] = v.x;
    w[i][1] = v.y;
    w[i][2] = v.z;
    w[i][3] = v.w;
  }
  const uint32_t ew[4] = {er.x, er.y, er.z, er.w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int k = emax - (int)((ew[i >> 2] >> (8 * (i & 3))) & 0xFFu);
    shift_row16(w[i], k);
  }
  // 16x16 transpose: output channel 4q+cc (q: word in the 16-byte chunk), token word v.
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t o[4][4];  // [cc][v]
#pragma unroll
    for (int v = 0; v < 4; ++v)
      transpose4x4(w[4 * v][q], w[4 * v + 1][q], w[4 * v + 2][q], w[4 * v + 3][q], o[0][v], o[1][v], o[2][v], o[3][v]);
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

  const int64_t ntiles = (valid_rows >> 7) * ncb;
  const int64_t gw = (int64_t)blockIdx.x * kWarps + warp, GW = (int64_t)gridDim.x * kWarps;
  const int64_t t_begin = gw * ntiles / GW, t_end = (gw + 1) * ntiles / GW;
  if (t_begin >= t_end) return;

  uint8_t(*ring)[kTileBytes] = sh.tile[warp];
  uint64_t* full = sh.full[warp];
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  auto issue = [&](int s, int64_t t) {
    const int64_t b = t / ncb;
    const int j = (int)(t - b * ncb);
    mbar_arrive_expect_tx(&full[s], kTileBytes);
    tma_load_2d(ring[s], &tmap_q, &full[s], j * 128, (int)(b * 128));
  };
  if (lane == 0)
    for (int s = 0; s < kStages && t_begin + s < t_end; ++s) issue(s, t_begin + s);

  const int a = lane >> 3, c = lane & 7;
  uint32_t sf_next = load_sf4(sf, t_begin / ncb, (int)(t_begin % ncb), ncb, lane);

  for (int64_t t = t_begin, i = 0; t < t_end; ++t, ++i) {
    const int s = (int)(i % kStages);
    const uint32_t parity = (uint32_t)((i / kStages) & 1);
    const int64_t b = t / ncb;
    const int j = (int)(t - b * ncb);
    const uint32_t sf_cur = sf_next;
    if (t + 1 < t_end) sf_next = load_sf4(sf, (t + 1) / ncb, (int)((t + 1) % ncb), ncb, lane);

    // e_max over the block's 128 row exponents; stage them for per-row lookups
    int m = (int)max(max(sf_cur & 0xFFu, (sf_cur >> 8) & 0xFFu), max((sf_cur >> 16) & 0xFFu, sf_cur >> 24));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 4; ++q) sh.e_row[warp][lane + 32 * q] = (uint8_t)(sf_cur >> (8 * q));
    __syncwarp();
    const uint4 eA = *reinterpret_cast<const uint4*>(&sh.e_row[warp][16 * a]);
    const uint4 eB = *reinterpret_cast<const uint4*>(&sh.e_row[warp][64 + 16 * a]);

    // output placement of row block b (dense: one group of all rows)
    int64_t o_g = 0, M = rows;
    bool valid = true;
    if (offsets != nullptr) valid = find_group(off, num_groups, b * 128, valid_rows, o_g, M);

    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], parity, kWaitTimeoutNs));
    if (!ok) {
      if (lane == 0) {
        record_status(status, FP8Q_ERR_TIMEOUT);
        // let the loads still in flight land before the CTA's shared memory is released
        for (int64_t u = t + 1; u < t_end && u < t + kStages; ++u) {
          const int64_t iu = i + (u - t);
          mbar_wait_bounded(&full[iu % kStages], (uint32_t)((iu / kStages) & 1), 10000000ull);
        }
      }
      __syncwarp();
      return;
    }
    if (valid) {
      const int64_t tok = b * 128 - o_g;  // first token of the block inside its group
      uint8_t* out = qt + (int64_t)cols * o_g + (int64_t)(j * 128) * M + tok;
      process_subtile(ring[s], 16 * a, c, eA, m, out + 16 * a, M);
      process_subtile(ring[s], 64 + 16 * a, c, eB, m, out + 64 + 16 * a, M);
      uint8_t* so = sft + (int64_t)cols * o_g / 128 + (int64_t)(j * 128) * (M >> 7) + (tok >> 7);
#pragma unroll
      for (int q = 0; q < 4; ++q) so[(int64_t)(lane + 32 * q) * (M >> 7)] = (uint8_t)m;
    } else if (lane == 0) {
      record_status(status, FP8Q_ERR_SHAPE);
    }
    __syncwarp();  // every lane has consumed stage s (its registers depend on the loads)
    if (lane == 0 && t + kStages < t_end) {
      fence_proxy_async_smem();
      issue(s, t + kStages);
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

fp8q_status launch_direct_transpose(const DeviceInfo& dev, const uint8_t* q, const uint8_t* sf, int64_t rows,
                                    int64_t cols, const int32_t* offsets, int32_t num_groups, uint8_t* qt,
                                    uint8_t* sft, cudaStream_t stream) {
  const int64_t ntiles_max = (rows / 128) * (cols / 128);
  if (ntiles_max == 0) return FP8Q_OK;
  auto encode = get_encoder();
  if (!encode) return FP8Q_ERR_CUDA;
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
  const int64_t warps_needed = ntiles_max;
  const int grid = (int)std::min<int64_t>(dev.num_sms, (warps_needed + kWarps - 1) / kWarps);
  direct_transpose_kernel<<<grid, kWarps * 32, smem, stream>>>(map, sf, rows, (int)cols, offsets, num_groups, qt, sft,
                                                               dev.status);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
