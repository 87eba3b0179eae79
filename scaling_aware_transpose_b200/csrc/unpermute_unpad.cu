// unpermute_unpad.cu — fused unpermute + unpad: the combine side of the expert path.
//
// FP8-Flow-MoE review, 核心方法 (fused Permute+Padding / Unpermute+Unpadding): after the
// expert GEMMs the rows are still in expert order, padded per expert; each token's K
// rows are gathered back and summed with its routing weights, and the padding rows are
// simply never read.  With unit weights this is the backward of the permute (the
// gradient of a token is the sum of its K copies' gradients).
//
// Arithmetic (this library's reading; the pages fix none): each input value in fp32
// (BF16 widened, or an E4M3 code decoded exactly and multiplied by its power-of-two
// scale), acc = fma(w[t,s], v, acc) for s = 0..K-1 starting from -0 (the additive
// identity that keeps the sign of a zero product: one slot gives its product exactly),
// then BF16 with round-to-nearest-even.
//
// HBM-bound gather: per token K rows in (2 or 1 + 1/128 bytes per element each), one
// BF16 row out.  Each thread owns 16 consecutive channels of one token (threads in
// token-major order, so a warp reads 512 or 256 contiguous bytes of each source row and
// writes 512 contiguous bytes), issues the loads of four slots before using any, and
// keeps 16 fp32 accumulators.  For FP8 rows with top-k <= 8 (one specialisation per k)
// the token's row indices and weights are all loaded first: a thread's 16-byte FP8 chunk
// takes as long to arrive as the index it depends on, so this saves a round trip per four
// slots.  BF16 rows keep the index loads inside each batch, which measured faster there.
//
// FP8 rows with top-k <= 8 and hidden % 512 == 0 take a warp-specialised ring instead
// (unpermute_fp8_ring): one CTA per SM walks its tokens (blockIdx.x, + gridDim.x, ...)
// through three shared-memory stages.  A producer warp keeps the next token's row
// indices and weights in flight while it fills a stage: the token's K rows of codes
// arrive by bulk copies (7 KB each at hidden 7168), its scale bytes by 8-byte cp.async
// (4-byte where hidden % 1024 != 0: the rows' scale bytes start 4-byte aligned there),
// both tracked by the stage's mbarrier; the consumer warps dequantize and accumulate from
// shared memory in the same slot order as above (identical bytes) and release the stage
// through a second mbarrier.  Row loads no longer wait on the index loads, and three
// tokens' rows are in flight per SM without holding registers.  Every wait is bounded:
// a timeout records FP8Q_ERR_TIMEOUT, raises an abort flag that stops both sides, and
// the producer waits (bounded again) for the copies it issued before the CTA exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 4;  // slots whose row loads are in flight together

// 2^(byte - 127) as fp32 for a UE8M0 byte in [0, 254] (byte 0 is the subnormal 2^-127).
__device__ __forceinline__ float ue8m0_scale(uint32_t byte) {
  return byte == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(byte << 23);
}

// Four E4M3 codes (one word) -> four exact fp32 values times the scale s.
__device__ __forceinline__ void dequant4(uint32_t w, float s, float* v) {
  const uint32_t lo = cvt_f16x2_e4m3x2(w & 0xFFFFu), hi = cvt_f16x2_e4m3x2(w >> 16);
  v[0] = __half2float(__ushort_as_half((unsigned short)(lo & 0xFFFFu))) * s;
  v[1] = __half2float(__ushort_as_half((unsigned short)(lo >> 16))) * s;
  v[2] = __half2float(__ushort_as_half((unsigned short)(hi & 0xFFFFu))) * s;
  v[3] = __half2float(__ushort_as_half((unsigned short)(hi >> 16))) * s;
}

template <bool kFp8, int kK>
__global__ void __launch_bounds__(kThreads) unpermute_unpad_kernel(const uint8_t* __restrict__ y,
                                                                   const uint8_t* __restrict__ y_sf, int64_t rows,
                                                                   int hidden, const int32_t* __restrict__ row_id_map,
                                                                   const float* __restrict__ weights, int64_t tokens,
                                                                   int topk, uint16_t* __restrict__ out,
                                                                   int* status) {
  pdl_wait_for(y, y_sf, row_id_map, weights);
  pdl_trigger();
  const int nch = hidden >> 4;
  const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (gid >= tokens * nch) return;
  const int64_t t = gid / nch;
  const int h0 = (int)(gid - t * nch) * 16;
  const int ntile = hidden >> 7;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = -0.0f;

  if constexpr (kFp8 && kK > 0) {
    // FP8 rows, top-k fixed at compile time: the token's indices and weights first, in one
    // round trip, then the rows, kBatch slots at a time.
    {
      int64_t rr[kK];
      float wg[kK];
#pragma unroll
      for (int s = 0; s < kK; ++s) {
        rr[s] = ld_g(row_id_map + t * kK + s);
        wg[s] = weights != nullptr ? ld_g(weights + t * kK + s) : 1.0f;
      }
#pragma unroll
      for (int s0 = 0; s0 < kK; s0 += kBatch) {
        uint4 d[kBatch];
        float sc[kBatch];
        bool use[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int s = s0 + b;
          const int64_t r = s < kK ? rr[s] : 0;
          use[b] = false;
          sc[b] = 1.0f;
          d[b] = make_uint4(0u, 0u, 0u, 0u);
          if (s < kK) {
            if (r < 0 || r >= rows) {
              record_status(status, FP8Q_ERR_DEVICE);  // the slot is skipped
            } else {
              use[b] = true;
              d[b] = ld_g(reinterpret_cast<const uint4*>(y + r * hidden + h0));
              sc[b] = ue8m0_scale(ld_g(y_sf + r * ntile + (h0 >> 7)));
            }
          }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          if (!use[b]) continue;
          float v[16];
          dequant4(d[b].x, sc[b], v);
          dequant4(d[b].y, sc[b], v + 4);
          dequant4(d[b].z, sc[b], v + 8);
          dequant4(d[b].w, sc[b], v + 12);
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = __fmaf_rn(wg[s0 + b < kK ? s0 + b : 0], v[i], acc[i]);
        }
      }
    }
  } else {  // BF16 rows, or FP8 rows with top-k > 8
    for (int s0 = 0; s0 < topk; s0 += kBatch) {
      uint4 d0[kBatch], d1[kBatch];  // 16 codes, or 16 bf16 in two halves
      float ws[kBatch], sc[kBatch];
      bool use[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int s = s0 + b;
        use[b] = false;
        ws[b] = 1.0f;
        sc[b] = 1.0f;
        d0[b] = d1[b] = make_uint4(0u, 0u, 0u, 0u);
        if (s < topk) {
          const int64_t r = ld_g(row_id_map + t * topk + s);
          if (r < 0 || r >= rows) {
            record_status(status, FP8Q_ERR_DEVICE);  // the slot is skipped
          } else {
            use[b] = true;
            if (weights != nullptr) ws[b] = ld_g(weights + t * topk + s);
            if (kFp8) {
              d0[b] = ld_g(reinterpret_cast<const uint4*>(y + r * hidden + h0));
              sc[b] = ue8m0_scale(ld_g(y_sf + r * ntile + (h0 >> 7)));
            } else {
              const uint4* src = reinterpret_cast<const uint4*>(y + (r * hidden + h0) * 2);
              d0[b] = ld_g(src);
              d1[b] = ld_g(src + 1);
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        if (!use[b]) continue;
        float v[16];
        if (kFp8) {
          dequant4(d0[b].x, sc[b], v);
          dequant4(d0[b].y, sc[b], v + 4);
          dequant4(d0[b].z, sc[b], v + 8);
          dequant4(d0[b].w, sc[b], v + 12);
        } else {
          const uint32_t wd[8] = {d0[b].x, d0[b].y, d0[b].z, d0[b].w, d1[b].x, d1[b].y, d1[b].z, d1[b].w};
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            v[2 * k] = __uint_as_float(wd[k] << 16);
            v[2 * k + 1] = __uint_as_float(wd[k] & 0xFFFF0000u);
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = __fmaf_rn(ws[b], v[i], acc[i]);
      }
    }
  }
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
    o[k] = *reinterpret_cast<const uint32_t*>(&p);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + t * hidden + h0);
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// ---- FP8 ring (see the header)
constexpr int kRingStages = 3;
constexpr int kRingConsumerWarps = 14;
constexpr int kRingThreads = (kRingConsumerWarps + 1) * 32;

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// Global -> shared bulk copy of `bytes` (16-byte aligned, a multiple of 16), completion
// counted on `bar` in bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Stage bytes: codes [kK][hidden] | scale bytes [kK][hidden/128] (padded to 16) | row ids
// int32 [kK] (-1: skipped) | weights fp32 [kK], rounded up to 128.
__host__ __device__ inline int ring_stage_bytes(int K, int hidden) {
  return (K * hidden + ((K * (hidden >> 7) + 15) & ~15) + 8 * K + 127) & ~127;
}

template <int kK>
__global__ void __launch_bounds__(kRingThreads, 1) unpermute_fp8_ring(const uint8_t* __restrict__ y,
                                                                      const uint8_t* __restrict__ y_sf, int64_t rows,
                                                                      int hidden,
                                                                      const int32_t* __restrict__ row_id_map,
                                                                      const float* __restrict__ weights,
                                                                      int64_t tokens, uint16_t* __restrict__ out,
                                                                      int* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait_for(y, y_sf, row_id_map, weights);
  pdl_trigger();
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // stage filled: 32 async arrivals + 1 expect-tx arrival
  uint64_t* empty = full + kRingStages;                 // stage released: one arrival per consumer warp
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kRingStages);
  uint8_t* base = smem + 128;
  const int ntile = hidden >> 7;
  const int stage_bytes = ring_stage_bytes(kK, hidden);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int st = 0; st < kRingStages; ++st) {
      mbar_init(&full[st], 33);
      mbar_init(&empty[st], kRingConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int64_t ntok = tokens > (int64_t)blockIdx.x ? (tokens - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto stage = [&](int st, uint8_t*& codes, uint8_t*& scales, int32_t*& rowsel, float*& wsel) {
    codes = base + (size_t)st * stage_bytes;
    scales = codes + (size_t)kK * hidden;
    rowsel = reinterpret_cast<int32_t*>(scales + ((kK * ntile + 15) & ~15));
    wsel = reinterpret_cast<float*>(rowsel + kK);
  };
  if (warp == kRingConsumerWarps) {
    // ---- producer warp
    int64_t issued = 0;
    int32_t r_next = -1;
    float w_next = 1.0f;
    if (ntok > 0 && lane < kK) {
      r_next = ld_g(row_id_map + (int64_t)blockIdx.x * kK + lane);
      w_next = weights != nullptr ? ld_g(weights + (int64_t)blockIdx.x * kK + lane) : 1.0f;
    }
    for (int64_t i = 0; i < ntok; ++i) {
      const int st = (int)(i % kRingStages);
      int32_t r = r_next;
      const float w = w_next;
      if (i + 1 < ntok && lane < kK) {  // the next token's indices, in flight while this one is issued
        const int64_t tn = blockIdx.x + (i + 1) * gridDim.x;
        r_next = ld_g(row_id_map + tn * kK + lane);
        w_next = weights != nullptr ? ld_g(weights + tn * kK + lane) : 1.0f;
      }
      if (i >= kRingStages &&
          !mbar_wait_bounded(&empty[st], (uint32_t)(((i / kRingStages) - 1) & 1), kWaitTimeoutNs)) {
        if (lane == 0) record_status(status, FP8Q_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (__any_sync(0xFFFFFFFFu, *abort_flag != 0)) break;
      uint8_t *codes, *scales;
      int32_t* rowsel;
      float* wsel;
      stage(st, codes, scales, rowsel, wsel);
      if (lane < kK) {
        if (r < 0 || r >= rows) {
          record_status(status, FP8Q_ERR_DEVICE);  // the slot is skipped
          r = -1;
        }
        rowsel[lane] = r;
        wsel[lane] = w;
      }
      const unsigned valid = __ballot_sync(0xFFFFFFFFu, lane < kK && r >= 0);
      // scale rows in 8-byte pieces (hidden % 1024 == 0) or 4-byte pieces (hidden % 512 ==
      // 0), spread over the lanes; every lane runs the same trip count so that the shuffle
      // sees the whole warp
      const bool wide = (ntile & 7) == 0;
      const int piece_bytes = wide ? 8 : 4;
      const int per_row = ntile / piece_bytes;
      for (int idx0 = 0; idx0 < kK * per_row; idx0 += 32) {
        const int idx = idx0 + lane;
        const int k = min(idx / per_row, kK - 1), piece = idx - k * per_row;
        const int32_t rk = __shfl_sync(0xFFFFFFFFu, r, k);
        if (idx < kK * per_row && rk >= 0) {
          const uint32_t dst = smem_u32(scales + k * ntile + piece_bytes * piece);
          const uint8_t* src = y_sf + (int64_t)rk * ntile + piece_bytes * piece;
          if (wide)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
          else
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
        }
      }
      // this lane's arrival fires when its cp.asyncs have landed
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[st])) : "memory");
      __syncwarp();  // orders every lane's row-id and weight stores before lane 0's release
      if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)(__popc(valid) * hidden));
      if (lane < kK && r >= 0)
        bulk_g2s(codes + (size_t)lane * hidden, y + (int64_t)r * hidden, (uint32_t)hidden, &full[st]);
      issued = i + 1;
    }
    // Every copy this warp issued lands before the CTA may exit: wait (bounded) for the last
    // phase issued on each stage.  On the normal path the consumers have already waited on
    // them and these return at once.
    for (int st = 0; st < kRingStages; ++st) {
      if (issued <= st) continue;
      const int64_t last = (issued - 1 - st) / kRingStages;  // phase index of stage st's last fill
      if (!mbar_wait_bounded(&full[st], (uint32_t)(last & 1), kWaitTimeoutNs) && lane == 0)
        record_status(status, FP8Q_ERR_TIMEOUT);
    }
    return;
  }
  // ---- consumer warps: 16 channels per thread and pass
  const int nch = hidden >> 4;
  for (int64_t i = 0; i < ntok; ++i) {
    const int st = (int)(i % kRingStages);
    if (!mbar_wait_bounded(&full[st], (uint32_t)((i / kRingStages) & 1), kWaitTimeoutNs)) {
      if (lane == 0) record_status(status, FP8Q_ERR_TIMEOUT);
      *abort_flag = 1;
      return;
    }
    if (*abort_flag != 0) return;
    const int64_t t = blockIdx.x + i * gridDim.x;
    uint8_t *codes, *scales;
    int32_t* rowsel;
    float* wsel;
    stage(st, codes, scales, rowsel, wsel);
    for (int c = tid; c < nch; c += kRingConsumerWarps * 32) {
      float acc[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) acc[q] = -0.0f;
#pragma unroll
      for (int k = 0; k < kK; ++k) {
        if (rowsel[k] < 0) continue;
        const uint4 d = *reinterpret_cast<const uint4*>(codes + (size_t)k * hidden + 16 * c);
        const float sc = ue8m0_scale(scales[k * ntile + (c >> 3)]);
        const float wk = wsel[k];
        float v[16];
        dequant4(d.x, sc, v);
        dequant4(d.y, sc, v + 4);
        dequant4(d.z, sc, v + 8);
        dequant4(d.w, sc, v + 12);
#pragma unroll
        for (int q = 0; q < 16; ++q) acc[q] = __fmaf_rn(wk, v[q], acc[q]);
      }
      uint32_t o[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        o[q] = *reinterpret_cast<const uint32_t*>(&p);
      }
      uint4* dst = reinterpret_cast<uint4*>(out + t * hidden + 16 * c);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
}

struct UnpermuteArgs {
  const uint8_t* y;
  const uint8_t* y_sf;
  int64_t rows;
  int hidden;
  const int32_t* row_id_map;
  const float* weights;
  int64_t tokens;
  int topk;
  uint16_t* out;
  int* status;
};

template <bool kFp8, int kK>
cudaError_t launch_k(const UnpermuteArgs& a, unsigned blocks, cudaStream_t stream) {
  return launch_after(unpermute_unpad_kernel<kFp8, kK>, dim3(blocks), kThreads, 0, stream, a.y, a.y_sf, a.rows,
                      a.hidden, a.row_id_map, a.weights, a.tokens, a.topk, a.out, a.status);
}

template <int kK>
cudaError_t launch_ring(const UnpermuteArgs& a, int grid, int smem, cudaStream_t stream) {
  const cudaError_t e = cudaFuncSetAttribute(unpermute_fp8_ring<kK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_after(unpermute_fp8_ring<kK>, dim3((unsigned)grid), kRingThreads, (size_t)smem, stream, a.y, a.y_sf,
                      a.rows, a.hidden, a.row_id_map, a.weights, a.tokens, a.out, a.status);
}

}  // namespace

fp8q_status launch_unpermute_unpad(const DeviceInfo& dev, const void* y, const uint8_t* y_sf, int64_t rows,
                                   int64_t hidden, const int32_t* row_id_map, const float* weights, int64_t tokens,
                                   int32_t topk, void* out, cudaStream_t stream) {
  const int64_t threads = tokens * (hidden / 16);
  if (threads == 0) return FP8Q_OK;
  const int64_t blocks64 = (threads + kThreads - 1) / kThreads;
  if (blocks64 > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const unsigned blocks = (unsigned)blocks64;
  const UnpermuteArgs a{static_cast<const uint8_t*>(y), y_sf, rows, (int)hidden, row_id_map, weights, tokens, topk,
                        static_cast<uint16_t*>(out), dev.status};
  const int ring_smem = 128 + kRingStages * ring_stage_bytes(topk, (int)hidden);
  // the scale rows' copy pieces: 8 bytes when hidden % 1024 == 0, else 4 (hidden % 512 == 0)
  const uintptr_t sf_align = hidden % 1024 == 0 ? 7u : 3u;
  if (y_sf != nullptr && topk >= 1 && topk <= 8 && hidden % 512 == 0 && ring_smem <= dev.max_smem_optin &&
      (reinterpret_cast<uintptr_t>(y_sf) & sf_align) == 0 && (reinterpret_cast<uintptr_t>(y) & 15u) == 0) {
    const int grid = (int)(tokens < dev.num_sms ? tokens : dev.num_sms);
    cudaError_t e = cudaSuccess;
    switch (topk) {
      case 1: e = launch_ring<1>(a, grid, ring_smem, stream); break;
      case 2: e = launch_ring<2>(a, grid, ring_smem, stream); break;
      case 3: e = launch_ring<3>(a, grid, ring_smem, stream); break;
      case 4: e = launch_ring<4>(a, grid, ring_smem, stream); break;
      case 5: e = launch_ring<5>(a, grid, ring_smem, stream); break;
      case 6: e = launch_ring<6>(a, grid, ring_smem, stream); break;
      case 7: e = launch_ring<7>(a, grid, ring_smem, stream); break;
      default: e = launch_ring<8>(a, grid, ring_smem, stream); break;
    }
    return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
  }
  cudaError_t e = cudaSuccess;
  if (y_sf == nullptr) {
    e = launch_k<false, 0>(a, blocks, stream);
  } else {
    switch (topk) {
      case 1: e = launch_k<true, 1>(a, blocks, stream); break;
      case 2: e = launch_k<true, 2>(a, blocks, stream); break;
      case 3: e = launch_k<true, 3>(a, blocks, stream); break;
      case 4: e = launch_k<true, 4>(a, blocks, stream); break;
      case 5: e = launch_k<true, 5>(a, blocks, stream); break;
      case 6: e = launch_k<true, 6>(a, blocks, stream); break;
      case 7: e = launch_k<true, 7>(a, blocks, stream); break;
      case 8: e = launch_k<true, 8>(a, blocks, stream); break;
      default: e = launch_k<true, 0>(a, blocks, stream); break;
    }
  }
  return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
