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
        rr[s] = __ldg(row_id_map + t * kK + s);
        wg[s] = weights != nullptr ? __ldg(weights + t * kK + s) : 1.0f;
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
              d[b] = __ldg(reinterpret_cast<const uint4*>(y + r * hidden + h0));
              sc[b] = ue8m0_scale(__ldg(y_sf + r * ntile + (h0 >> 7)));
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
          const int64_t r = __ldg(row_id_map + t * topk + s);
          if (r < 0 || r >= rows) {
            record_status(status, FP8Q_ERR_DEVICE);  // the slot is skipped
          } else {
            use[b] = true;
            if (weights != nullptr) ws[b] = __ldg(weights + t * topk + s);
            if (kFp8) {
              d0[b] = __ldg(reinterpret_cast<const uint4*>(y + r * hidden + h0));
              sc[b] = ue8m0_scale(__ldg(y_sf + r * ntile + (h0 >> 7)));
            } else {
              const uint4* src = reinterpret_cast<const uint4*>(y + (r * hidden + h0) * 2);
              d0[b] = __ldg(src);
              d1[b] = __ldg(src + 1);
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
void launch_k(const UnpermuteArgs& a, unsigned blocks, cudaStream_t stream) {
  unpermute_unpad_kernel<kFp8, kK><<<blocks, kThreads, 0, stream>>>(a.y, a.y_sf, a.rows, a.hidden, a.row_id_map,
                                                                    a.weights, a.tokens, a.topk, a.out, a.status);
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
  if (y_sf == nullptr) {
    launch_k<false, 0>(a, blocks, stream);
  } else {
    switch (topk) {
      case 1: launch_k<true, 1>(a, blocks, stream); break;
      case 2: launch_k<true, 2>(a, blocks, stream); break;
      case 3: launch_k<true, 3>(a, blocks, stream); break;
      case 4: launch_k<true, 4>(a, blocks, stream); break;
      case 5: launch_k<true, 5>(a, blocks, stream); break;
      case 6: launch_k<true, 6>(a, blocks, stream); break;
      case 7: launch_k<true, 7>(a, blocks, stream); break;
      case 8: launch_k<true, 8>(a, blocks, stream); break;
      default: launch_k<true, 0>(a, blocks, stream); break;
    }
  }
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
