// permute_common.cuh — pieces shared by the permute kernels (permute_pad_quant.cu) and
// the expert-parallel dispatch (ep_dispatch.cu): chunking of the routing pairs and the
// padding-row fill.
#pragma once

#include "common.cuh"

namespace fp8q {

constexpr int kChunk = 1024;  // routing pairs per chunk, in row-major (row, slot) order
constexpr int kMaxExperts = 4096;
constexpr int kPadRowsPerCta = 8;
constexpr int kSThreads = 256;  // payload kernels: threads per CTA
constexpr int kSUnroll = 2;     // payload kernels: tile slots per warp (four tiles each)

inline int64_t num_chunks(int64_t rows, int32_t slots) { return (rows * slots + kChunk - 1) / kChunk; }

// Padding rows: CTA slot `slot` of expert e zeroes rows offsets[e] + totals[e] + 8*slot ..
// (at most 8 rows, never past offsets[e+1]): codes 0x00, scale byte 127.  Run by the
// trailing CTAs of a payload launch (E x ceil((align-1)/8) of them).  Rows outside
// [0, max_rows), the output's capacity, are never written (a consistent routing has none).
__device__ __forceinline__ void pad_rows(int64_t pad_cta, int pad_slots, const int32_t* __restrict__ offsets,
                                         const int32_t* __restrict__ totals, int64_t hidden, uint8_t* __restrict__ q,
                                         uint8_t* __restrict__ sf, int64_t max_rows) {
  const int e = (int)(pad_cta / pad_slots);
  const int slot = (int)(pad_cta - (int64_t)e * pad_slots);
  const int64_t start = (int64_t)offsets[e] + totals[e], end = offsets[e + 1];
  const int64_t ncb = hidden >> 7;
  for (int rr = 0; rr < kPadRowsPerCta; ++rr) {
    const int64_t r = start + (int64_t)slot * kPadRowsPerCta + rr;
    if (r >= end || r < 0 || r >= max_rows) return;
    uint4* row = reinterpret_cast<uint4*>(q + r * hidden);
    for (int64_t i = threadIdx.x; i < hidden / 16; i += blockDim.x) row[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t i = threadIdx.x; i < ncb; i += blockDim.x) sf[r * ncb + i] = 127;
  }
}

}  // namespace fp8q
