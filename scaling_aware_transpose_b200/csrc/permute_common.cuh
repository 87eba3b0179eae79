// permute_common.cuh — pieces shared by the permute kernels (permute_pad_quant.cu) and
// the expert-parallel dispatch (ep_dispatch.cu): chunking of the routing pairs, the
// programmatic-dependent-launch helpers, the padding-row fill and the dependent launch.
#pragma once

#include "common.cuh"

namespace fp8q {

constexpr int kChunk = 1024;  // routing pairs per chunk, in row-major (row, slot) order
constexpr int kMaxExperts = 4096;
constexpr int kPadRowsPerCta = 8;
constexpr int kSThreads = 256;  // payload kernels: threads per CTA
constexpr int kSUnroll = 2;     // payload kernels: tile slots per warp (four tiles each)

inline int64_t num_chunks(int64_t rows, int32_t slots) { return (rows * slots + kChunk - 1) / kChunk; }

// Programmatic dependent launch (sm_90 and later): the scan, rank and payload launches
// carry the programmatic-stream-serialization attribute, so each may be scheduled while
// its predecessor in the chain still runs.  pdl_wait() returns once the predecessor grid
// has completed and its writes are visible (a hardware dependency, not a spin loop);
// pdl_trigger() lets the successor be scheduled.  In a launch without the attribute both
// are no-ops.  The first kernel of a call is launched plainly, so no part of a call
// overlaps work queued before it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Padding rows: CTA slot `slot` of expert e zeroes rows offsets[e] + totals[e] + 8*slot ..
// (at most 8 rows, never past offsets[e+1]): codes 0x00, scale byte 127.  Run by the
// trailing CTAs of a payload launch (E x ceil((align-1)/8) of them).
__device__ __forceinline__ void pad_rows(int64_t pad_cta, int pad_slots, const int32_t* __restrict__ offsets,
                                         const int32_t* __restrict__ totals, int64_t hidden, uint8_t* __restrict__ q,
                                         uint8_t* __restrict__ sf) {
  const int e = (int)(pad_cta / pad_slots);
  const int slot = (int)(pad_cta - (int64_t)e * pad_slots);
  const int64_t start = (int64_t)offsets[e] + totals[e], end = offsets[e + 1];
  const int64_t ncb = hidden >> 7;
  for (int rr = 0; rr < kPadRowsPerCta; ++rr) {
    const int64_t r = start + (int64_t)slot * kPadRowsPerCta + rr;
    if (r >= end) return;
    uint4* row = reinterpret_cast<uint4*>(q + r * hidden);
    for (int64_t i = threadIdx.x; i < hidden / 16; i += blockDim.x) row[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t i = threadIdx.x; i < ncb; i += blockDim.x) sf[r * ncb + i] = 127;
  }
}

// A launch that may begin while the previous kernel in the stream finishes (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                         Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace fp8q
