// naive_transpose.cu — the three-pass dequant -> transpose -> requant baseline.
//
// FP8-Flow-MoE review, 问题与动机 and 核心方法: without the scaling-aware transpose the
// column-wise copy for wgrad is made by dequantizing the row-wise FP8 tensor, transposing
// it and quantizing it again along the other dimension (the path its Fig. 1 compares
// against).  Here: (1) dequant to the BF16 backbone dtype, (2) a shared-memory tiled
// BF16 transpose, (3) the row-wise quantization kernel run over the transposed buffer,
// whose consecutive 128-element tiles are exactly the 128-token column tiles of every
// group.  Each pass is a reasonable streaming kernel; the baseline is not slowed on
// purpose.  Workspace: v [rows, cols] bf16 and vt (same size).
#include "common.cuh"
#include "launch.h"

#include <cuda_bf16.h>

namespace fp8q {
namespace {

// ---- (1) dequantize: 16 codes per thread -> 16 bf16
__global__ void __launch_bounds__(256) dequant_kernel(const uint4* __restrict__ q, const uint8_t* __restrict__ sf,
                                                      int64_t rows, int cols, const int32_t* __restrict__ offsets,
                                                      int num_groups, uint4* __restrict__ v, int* status) {
  pdl_wait_for(q, sf, offsets);
  pdl_trigger();
  const int64_t valid_rows =
      offsets ? grouped_rows(offsets, num_groups, rows, blockIdx.x == 0 && threadIdx.x == 0 ? status : nullptr) : rows;
  if (offsets != nullptr && blockIdx.x == 0) validate_groups_cta(offsets, num_groups, status);
  const int64_t n16 = valid_rows * cols / 16;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n16) return;
  const int64_t elem = i * 16;
  const int64_t r = elem / cols;
  const int h = (int)(elem - r * cols);
  const int e = (int)ld_g(sf + r * (cols >> 7) + (h >> 7)) - 127;
  // 2^e as fp32, e in [-127, 127]: 2^-127 is the subnormal 0x00400000
  const float s = e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
  const uint4 c = ld_stream(q + i);
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
  uint32_t out[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t f2 = cvt_f16x2_e4m3x2(cw[k] >> (16 * hh));
      const float lo = __half2float(__ushort_as_half((unsigned short)(f2 & 0xFFFFu))) * s;
      const float hi = __half2float(__ushort_as_half((unsigned short)(f2 >> 16))) * s;
      const __nv_bfloat16 blo = __float2bfloat16_rn(lo), bhi = __float2bfloat16_rn(hi);
      out[2 * k + hh] = (uint32_t)__bfloat16_as_ushort(blo) | ((uint32_t)__bfloat16_as_ushort(bhi) << 16);
    }
  }
  v[2 * i] = make_uint4(out[0], out[1], out[2], out[3]);
  v[2 * i + 1] = make_uint4(out[4], out[5], out[6], out[7]);
}

// ---- (2) BF16 transpose, 64x64 tiles through padded shared memory
constexpr int kT = 64;
constexpr int kPad = 2;  // halves of padding per shared row

__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t* __restrict__ v, int64_t rows, int cols,
                                                             const int32_t* __restrict__ offsets, int num_groups,
                                                             uint16_t* __restrict__ vt, int* status) {
  __shared__ uint16_t tile[kT][kT + kPad];
  pdl_wait_for(v, offsets);
  pdl_trigger();
  const int64_t valid_rows = offsets ? grouped_rows(offsets, num_groups, rows, nullptr) : rows;
  const int64_t r0 = (int64_t)blockIdx.y * kT;
  const int h0 = blockIdx.x * kT;
  if (r0 >= valid_rows) return;
  int64_t o_g = 0, M = rows;
  if (offsets && !find_group(offsets, num_groups, r0, valid_rows, o_g, M)) {
    if (threadIdx.x == 0) record_status(status, FP8Q_ERR_SHAPE);
    return;
  }
  // load 64 rows x 64 halves: thread -> (row, 8-half chunk), two passes
  for (int p = threadIdx.x; p < kT * 8; p += blockDim.x) {
    const int rr = p >> 3, ch = p & 7;
    const uint4 x = *reinterpret_cast<const uint4*>(v + (r0 + rr) * cols + h0 + ch * 8);
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      tile[rr][ch * 8 + 2 * k] = (uint16_t)(xs[k] & 0xFFFFu);
      tile[rr][ch * 8 + 2 * k + 1] = (uint16_t)(xs[k] >> 16);
    }
  }
  __syncthreads();
  // store 64 channels x 64 tokens: thread -> (channel, 8-token chunk)
  for (int p = threadIdx.x; p < kT * 8; p += blockDim.x) {
    const int hh = p >> 3, ch = p & 7;
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      o[k] = (uint32_t)tile[ch * 8 + 2 * k][hh] | ((uint32_t)tile[ch * 8 + 2 * k + 1][hh] << 16);
    uint16_t* dst = vt + (int64_t)cols * o_g + (int64_t)(h0 + hh) * M + (r0 - o_g) + ch * 8;
    *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

fp8q_status launch_naive_transpose(const DeviceInfo& dev, const uint8_t* q, const uint8_t* sf, int64_t rows,
                                   int64_t cols, const int32_t* offsets, int32_t num_groups, uint8_t* qt,
                                   uint8_t* sft, void* workspace, cudaStream_t stream) {
  if (rows == 0 || cols == 0) return FP8Q_OK;
  uint16_t* v = static_cast<uint16_t*>(workspace);
  uint16_t* vt = v + rows * cols;
  const int64_t n16 = rows * cols / 16;
  if (launch_after(dequant_kernel, dim3((unsigned)((n16 + 255) / 256)), 256, 0, stream,
                   reinterpret_cast<const uint4*>(q), sf, rows, (int)cols, offsets, (int)num_groups,
                   reinterpret_cast<uint4*>(v), dev.status) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  const dim3 grid((unsigned)(cols / kT), (unsigned)((rows + kT - 1) / kT));
  if (launch_after(transpose_bf16_kernel, grid, 256, 0, stream, (const uint16_t*)v, rows, (int)cols, offsets,
                   (int)num_groups, vt, dev.status) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  // (3) requantize the valid part of the transposed buffer; for groups the row count
  // lives on the device (offsets[num_groups]) and the kernel reads it there.
  if (launch_quantize_tiles(vt, rows * cols / 128, qt, sft, stream, offsets ? offsets + num_groups : nullptr,
                            cols / 128) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  return FP8Q_OK;
}

}  // namespace fp8q
