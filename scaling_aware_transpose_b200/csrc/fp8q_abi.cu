// fp8q_abi.cu — extern "C" entry points of libfp8q: argument checks, per-device facts,
// the device status word, and dispatch to the kernel launchers.  Every host-detectable
// error returns before any CUDA call that could touch an output.
#include <mutex>

#include "common.cuh"
#include "launch.h"

// The library's only device state: the first device-side error since the last read.
__device__ int g_fp8q_status = 0;

namespace fp8q {

fp8q_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8Q_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& d = cache[dev];
  if (d.device != dev) {
    DeviceInfo n;
    n.device = dev;
    void* p = nullptr;
    if (cudaDeviceGetAttribute(&n.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaGetSymbolAddress(&p, g_fp8q_status) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    n.status = static_cast<int*>(p);
    d = n;
  }
  *out = d;
  return FP8Q_OK;
}

// ---- bounded-wait test hook: one mbarrier nobody arrives at
__global__ void expire_wait_kernel(uint64_t timeout_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_bounded(&bar, 0u, timeout_ns)) record_status(status, FP8Q_ERR_TIMEOUT);
  }
}

// ---- encoder test hook: the E4M3 conversion every kernel uses, over raw fp32 bit patterns
__global__ void encode_range_kernel(uint32_t first, int64_t n, uint8_t* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (uint8_t)cvt_e4m3x2_f32(__uint_as_float(first + (uint32_t)i), 0.0f);
}

fp8q_status launch_debug_encode_range(uint32_t first, int64_t n, uint8_t* out, cudaStream_t stream) {
  if (n <= 0) return FP8Q_OK;
  encode_range_kernel<<<1184, 256, 0, stream>>>(first, n, out);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

fp8q_status launch_debug_expire_wait(const DeviceInfo& dev, uint64_t timeout_ns, cudaStream_t stream) {
  expire_wait_kernel<<<1, 32, 0, stream>>>(timeout_ns, dev.status);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(fp8q_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }
constexpr int64_t kMaxDim = 0x7FFFFFFFll;  // grid sizes, group offsets and row ids are int32

// Shape rules shared by the two transposes.
fp8q_status check_transpose_args(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t cols,
                                 const int32_t* offsets, int32_t num_groups, const uint8_t* qt, const uint8_t* sft) {
  if (rows < 0 || cols < 0 || cols % 128 || rows > kMaxDim || cols > kMaxDim) return FP8Q_ERR_SHAPE;
  if (num_groups < 1 || (offsets == nullptr && num_groups != 1)) return FP8Q_ERR_ARG;
  if (offsets == nullptr && rows % 128) return FP8Q_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  if (!q || !sf || !qt || !sft) return FP8Q_ERR_NULL;
  if (!aligned16(q) || !aligned16(qt) || (offsets && (reinterpret_cast<uintptr_t>(offsets) & 3u))) return FP8Q_ERR_ALIGN;
  return FP8Q_OK;
}

// Rules shared by the two permutes (BF16 input x, or FP8 input x = codes with scales xsf).
fp8q_status check_permute_args(const void* x, const uint8_t* xsf, bool fp8_input, int64_t tokens, int64_t hidden,
                               const int32_t* topk_idx, int32_t topk, int32_t num_experts, int32_t align,
                               const uint8_t* q, const uint8_t* sf, int64_t max_out_rows,
                               const int32_t* expert_offsets, const int32_t* row_id_map, const void* workspace,
                               size_t workspace_bytes) {
  if (tokens < 0 || hidden < 0 || hidden % 128 || hidden > kMaxDim) return FP8Q_ERR_SHAPE;
  if (topk < 1 || topk > 64 || num_experts < 1 || num_experts > 4096 || align < 1 || align > 4096) return FP8Q_ERR_ARG;
  if (tokens > kMaxDim / topk) return FP8Q_ERR_SHAPE;  // row ids are int32: tokens*topk must fit
  const int64_t need = tokens * topk + (int64_t)num_experts * (align - 1);
  if (max_out_rows < need || max_out_rows > kMaxDim) return FP8Q_ERR_ARG;
  if (!expert_offsets) return FP8Q_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(expert_offsets) & 3u)) return FP8Q_ERR_ALIGN;
  if (tokens > 0) {
    if (!topk_idx || !row_id_map || !workspace) return FP8Q_ERR_NULL;
    if (!aligned16(workspace) || (reinterpret_cast<uintptr_t>(topk_idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(row_id_map) & 3u))
      return FP8Q_ERR_ALIGN;
    if (workspace_bytes < fp8q_permute_workspace_bytes(tokens, topk, num_experts)) return FP8Q_ERR_ARG;
    if (hidden > 0) {
      if (!x || !q || !sf || (fp8_input && !xsf)) return FP8Q_ERR_NULL;
      if (!aligned16(x) || !aligned16(q)) return FP8Q_ERR_ALIGN;
    }
  }
  return FP8Q_OK;
}

}  // namespace

extern "C" {

const char* fp8q_status_string(fp8q_status s) {
  switch (s) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_NULL: return "a required pointer is NULL";
    case FP8Q_ERR_SHAPE: return "sizes violate the layout rules";
    case FP8Q_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case FP8Q_ERR_ARG: return "invalid argument";
    case FP8Q_ERR_CUDA: return "a CUDA call failed";
    case FP8Q_ERR_TIMEOUT: return "a bounded device wait expired";
    case FP8Q_ERR_DEVICE: return "a kernel saw invalid data";
  }
  return "unknown status";
}

fp8q_status fp8q_debug_e4m3_encode_range(uint32_t first_bits, int64_t n, uint8_t* out, fp8q_stream_t stream) {
  if (n < 0 || n > (int64_t)1 << 32 || (int64_t)first_bits + n > (int64_t)1 << 32) return FP8Q_ERR_ARG;
  if (n == 0) return FP8Q_OK;
  if (!out) return FP8Q_ERR_NULL;
  return fp8q::launch_debug_encode_range(first_bits, n, out, as_stream(stream));
}

fp8q_status fp8q_debug_exp_spec_range(uint32_t first_bits, int64_t n, float* out, fp8q_stream_t stream) {
  if (n < 0 || n > (int64_t)1 << 32 || (int64_t)first_bits + n > (int64_t)1 << 32) return FP8Q_ERR_ARG;
  if (n == 0) return FP8Q_OK;
  if (!out) return FP8Q_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(out) & 3u) return FP8Q_ERR_ALIGN;
  return fp8q::launch_debug_exp_spec_range(first_bits, n, out, as_stream(stream));
}

fp8q_status fp8q_debug_swiglu_spec(const float* gate, const float* up, int64_t n, float* y, fp8q_stream_t stream) {
  if (n < 0) return FP8Q_ERR_ARG;
  if (n == 0) return FP8Q_OK;
  if (!gate || !up || !y) return FP8Q_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(gate) | reinterpret_cast<uintptr_t>(up) | reinterpret_cast<uintptr_t>(y)) & 3u)
    return FP8Q_ERR_ALIGN;
  return fp8q::launch_debug_swiglu_spec(gate, up, n, y, as_stream(stream));
}

fp8q_status fp8q_debug_silu_bf16(const void* gate, int64_t n, float* y, fp8q_stream_t stream) {
  if (n < 0 || n % 2) return FP8Q_ERR_ARG;
  if (n == 0) return FP8Q_OK;
  if (!gate || !y) return FP8Q_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(gate) & 3u) || (reinterpret_cast<uintptr_t>(y) & 7u)) return FP8Q_ERR_ALIGN;
  return fp8q::launch_debug_silu_bf16(gate, n, y, as_stream(stream));
}

int fp8q_version(void) { return 10000; }

fp8q_status fp8q_last_device_status(fp8q_stream_t stream) {
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return FP8Q_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, dev.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (v != 0 && cudaMemset(dev.status, 0, sizeof(int)) != cudaSuccess) return FP8Q_ERR_CUDA;
  return static_cast<fp8q_status>(v);
}

fp8q_status fp8q_quantize_rowwise(const void* x, int64_t rows, int64_t cols, uint8_t* q, uint8_t* sf,
                                  fp8q_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 128) return FP8Q_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  if (!x || !q || !sf) return FP8Q_ERR_NULL;
  if (!aligned16(x) || !aligned16(q)) return FP8Q_ERR_ALIGN;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_quantize_tiles(x, rows * (cols / 128), q, sf, as_stream(stream)) == cudaSuccess ? FP8Q_OK
                                                                                                      : FP8Q_ERR_CUDA;
}

fp8q_status fp8q_direct_transpose(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t cols,
                                  const int32_t* group_offsets, int32_t num_groups, uint8_t* qt, uint8_t* sft,
                                  fp8q_stream_t stream) {
  const fp8q_status c = check_transpose_args(q, sf, rows, cols, group_offsets, num_groups, qt, sft);
  if (c != FP8Q_OK || rows == 0 || cols == 0) return c;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_direct_transpose(dev, q, sf, rows, cols, group_offsets, num_groups, qt, sft, as_stream(stream));
}

size_t fp8q_naive_workspace_bytes(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return (size_t)(4 * rows * cols);
}

fp8q_status fp8q_naive_transpose(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t cols,
                                 const int32_t* group_offsets, int32_t num_groups, uint8_t* qt, uint8_t* sft,
                                 void* workspace, size_t workspace_bytes, fp8q_stream_t stream) {
  const fp8q_status c = check_transpose_args(q, sf, rows, cols, group_offsets, num_groups, qt, sft);
  if (c != FP8Q_OK || rows == 0 || cols == 0) return c;
  if (!workspace) return FP8Q_ERR_NULL;
  if (!aligned16(workspace)) return FP8Q_ERR_ALIGN;
  if (workspace_bytes < fp8q_naive_workspace_bytes(rows, cols)) return FP8Q_ERR_ARG;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_naive_transpose(dev, q, sf, rows, cols, group_offsets, num_groups, qt, sft, workspace,
                                      as_stream(stream));
}

fp8q_status fp8q_swiglu_quant(const void* gate, const void* up, int64_t rows, int64_t cols, uint8_t* q, uint8_t* sf,
                              uint8_t* qt, uint8_t* sft, fp8q_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 128 || rows > kMaxDim || cols > kMaxDim) return FP8Q_ERR_SHAPE;
  if ((qt == nullptr) != (sft == nullptr)) return FP8Q_ERR_ARG;
  if (qt && rows % 128) return FP8Q_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  if (!gate || !up || !q || !sf) return FP8Q_ERR_NULL;
  if (!aligned16(gate) || !aligned16(up) || !aligned16(q) || (qt && (reinterpret_cast<uintptr_t>(qt) & 3u)))
    return FP8Q_ERR_ALIGN;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_swiglu_quant(dev, gate, up, rows, cols, q, sf, qt, sft, as_stream(stream));
}

size_t fp8q_packed_sf_bytes(int64_t mn, int64_t k) {
  if (mn <= 0 || k <= 0) return 0;
  return (size_t)(4 * ((k / 128 + 3) / 4) * ((mn + 3) / 4 * 4));
}

fp8q_status fp8q_quantize_rowwise_colwise(const void* x, int64_t rows, int64_t cols, uint32_t flags, uint8_t* q,
                                          void* sf, uint8_t* qt, void* sft, fp8q_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 128 || rows > kMaxDim || cols > kMaxDim) return FP8Q_ERR_SHAPE;
  if (flags & ~(FP8Q_ZERO_TILE_MIN_SCALE | FP8Q_SF_PACKED_UE8M0)) return FP8Q_ERR_ARG;
  if ((qt == nullptr) != (sft == nullptr)) return FP8Q_ERR_ARG;
  if (qt && rows % 128) return FP8Q_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  if (!x || !q || !sf) return FP8Q_ERR_NULL;
  const bool packed = (flags & FP8Q_SF_PACKED_UE8M0) != 0;
  const uintptr_t sf_mask = packed ? 3u : 0u;
  if (!aligned16(x) || !aligned16(q) || (qt && !aligned16(qt)) || (reinterpret_cast<uintptr_t>(sf) & sf_mask) ||
      (reinterpret_cast<uintptr_t>(sft) & sf_mask))
    return FP8Q_ERR_ALIGN;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_quantize_rowwise_colwise(dev, x, rows, cols, flags, q, sf, qt, sft, as_stream(stream));
}

size_t fp8q_permute_workspace_bytes(int64_t tokens, int32_t topk, int32_t num_experts) {
  if (tokens < 0 || topk < 1 || num_experts < 1 || tokens > kMaxDim / topk) return 0;
  return fp8q::permute_workspace_bytes(tokens, topk, num_experts);
}

fp8q_status fp8q_permute_pad_quant(const void* x, int64_t tokens, int64_t hidden, const int32_t* topk_idx,
                                   int32_t topk, int32_t num_experts, int32_t align, uint8_t* q, uint8_t* sf,
                                   int64_t max_out_rows, int32_t* expert_offsets, int32_t* row_id_map,
                                   void* workspace, size_t workspace_bytes, fp8q_stream_t stream) {
  const fp8q_status c = check_permute_args(x, nullptr, false, tokens, hidden, topk_idx, topk, num_experts, align, q, sf,
                                           max_out_rows, expert_offsets, row_id_map, workspace, workspace_bytes);
  if (c != FP8Q_OK) return c;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_permute_pad_quant(dev, x, tokens, hidden, topk_idx, topk, num_experts, align, q, sf, max_out_rows,
                                        expert_offsets, row_id_map, workspace, as_stream(stream));
}

fp8q_status fp8q_permute_pad_fp8(const uint8_t* xq, const uint8_t* xsf, int64_t tokens, int64_t hidden,
                                 const int32_t* topk_idx, int32_t topk, int32_t num_experts, int32_t align, uint8_t* q,
                                 uint8_t* sf, int64_t max_out_rows, int32_t* expert_offsets, int32_t* row_id_map,
                                 void* workspace, size_t workspace_bytes, fp8q_stream_t stream) {
  const fp8q_status c = check_permute_args(xq, xsf, true, tokens, hidden, topk_idx, topk, num_experts, align, q, sf,
                                           max_out_rows, expert_offsets, row_id_map, workspace, workspace_bytes);
  if (c != FP8Q_OK) return c;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_permute_pad_fp8(dev, xq, xsf, tokens, hidden, topk_idx, topk, num_experts, align, q, sf,
                                      max_out_rows, expert_offsets, row_id_map, workspace, as_stream(stream));
}

fp8q_status fp8q_unpermute_unpad(const void* y, const uint8_t* y_sf, int64_t rows, int64_t hidden,
                                 const int32_t* row_id_map, const float* weights, int64_t tokens, int32_t topk,
                                 void* out, fp8q_stream_t stream) {
  if (rows < 0 || hidden < 0 || tokens < 0 || hidden % 128 || rows > kMaxDim || hidden > kMaxDim) return FP8Q_ERR_SHAPE;
  if (topk < 1 || topk > 64) return FP8Q_ERR_ARG;
  if (tokens == 0 || hidden == 0) return FP8Q_OK;
  if (!y || !row_id_map || !out) return FP8Q_ERR_NULL;
  if (!aligned16(y) || !aligned16(out) || (reinterpret_cast<uintptr_t>(row_id_map) & 3u) ||
      (reinterpret_cast<uintptr_t>(weights) & 3u))
    return FP8Q_ERR_ALIGN;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_unpermute_unpad(dev, y, y_sf, rows, hidden, row_id_map, weights, tokens, topk, out,
                                      as_stream(stream));
}

fp8q_status fp8q_quantize_rowwise_mx32(const void* x, int64_t rows, int64_t cols, uint8_t* q, uint8_t* sf,
                                       fp8q_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 32 || rows > kMaxDim || cols > kMaxDim) return FP8Q_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  if (!x || !q || !sf) return FP8Q_ERR_NULL;
  if (!aligned16(x) || !aligned16(q)) return FP8Q_ERR_ALIGN;
  return fp8q::launch_quantize_mx32(x, rows, cols, q, sf, as_stream(stream));
}

fp8q_status fp8q_direct_transpose_mx32(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t cols, uint8_t* qt,
                                       uint8_t* sft, fp8q_stream_t stream) {
  if (rows < 0 || cols < 0 || rows % 128 || cols % 128 || rows > kMaxDim || cols > kMaxDim) return FP8Q_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  if (!q || !sf || !qt || !sft) return FP8Q_ERR_NULL;
  if (!aligned16(q) || !aligned16(qt) || (reinterpret_cast<uintptr_t>(sf) & 3u) || (reinterpret_cast<uintptr_t>(sft) & 3u))
    return FP8Q_ERR_ALIGN;
  return fp8q::launch_direct_transpose_mx32(q, sf, rows, cols, qt, sft, as_stream(stream));
}

fp8q_status fp8q_debug_expire_wait(uint64_t timeout_ns, fp8q_stream_t stream) {
  if (timeout_ns < 1000ull) timeout_ns = 1000ull;
  if (timeout_ns > 2000000000ull) timeout_ns = 2000000000ull;
  fp8q::DeviceInfo dev;
  if (fp8q::device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  return fp8q::launch_debug_expire_wait(dev, timeout_ns, as_stream(stream));
}

}  // extern "C"
