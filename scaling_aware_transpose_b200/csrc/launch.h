// launch.h — internal (host-side) launchers shared between the C-ABI entry points.
// Not part of the public ABI; arguments are assumed validated by the caller.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fp8q.h"

namespace fp8q {

struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int max_smem_optin = 0;
  int* status = nullptr;  // device address of the status word
};
// Per-device facts, queried once per device and cached; also resolves the status
// word's device address with the device current.
fp8q_status device_info(DeviceInfo* out);

// Row-wise quantization of n_tiles consecutive 128-element bf16 tiles:
// x[n_tiles*128] -> q[n_tiles*128], sf[n_tiles].  With limit_rows (a device int32),
// only the first limit_rows[0] * tiles_per_row tiles are processed.
cudaError_t launch_quantize_tiles(const void* x, int64_t n_tiles, uint8_t* q, uint8_t* sf, cudaStream_t stream,
                                  const int32_t* limit_rows = nullptr, int64_t tiles_per_row = 0);

fp8q_status launch_direct_transpose(const DeviceInfo& dev, const uint8_t* q, const uint8_t* sf, int64_t rows,
                                    int64_t cols, const int32_t* offsets, int32_t num_groups, uint8_t* qt,
                                    uint8_t* sft, cudaStream_t stream);

fp8q_status launch_naive_transpose(const DeviceInfo& dev, const uint8_t* q, const uint8_t* sf, int64_t rows,
                                   int64_t cols, const int32_t* offsets, int32_t num_groups, uint8_t* qt,
                                   uint8_t* sft, void* workspace, cudaStream_t stream);

fp8q_status launch_swiglu_quant(const DeviceInfo& dev, const void* gate, const void* up, int64_t rows, int64_t cols,
                                uint8_t* q, uint8_t* sf, uint8_t* qt, uint8_t* sft, cudaStream_t stream);

fp8q_status launch_quantize_rowwise_colwise(const DeviceInfo& dev, const void* x, int64_t rows, int64_t cols,
                                            uint32_t flags, uint8_t* q, void* sf, uint8_t* qt, void* sft,
                                            cudaStream_t stream);

size_t permute_workspace_bytes(int64_t tokens, int32_t topk, int32_t num_experts);
// Routing of rows x slots pairs (idx [rows, slots], ids in [0, E)) to E groups: counts,
// offsets of the groups padded to `align`, stable (row, slot) row ids.  With allow_drop
// an id of -1 gives row id -1 and no row.  workspace >= permute_workspace_bytes(rows,
// slots, E); route_totals() points at the per-group pair counts inside it.
fp8q_status route_pairs(const DeviceInfo& dev, int64_t rows, const int32_t* idx, int32_t slots, int32_t E,
                        int32_t align, bool allow_drop, int32_t* offsets, int32_t* row_id_map, void* workspace,
                        cudaStream_t stream);
// The part of route_pairs after its histogram launch, for callers whose own kernel wrote
// the per-chunk histograms (counts[c][e] of chunk c's kChunk pairs, at the workspace's
// start).  ids_wait: the ids were written by the kernel launched just before (the rank
// kernels then wait for it before loading them).
fp8q_status route_ranks(const DeviceInfo& dev, int64_t rows, const int32_t* idx, int32_t slots, int32_t E,
                        int32_t align, int32_t* offsets, int32_t* row_id_map, void* workspace, bool ids_wait,
                        cudaStream_t stream);
const int32_t* route_totals(const void* workspace, int64_t rows, int32_t slots, int32_t E);
// FP8 payload of a routing: row r's codes and scale bytes go to rows row_id_map[r*slots
// + s] (skipped where -1); the trailing CTAs zero-fill each group's padding rows.  A
// programmatic dependent launch: it waits for the routing kernels before reading ids.
fp8q_status launch_scatter_copy(const uint8_t* xq, const uint8_t* xsf, int64_t rows, int64_t hidden,
                                const int32_t* row_id_map, int32_t slots, int32_t E, int32_t align, uint8_t* q,
                                uint8_t* sf, int64_t max_rows, const int32_t* offsets, const int32_t* totals,
                                cudaStream_t stream);
fp8q_status launch_permute_pad_quant(const DeviceInfo& dev, const void* x, int64_t tokens, int64_t hidden,
                                     const int32_t* topk_idx, int32_t topk, int32_t num_experts, int32_t align,
                                     uint8_t* q, uint8_t* sf, int64_t max_out_rows, int32_t* expert_offsets,
                                     int32_t* row_id_map, void* workspace, cudaStream_t stream);

fp8q_status launch_unpermute_unpad(const DeviceInfo& dev, const void* y, const uint8_t* y_sf, int64_t rows,
                                   int64_t hidden, const int32_t* row_id_map, const float* weights, int64_t tokens,
                                   int32_t topk, void* out, cudaStream_t stream);

fp8q_status launch_permute_pad_fp8(const DeviceInfo& dev, const uint8_t* xq, const uint8_t* xsf, int64_t tokens,
                                   int64_t hidden, const int32_t* topk_idx, int32_t topk, int32_t num_experts,
                                   int32_t align, uint8_t* q, uint8_t* sf, int64_t max_out_rows,
                                   int32_t* expert_offsets, int32_t* row_id_map, void* workspace,
                                   cudaStream_t stream);

fp8q_status launch_quantize_mx32(const void* x, int64_t rows, int64_t cols, uint8_t* q, uint8_t* sf,
                                 cudaStream_t stream);
fp8q_status launch_direct_transpose_mx32(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t cols, uint8_t* qt,
                                         uint8_t* sft, cudaStream_t stream);

fp8q_status launch_debug_encode_range(uint32_t first, int64_t n, uint8_t* out, cudaStream_t stream);
fp8q_status launch_debug_exp_spec_range(uint32_t first, int64_t n, float* out, cudaStream_t stream);
fp8q_status launch_debug_swiglu_spec(const float* g, const float* u, int64_t n, float* y, cudaStream_t stream);
fp8q_status launch_debug_silu_bf16(const void* g, int64_t n, float* y, cudaStream_t stream);

fp8q_status launch_debug_expire_wait(const DeviceInfo& dev, uint64_t timeout_ns, cudaStream_t stream);

}  // namespace fp8q
