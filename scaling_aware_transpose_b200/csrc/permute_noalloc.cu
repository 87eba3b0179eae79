// permute_noalloc.cu — fp8q_permute_pad_quant_noalloc: the fused permute + pad +
// quantize for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc at the point where they route tokens: a
// runtime whose memory is owned by a separate allocator they cannot reach, code that
// runs inside a region where allocation is forbidden (a real-time or pre-planned memory
// budget), or a plugin that is handed only the input and output buffers.  The ordinary
// entry point needs a small caller-provided workspace for its routing pass (per-chunk
// expert counts and bases); this variant keeps that scratch in a file-scope device
// array instead, so the caller passes only inputs and outputs.
//
// The array is fixed-size device memory of this library: every GPU that loads the
// library holds it until the process exits.  In host code its name is only a host-side
// stand-in, not a device address, so the host resolves the address with
// cudaGetSymbolAddress (with the target device current) and hands the pointer to the
// kernels.  It does so on every call: the address belongs to the module instance loaded
// in the current context, and a device reset or a second context on the same device
// loads another instance, so an address remembered per device could go stale.  Once the
// module is loaded the lookup is a host-side table search.
#include "common.cuh"
#include "launch.h"

namespace {

static __device__ __align__(256) unsigned char g_permute_scratch[FP8Q_NOALLOC_SCRATCH_BYTES];

// Device address of g_permute_scratch in the current context; nullptr if the runtime
// call fails.
void* scratch_in_current_context() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace

extern "C" fp8q_status fp8q_permute_pad_quant_noalloc(const void* x, int64_t tokens, int64_t hidden,
                                                      const int32_t* topk_idx, int32_t topk, int32_t num_experts,
                                                      int32_t align, uint8_t* q, uint8_t* sf, int64_t max_out_rows,
                                                      int32_t* expert_offsets, int32_t* row_id_map,
                                                      fp8q_stream_t stream) {
  // Size limits first, so that an oversized request fails before any CUDA call; the
  // token-slot count is bounded before anything multiplies it.
  if (tokens > 0 && topk >= 1 && tokens > (int64_t)0x7FFFFFFF / topk) return FP8Q_ERR_SHAPE;
  if (tokens > 0 && topk >= 1 && num_experts >= 1 &&
      fp8q_permute_workspace_bytes(tokens, topk, num_experts) > (size_t)FP8Q_NOALLOC_SCRATCH_BYTES)
    return FP8Q_ERR_ARG;
  // Remaining argument checks that do not depend on the scratch pointer: identical to
  // the allocating entry point, which is then called with the static scratch.  The
  // routing kernels write every scratch word before reading it (counts, then bases and
  // totals), so nothing has to be cleared between calls.
  void* scratch = nullptr;
  if (tokens > 0) {
    scratch = scratch_in_current_context();
    if (scratch == nullptr) return FP8Q_ERR_CUDA;
  }
  return fp8q_permute_pad_quant(x, tokens, hidden, topk_idx, topk, num_experts, align, q, sf, max_out_rows,
                                expert_offsets, row_id_map, scratch, (size_t)FP8Q_NOALLOC_SCRATCH_BYTES, stream);
}
