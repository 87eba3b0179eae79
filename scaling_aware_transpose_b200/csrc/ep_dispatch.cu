// ep_dispatch.cu — expert-parallel FP8 dispatch: the send-side pack of one source rank
// and the receive-side permute of one destination rank.
//
// FP8-Flow-MoE review, 核心方法 and Table 1: the all-to-all dispatch carries row-wise FP8
// codes with their scale metadata instead of BF16 rows (about 1.6x less time on the
// wire), and the receiving side feeds the experts' grouped GEMM, which reads each
// expert's rows as one contiguous, aligned group (DeepSeek FP8 §5.6).
//
// Send side: each token goes once to every rank holding one of its experts.  The pack
// is the permute's routing run over (token, destination rank) pairs with one group per
// rank and alignment 1 — pair (t, d) present iff some slot of t has its expert on d —
// followed by the FP8 payload copy into the rank-grouped send buffer and one small
// kernel that writes each sent row's slot ids re-expressed for its destination rank
// (local expert id, or -1).
//
// Receive side: the rows arrive as one segment per source rank (for example the
// segments of an all-to-all receive buffer).  The kernel reads them where they lie,
// through a table of segment pointers passed as a kernel parameter, and writes each row
// straight into its expert groups: no concatenation or unpacking pass.  Routing: the
// slot ids of all segments are gathered into one array (4 bytes per slot, a small
// fraction of the rows' bytes) and routed with -1 meaning "expert on another rank";
// payload: tiles (row, 128-column block) of each segment, 8 lanes per tile, CTAs
// assigned to segments by a prefix over the segments' CTA counts.
#include "launch.h"
#include "permute_common.cuh"

namespace fp8q {
namespace {

constexpr int kMaxRanks = FP8Q_EP_MAX_RANKS;

// The receive side's segment table, passed by value as a __grid_constant__ parameter.
struct SegmentTable {
  const uint4* q[kMaxRanks];
  const uint8_t* sf[kMaxRanks];
  const int32_t* ids[kMaxRanks];
  int64_t row_start[kMaxRanks + 1];  // prefix of the segments' rows
  int64_t cta_start[kMaxRanks + 1];  // prefix of the segments' payload CTAs
  int n;
};

// Largest i in [0, n) with start[i] <= x, for non-decreasing start[0..n] with
// start[0] <= x < start[n]: the segment holding x (never an empty one).
__device__ __forceinline__ int segment_of(const int64_t* start, int n, int64_t x) {
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (start[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// Pair (t, d) of the send-side routing: d if some slot of token t has its expert on rank
// d, else -1; the d == 0 thread of each token checks the ids.  Fused with the routing's
// first step: each CTA takes one chunk of kChunk pairs (p = t*W + d, row-major) and also
// writes that chunk's per-destination pair counts, the histogram layout the rank kernels
// read (counts[chunk][d]).  One thread per pair.
__global__ void __launch_bounds__(kChunk) dest_count_kernel(const int32_t* __restrict__ idx, int64_t tokens, int K,
                                                             int W, int Eloc, int32_t* __restrict__ didx,
                                                             int32_t* __restrict__ counts, int* status) {
  extern __shared__ int32_t hist[];  // W entries
  pdl_wait_for(idx);
  pdl_trigger();
  for (int e = threadIdx.x; e < W; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t npairs = tokens * W;
  const int64_t E = (int64_t)W * Eloc;
  const int64_t p0 = (int64_t)blockIdx.x * kChunk;
  for (int i = threadIdx.x; i < kChunk; i += blockDim.x) {
    const int64_t p = p0 + i;
    if (p >= npairs) break;
    const int64_t t = p / W;
    const int d = (int)(p - t * W);
    bool hit = false, bad = false;
    for (int k = 0; k < K; ++k) {
      const int32_t e = ld_g(idx + t * K + k);
      if (e < 0 || e >= E) {
        bad = true;
        continue;
      }
      hit |= e / Eloc == d;
    }
    if (bad && d == 0) record_status(status, FP8Q_ERR_DEVICE);
    didx[p] = hit ? d : -1;
    if (hit) atomicAdd(&hist[d], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < W; e += blockDim.x) counts[(int64_t)blockIdx.x * W + e] = hist[e];
}

// Slot ids of each sent row, re-expressed for its destination rank.  A dependent launch
// after the routing: it waits for the send map before reading it.
__global__ void __launch_bounds__(256) send_ids_kernel(const int32_t* __restrict__ idx, int64_t tokens, int K, int W,
                                                       int Eloc, const int32_t* __restrict__ send_map,
                                                       int32_t* __restrict__ send_ids, int64_t max_rows) {
  pdl_trigger();
  pdl_wait_for(send_map, idx);
  const int64_t p = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (p >= tokens * W) return;
  const int32_t row = ld_g(send_map + p);
  if (row < 0 || row >= max_rows) return;  // (never out of range for a consistent routing)
  const int64_t t = p / W;
  const int d = (int)(p - t * W);
  const int64_t E = (int64_t)W * Eloc;
  for (int k = 0; k < K; ++k) {
    const int32_t e = ld_g(idx + t * K + k);
    send_ids[(int64_t)row * K + k] = (e >= 0 && e < E && e / Eloc == d) ? e - d * Eloc : -1;
  }
}

// Received slot ids of all segments -> one array [R * K] (the routing's input).
__global__ void __launch_bounds__(256) gather_ids_kernel(const __grid_constant__ SegmentTable tab, int K,
                                                         int64_t npairs, int32_t* __restrict__ rid) {
  pdl_wait();
  pdl_trigger();
  const int64_t p = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (p >= npairs) return;
  const int64_t r = p / K;
  const int s = segment_of(tab.row_start, tab.n, r);
  const int32_t* ids = tab.ids[s];
  make_opaque(ids);  // after the wait (see pdl_wait_for)
  rid[p] = ld_g(ids + (r - tab.row_start[s]) * K + (p - r * K));
}

// Payload of the receive side: the CTAs of segment s cover its tiles (row, column block)
// in row-major order, 8 lanes per tile, four tiles per warp per slot, all loads issued
// before the wait on the routing; each tile's codes and scale byte go to the rows of the
// row's local slots.  Trailing CTAs zero-fill the padding rows.
__global__ void __launch_bounds__(kSThreads) scatter_segments_kernel(const __grid_constant__ SegmentTable tab,
                                                                     int ncb, const int32_t* __restrict__ row_id_map,
                                                                     int topk, uint4* __restrict__ q,
                                                                     uint8_t* __restrict__ sf, int64_t scatter_ctas,
                                                                     int pad_slots,
                                                                     const int32_t* __restrict__ offsets,
                                                                     const int32_t* __restrict__ totals,
                                                                     int64_t max_rows) {
  if ((int64_t)blockIdx.x >= scatter_ctas) {
    pdl_wait_for(offsets, totals);  // the offsets
    pad_rows((int64_t)blockIdx.x - scatter_ctas, pad_slots, offsets, totals, (int64_t)ncb * 128,
             reinterpret_cast<uint8_t*>(q), sf, max_rows);
    return;
  }
  const int s = segment_of(tab.cta_start, tab.n, (int64_t)blockIdx.x);
  const uint4* __restrict__ xq = tab.q[s];
  const uint8_t* __restrict__ xsf = tab.sf[s];
  const int64_t r0 = tab.row_start[s];
  const int64_t n_tiles = (tab.row_start[s + 1] - r0) * ncb;
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int64_t warp = (((int64_t)blockIdx.x - tab.cta_start[s]) * kSThreads + threadIdx.x) >> 5;
  int64_t tile[kSUnroll];
  uint4 v[kSUnroll];
  uint8_t e[kSUnroll];
#pragma unroll
  for (int u = 0; u < kSUnroll; ++u) {
    tile[u] = (warp * kSUnroll + u) * 4 + (lane >> 3);
    v[u] = make_uint4(0u, 0u, 0u, 0u);
    e[u] = 0;
    if (tile[u] < n_tiles) {
      v[u] = ld_stream(xq + tile[u] * 8 + sub);
      if (sub == 0) e[u] = ld_g(xsf + tile[u]);
    }
  }
  pdl_wait_for(row_id_map);  // the row ids
#pragma unroll
  for (int u = 0; u < kSUnroll; ++u) {
    if (tile[u] >= n_tiles) continue;
    const int64_t t = tile[u] / ncb;
    const int j = (int)(tile[u] - t * ncb);
    const int32_t* ids = row_id_map + (r0 + t) * topk;
    for (int k = 0; k < topk; ++k) {
      const int32_t row = ld_g(ids + k);
      if (row < 0 || row >= max_rows) continue;  // (never out of range for a consistent routing)
      q[((int64_t)row * ncb + j) * 8 + sub] = v[u];
      if (sub == 0) sf[(int64_t)row * ncb + j] = e[u];
    }
  }
}

constexpr int64_t kMaxDim = 0x7FFFFFFFll;
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline size_t round16(size_t b) { return (b + 15) & ~(size_t)15; }

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" size_t fp8q_ep_pack_workspace_bytes(int64_t tokens, int32_t num_ranks) {
  if (tokens < 0 || num_ranks < 1 || num_ranks > kMaxRanks || tokens > kMaxDim / num_ranks) return 0;
  return round16((size_t)(tokens * num_ranks) * sizeof(int32_t)) + permute_workspace_bytes(tokens, num_ranks,
                                                                                            num_ranks);
}

extern "C" size_t fp8q_ep_recv_workspace_bytes(int64_t rows, int32_t topk, int32_t experts_per_rank) {
  if (rows < 0 || topk < 1 || experts_per_rank < 1 || rows > kMaxDim / topk) return 0;
  return round16((size_t)(rows * topk) * sizeof(int32_t)) + permute_workspace_bytes(rows, topk, experts_per_rank);
}

extern "C" fp8q_status fp8q_ep_dispatch_pack(const uint8_t* xq, const uint8_t* xsf, int64_t tokens, int64_t hidden,
                                             const int32_t* topk_idx, int32_t topk, int32_t num_ranks,
                                             int32_t experts_per_rank, uint8_t* send_q, uint8_t* send_sf,
                                             int32_t* send_ids, int64_t max_send_rows, int32_t* send_offsets,
                                             int32_t* send_map, void* workspace, size_t workspace_bytes,
                                             fp8q_stream_t stream) {
  const int W = num_ranks, K = topk, Eloc = experts_per_rank;
  if (tokens < 0 || hidden < 0 || hidden % 128 || hidden > kMaxDim) return FP8Q_ERR_SHAPE;
  if (K < 1 || K > 64 || W < 1 || W > kMaxRanks || Eloc < 1 || Eloc > 4096) return FP8Q_ERR_ARG;
  if (tokens > kMaxDim / W || tokens > kMaxDim / K) return FP8Q_ERR_SHAPE;
  if (max_send_rows < tokens * (W < K ? W : K) || max_send_rows > kMaxDim) return FP8Q_ERR_ARG;
  if (!send_offsets) return FP8Q_ERR_NULL;
  if (!aligned4(send_offsets)) return FP8Q_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (tokens == 0)
    return cudaMemsetAsync(send_offsets, 0, (size_t)(W + 1) * sizeof(int32_t), st) == cudaSuccess ? FP8Q_OK
                                                                                                  : FP8Q_ERR_CUDA;
  if (!topk_idx || !send_map || !send_ids || !workspace) return FP8Q_ERR_NULL;
  if (!aligned4(topk_idx) || !aligned4(send_map) || !aligned4(send_ids) || !aligned16(workspace))
    return FP8Q_ERR_ALIGN;
  if (workspace_bytes < fp8q_ep_pack_workspace_bytes(tokens, W)) return FP8Q_ERR_ARG;
  if (hidden > 0) {
    if (!xq || !xsf || !send_q || !send_sf) return FP8Q_ERR_NULL;
    if (!aligned16(xq) || !aligned16(send_q)) return FP8Q_ERR_ALIGN;
  }
  DeviceInfo dev;
  if (device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  int32_t* didx = static_cast<int32_t*>(workspace);
  void* route_ws = static_cast<uint8_t*>(workspace) + round16((size_t)(tokens * W) * sizeof(int32_t));
  const int64_t npairs = tokens * W;
  if (launch_after(dest_count_kernel, dim3((unsigned)num_chunks(tokens, W)), kChunk, (size_t)W * sizeof(int32_t), st,
                   topk_idx, tokens, (int)K, (int)W, (int)Eloc, didx, static_cast<int32_t*>(route_ws),
                   dev.status) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  fp8q_status rs = route_ranks(dev, tokens, didx, W, W, 1, send_offsets, send_map, route_ws, true, st);
  if (rs != FP8Q_OK) return rs;
  // The slot ids need only the send map; launched before the payload (both as dependent
  // launches), so the payload's loads overlap them.
  const int32_t* smap = send_map;
  if (launch_after(send_ids_kernel, (unsigned)((npairs + 255) / 256), 256, 0, st, topk_idx, tokens, K, W, Eloc, smap,
                   send_ids, max_send_rows) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (hidden > 0)
    return launch_scatter_copy(xq, xsf, tokens, hidden, send_map, W, W, 1, send_q, send_sf, max_send_rows,
                               send_offsets, route_totals(route_ws, tokens, W, W), st);
  return FP8Q_OK;
}

extern "C" fp8q_status fp8q_ep_recv_permute_fp8(const fp8q_ep_source* sources, int32_t num_sources, int64_t hidden,
                                                int32_t topk, int32_t experts_per_rank, int32_t align, uint8_t* q,
                                                uint8_t* sf, int64_t max_out_rows, int32_t* expert_offsets,
                                                int32_t* row_id_map, void* workspace, size_t workspace_bytes,
                                                fp8q_stream_t stream) {
  const int K = topk, Eloc = experts_per_rank;
  if (hidden < 0 || hidden % 128 || hidden > kMaxDim) return FP8Q_ERR_SHAPE;
  if (num_sources < 1 || num_sources > kMaxRanks || K < 1 || K > 64 || Eloc < 1 || Eloc > 4096 || align < 1 ||
      align > 4096)
    return FP8Q_ERR_ARG;
  if (!sources) return FP8Q_ERR_NULL;
  const int ncb = (int)(hidden / 128);
  const int64_t tiles_per_cta = (kSThreads / 32) * kSUnroll * 4;
  SegmentTable tab = {};
  tab.n = num_sources;
  int64_t R = 0, ctas = 0;
  for (int s = 0; s < num_sources; ++s) {
    const fp8q_ep_source& src = sources[s];
    if (src.rows < 0 || src.rows > kMaxDim) return FP8Q_ERR_SHAPE;
    tab.row_start[s] = R;
    tab.cta_start[s] = ctas;
    R += src.rows;
    if (R > kMaxDim / K) return FP8Q_ERR_SHAPE;  // row ids are int32: R*topk must fit
    if (src.rows > 0) {
      if (!src.ids) return FP8Q_ERR_NULL;
      if (!aligned4(src.ids)) return FP8Q_ERR_ALIGN;
      if (hidden > 0) {
        if (!src.q || !src.sf) return FP8Q_ERR_NULL;
        if (!aligned16(src.q)) return FP8Q_ERR_ALIGN;
      }
      ctas += (src.rows * ncb + tiles_per_cta - 1) / tiles_per_cta;
    }
    tab.q[s] = reinterpret_cast<const uint4*>(src.q);
    tab.sf[s] = src.sf;
    tab.ids[s] = src.ids;
  }
  tab.row_start[num_sources] = R;
  tab.cta_start[num_sources] = ctas;
  const int64_t need = R * K + (int64_t)Eloc * (align - 1);
  if (max_out_rows < need || max_out_rows > kMaxDim) return FP8Q_ERR_ARG;
  if (!expert_offsets) return FP8Q_ERR_NULL;
  if (!aligned4(expert_offsets)) return FP8Q_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (R == 0)
    return cudaMemsetAsync(expert_offsets, 0, (size_t)(Eloc + 1) * sizeof(int32_t), st) == cudaSuccess
               ? FP8Q_OK
               : FP8Q_ERR_CUDA;
  if (!row_id_map || !workspace) return FP8Q_ERR_NULL;
  if (!aligned4(row_id_map) || !aligned16(workspace)) return FP8Q_ERR_ALIGN;
  if (workspace_bytes < fp8q_ep_recv_workspace_bytes(R, K, Eloc)) return FP8Q_ERR_ARG;
  if (hidden > 0 && (!q || !sf)) return FP8Q_ERR_NULL;
  if (hidden > 0 && !aligned16(q)) return FP8Q_ERR_ALIGN;
  DeviceInfo dev;
  if (device_info(&dev) != FP8Q_OK) return FP8Q_ERR_CUDA;
  int32_t* rid = static_cast<int32_t*>(workspace);
  void* route_ws = static_cast<uint8_t*>(workspace) + round16((size_t)(R * K) * sizeof(int32_t));
  const int64_t npairs = R * K;
  if (launch_after(gather_ids_kernel, dim3((unsigned)((npairs + 255) / 256)), 256, 0, st, tab, (int)K, npairs, rid) !=
      cudaSuccess)
    return FP8Q_ERR_CUDA;
  fp8q_status rs = route_pairs(dev, R, rid, K, Eloc, align, true, expert_offsets, row_id_map, route_ws, st);
  if (rs != FP8Q_OK || hidden == 0) return rs;
  const int pad_slots = (align - 1 + kPadRowsPerCta - 1) / kPadRowsPerCta;
  const int64_t blocks = ctas + (int64_t)Eloc * pad_slots;
  if (blocks > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const int32_t* rmap = row_id_map;
  const int32_t* offs = expert_offsets;
  const int32_t* tots = route_totals(route_ws, R, K, Eloc);
  const cudaError_t rc = launch_after(scatter_segments_kernel, (unsigned)blocks, kSThreads, 0, st, tab, ncb, rmap, K,
                                      reinterpret_cast<uint4*>(q), sf, ctas, pad_slots, offs, tots, max_out_rows);
  return rc == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}
