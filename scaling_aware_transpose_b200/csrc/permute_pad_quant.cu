// permute_pad_quant.cu — fused MoE permute + padding + row-wise FP8 quantization.
//
// FP8-Flow-MoE review, 核心方法 (Fused Permute+Padding): expert reordering and padding
// of each expert's segment to an alignment are merged into one pass; DeepSeek FP8 §5.6:
// the grouped GEMM reads the experts' rows concatenated along M (contiguous groups).
// Each source token is read once, its 1x128 tiles quantized once, and the codes written
// to its top-k destination rows.  Pairs (token t, slot s) go to expert topk_idx[t, s] in
// (t, s) row-major order; each expert segment is padded with zero rows (codes 0, scale
// byte 127) to a multiple of `align`.
//
// Launches: (1) per-chunk expert histograms, (2) one CTA scans them into padded expert
// offsets and per-chunk bases, (3) one warp per chunk assigns stable ranks with
// __match_any_sync, (4) the streaming scatter-quantize over all (token, tile) pairs,
// (5) zero-fill of the padding rows.  Workspace: counts[C][E], bases[C][E], totals[E].
#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr int kChunk = 1024;  // (t, s) pairs per chunk, in row-major order
constexpr int kMaxExperts = 4096;

int64_t num_chunks(int64_t tokens, int32_t topk) { return (tokens * topk + kChunk - 1) / kChunk; }

__global__ void __launch_bounds__(256) count_kernel(const int32_t* __restrict__ idx, int64_t npairs, int E,
                                                    int32_t* __restrict__ counts, int* status) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t p0 = (int64_t)blockIdx.x * kChunk;
  for (int i = threadIdx.x; i < kChunk; i += blockDim.x) {
    const int64_t p = p0 + i;
    if (p >= npairs) break;
    const int32_t e = __ldg(idx + p);
    if (e < 0 || e >= E) {
      record_status(status, FP8Q_ERR_DEVICE);
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One CTA: totals, padded exclusive scan into expert offsets, per-chunk bases.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ counts, int64_t C, int E, int align,
                                                    int32_t* __restrict__ offsets, int32_t* __restrict__ bases,
                                                    int32_t* __restrict__ totals) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  // thread tid owns experts [tid*per, (tid+1)*per)
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int64_t local = 0;
  for (int e = e0; e < e1; ++e) {
    int64_t tot = 0;
    for (int64_t c = 0; c < C; ++c) tot += counts[c * E + e];
    totals[e] = (int32_t)tot;
    local += (tot + align - 1) / align * align;
  }
  part[tid] = local;
  __syncthreads();
  // inclusive scan of part[] (Hillis-Steele)
  for (int o = 1; o < (int)blockDim.x; o <<= 1) {
    const int64_t v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int64_t run = part[tid] - local;  // exclusive prefix of this thread's experts
  for (int e = e0; e < e1; ++e) {
    offsets[e] = (int32_t)run;
    int64_t base = run;
    for (int64_t c = 0; c < C; ++c) {
      bases[c * E + e] = (int32_t)base;
      base += counts[c * E + e];
    }
    const int64_t tot = totals[e];
    run += (tot + align - 1) / align * align;
  }
  if (tid == blockDim.x - 1) offsets[E] = (int32_t)part[tid];
}

// One warp per chunk: stable destination rows in (t, s) order.
__global__ void __launch_bounds__(32) rank_kernel(const int32_t* __restrict__ idx, int64_t npairs, int E,
                                                  const int32_t* __restrict__ bases, int32_t* __restrict__ row_id_map) {
  extern __shared__ int32_t run[];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) run[e] = bases[(int64_t)blockIdx.x * E + e];
  __syncwarp();
  const int64_t p0 = (int64_t)blockIdx.x * kChunk;
  for (int i = 0; i < kChunk; i += 32) {
    const int64_t p = p0 + i + lane;
    const bool live = p < npairs;
    const int32_t e = live ? __ldg(idx + p) : -1;
    const bool ok = live && e >= 0 && e < E;
    const int32_t key = ok ? e : -1 - lane;  // invalid lanes never match anyone
    const unsigned same = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(same & ((1u << lane) - 1u));
    const int base = ok ? run[e] : 0;
    __syncwarp();
    if (ok) {
      row_id_map[p] = base + rank;
      if (rank == 0) run[e] = base + __popc(same);
    } else if (live) {
      row_id_map[p] = -1;
    }
    __syncwarp();
  }
}

__device__ __forceinline__ uint32_t absmax8_bits(const uint4& v) {
  const uint32_t m0 = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  const uint32_t m1 = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
  const uint32_t m = __vmaxu2(m0, m1);
  return max(m & 0xFFFFu, m >> 16) << 16;
}
__device__ __forceinline__ uint32_t encode4(uint32_t a, uint32_t b, float s) {
  const float f0 = __uint_as_float(a << 16) * s, f1 = __uint_as_float(a & 0xFFFF0000u) * s;
  const float f2 = __uint_as_float(b << 16) * s, f3 = __uint_as_float(b & 0xFFFF0000u) * s;
  return cvt_e4m3x2_f32(f0, f1) | (cvt_e4m3x2_f32(f2, f3) << 16);
}

constexpr int kSThreads = 256;
constexpr int kSUnroll = 4;

// Tiles of x (token t, column block j) in row-major order; 16 lanes per tile.
__global__ void __launch_bounds__(kSThreads) scatter_quant_kernel(const uint4* __restrict__ x, int64_t tokens, int ncb,
                                                                  const int32_t* __restrict__ row_id_map, int topk,
                                                                  uint2* __restrict__ q, uint8_t* __restrict__ sf) {
  const int lane = threadIdx.x & 31, sub = lane & 15;
  const int64_t n_tiles = tokens * ncb;
  const int64_t warp = ((int64_t)blockIdx.x * kSThreads + threadIdx.x) >> 5;
  int64_t tile[kSUnroll];
  uint4 v[kSUnroll];
#pragma unroll
  for (int u = 0; u < kSUnroll; ++u) {
    tile[u] = (warp * kSUnroll + u) * 2 + (lane >> 4);
    v[u] = tile[u] < n_tiles ? ld_stream(x + tile[u] * 16 + sub) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < kSUnroll; ++u) {
    uint32_t m = absmax8_bits(v[u]);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (tile[u] >= n_tiles) continue;
    const int e = tile_exponent(__uint_as_float(m));
    const float s = exp2_neg(e);
    uint2 out;
    out.x = encode4(v[u].x, v[u].y, s);
    out.y = encode4(v[u].z, v[u].w, s);
    const int64_t t = tile[u] / ncb;
    const int j = (int)(tile[u] - t * ncb);
    for (int k = 0; k < topk; ++k) {
      const int32_t row = __ldg(row_id_map + t * topk + k);
      if (row < 0) continue;
      q[((int64_t)row * ncb + j) * 16 + sub] = out;
      if (sub == 0) sf[(int64_t)row * ncb + j] = (uint8_t)(e + 127);
    }
  }
}

// grid (E, row slots): zero rows offsets[e] + totals[e] .. offsets[e+1]
constexpr int kPadRowsPerCta = 8;
__global__ void __launch_bounds__(256) pad_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ totals,
                                                  int64_t hidden, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int e = blockIdx.x;
  const int64_t start = (int64_t)offsets[e] + totals[e], end = offsets[e + 1];
  const int64_t ncb = hidden >> 7;
  for (int rr = 0; rr < kPadRowsPerCta; ++rr) {
    const int64_t r = start + (int64_t)blockIdx.y * kPadRowsPerCta + rr;
    if (r >= end) return;
    uint4* row = reinterpret_cast<uint4*>(q + r * hidden);
    for (int64_t i = threadIdx.x; i < hidden / 16; i += blockDim.x) row[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t i = threadIdx.x; i < ncb; i += blockDim.x) sf[r * ncb + i] = 127;
  }
}

}  // namespace

size_t permute_workspace_bytes(int64_t tokens, int32_t topk, int32_t num_experts) {
  const int64_t C = num_chunks(tokens, topk);
  return (size_t)(2 * C * num_experts + num_experts) * sizeof(int32_t) + 16;
}

fp8q_status launch_permute_pad_quant(const DeviceInfo& dev, const void* x, int64_t tokens, int64_t hidden,
                                     const int32_t* topk_idx, int32_t topk, int32_t num_experts, int32_t align,
                                     uint8_t* q, uint8_t* sf, int64_t max_out_rows, int32_t* expert_offsets,
                                     int32_t* row_id_map, void* workspace, cudaStream_t stream) {
  (void)max_out_rows;
  const int E = num_experts;
  if (tokens == 0) {
    return cudaMemsetAsync(expert_offsets, 0, (size_t)(E + 1) * sizeof(int32_t), stream) == cudaSuccess
               ? FP8Q_OK
               : FP8Q_ERR_CUDA;
  }
  const int64_t npairs = tokens * topk;
  const int64_t C = num_chunks(tokens, topk);
  int32_t* counts = static_cast<int32_t*>(workspace);
  int32_t* bases = counts + C * E;
  int32_t* totals = bases + C * E;
  const size_t hist_smem = (size_t)E * sizeof(int32_t);
  count_kernel<<<(unsigned)C, 256, hist_smem, stream>>>(topk_idx, npairs, E, counts, dev.status);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  scan_kernel<<<1, 1024, 0, stream>>>(counts, C, E, align, expert_offsets, bases, totals);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  rank_kernel<<<(unsigned)C, 32, hist_smem, stream>>>(topk_idx, npairs, E, bases, row_id_map);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  if (hidden == 0) return FP8Q_OK;  // routing only: offsets and row ids, no payload
  const int ncb = (int)(hidden / 128);
  const int64_t n_tiles = tokens * ncb;
  const int64_t tiles_per_block = (kSThreads / 32) * kSUnroll * 2;
  scatter_quant_kernel<<<(unsigned)((n_tiles + tiles_per_block - 1) / tiles_per_block), kSThreads, 0, stream>>>(
      static_cast<const uint4*>(x), tokens, ncb, row_id_map, topk, reinterpret_cast<uint2*>(q), sf);
  if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  if (align > 1) {
    dim3 grid((unsigned)E, (unsigned)((align - 1 + kPadRowsPerCta - 1) / kPadRowsPerCta));
    pad_kernel<<<grid, 256, 0, stream>>>(expert_offsets, totals, hidden, q, sf);
    if (cudaGetLastError() != cudaSuccess) return FP8Q_ERR_CUDA;
  }
  return FP8Q_OK;
}

}  // namespace fp8q
