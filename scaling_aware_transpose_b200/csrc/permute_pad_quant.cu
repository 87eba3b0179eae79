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
// Launches: (1) per-chunk expert histograms, (2) a CTA per 32 experts scans them over the
// chunks into per-chunk bases and expert totals, (3) stable ranks within each chunk with
// __match_any_sync, eight warps per chunk, each CTA scanning the padded totals into the
// expert offsets itself (for small routings (2) is folded into (3)), (4) the streaming
// scatter-quantize over all (token, tile) pairs,
// whose trailing CTAs zero-fill the padding rows.  All are programmatic dependent
// launches (see pdl_wait): (1) waits for the previous kernel in the stream before its
// first access, (2)-(4) overlap their predecessor and wait only where they first read
// its output.  Workspace: counts[C][E], bases[C][E], totals[E].
// The FP8-input variant (the dispatch already delivered row-wise codes and scales) shares
// (1)-(3) and the padding; its step (4) copies each token's codes and scale bytes to its
// rows.
#include "launch.h"
#include "permute_common.cuh"

namespace fp8q {
namespace {

// allow_drop: an id of -1 means "not routed here" (no row, no error); any other id
// outside [0, E) records FP8Q_ERR_DEVICE.  Launched with 256 threads.
__global__ void __launch_bounds__(256) count_kernel(const int32_t* __restrict__ idx, int64_t npairs, int E,
                                                    bool allow_drop, int32_t* __restrict__ counts, int* status) {
  extern __shared__ int32_t hist[];
  pdl_wait_for(idx);
  pdl_trigger();
  const int64_t p0 = (int64_t)blockIdx.x * kChunk;
  constexpr int kPer = kChunk / 256;
  int32_t ids[kPer];  // this thread's ids, in flight while the histogram is cleared
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t p = p0 + u * 256 + threadIdx.x;
    ids[u] = p < npairs ? ld_g(idx + p) : -1;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    if (p0 + u * 256 + threadIdx.x >= npairs) break;
    const int32_t e = ids[u];
    if (e < 0 || e >= E) {
      if (!(allow_drop && e == -1)) record_status(status, FP8Q_ERR_DEVICE);
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// Inclusive warp scan of a 32-bit value.
__device__ __forceinline__ int32_t warp_incl_scan32(int32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t t = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Per-expert prefix over the chunks, for routings too large for the fused rank kernel.
// CTA b owns experts 32b..32b+31 with one lane per expert, so each chunk's 32 counts are
// one 128-byte load; its 32 warps split the chunks into contiguous ranges.  Each lane sums
// its range, the ranges' sums are scanned across the warps in shared memory, and each lane
// then walks its range again writing bases[c][e] = the pairs of expert e in chunks before
// c.  Warp 0 writes totals[e].  The padded offsets are left to the rank kernel, whose CTAs
// each scan the E totals themselves (no cross-CTA step here).
__global__ void __launch_bounds__(1024) chunk_scan_kernel(const int32_t* __restrict__ counts, int64_t C, int E,
                                                          int32_t* __restrict__ bases, int32_t* __restrict__ totals) {
  __shared__ int32_t s_part[32][32];  // [warp][lane]: the warp's range sum for the lane's expert
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  const bool live = e < E;
  const int64_t per = (C + 31) / 32;
  const int64_t c0 = min(C, w * per), c1 = min(C, c0 + per);
  pdl_trigger();
  pdl_wait_for(counts);  // the histograms
  int32_t sum = 0;
  for (int64_t c = c0; c < c1; c += 8) {
    int32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = live && c + u < c1 ? ld_g(counts + (c + u) * E + e) : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) sum += v[u];
  }
  s_part[w][lane] = sum;
  __syncthreads();
  int32_t run = 0, tot = 0;
#pragma unroll 8
  for (int ww = 0; ww < 32; ++ww) {
    const int32_t v = s_part[ww][lane];
    run += ww < w ? v : 0;
    tot += v;
  }
  if (w == 0 && live) totals[e] = tot;
  for (int64_t c = c0; c < c1; c += 8) {
    int32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = live && c + u < c1 ? ld_g(counts + (c + u) * E + e) : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (live && c + u < c1) bases[(c + u) * E + e] = run;
      run += v[u];
    }
  }
}

// Exclusive scan of the padded group sizes ceil(s[e]/align)*align over the groups by the
// whole CTA, in place: s[e] holds group e's total on entry and its offset on return.  Warp
// w takes the w-th contiguous segment of the groups: it sums the segment (lanes striding),
// the warps' sums are scanned through s_wsum (one word per warp), and the warp walks its
// segment again 32 groups per step (lane = group, so shared accesses are conflict-free)
// with a warp scan and a carry.  offsets != nullptr also stores offsets[0..E].  Ends with
// a barrier.
__device__ __forceinline__ void block_pad_offsets(int32_t* s, int32_t* s_wsum, int E, int align,
                                                  int32_t* __restrict__ offsets) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int seg = (E + nw - 1) / nw;
  const int e0 = min(E, w * seg), e1 = min(E, e0 + seg);
  int32_t acc = 0;
  for (int e = e0 + lane; e < e1; e += 32) acc += (s[e] + align - 1) / align * align;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) s_wsum[w] = acc;
  __syncthreads();
  int32_t run = 0;
  for (int ww = 0; ww < w; ++ww) run += s_wsum[ww];
  for (int eb = e0; eb < e1; eb += 32) {
    const int e = eb + lane;
    const int32_t padded = e < e1 ? (s[e] + align - 1) / align * align : 0;
    const int32_t incl = warp_incl_scan32(padded, lane);
    if (e < e1) {
      s[e] = run + incl - padded;
      if (offsets) offsets[e] = run + incl - padded;
    }
    run += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  if (offsets && w == nw - 1 && lane == 0) offsets[E] = run;  // past every segment: the grand total
  __syncthreads();
}

// Rank with 8 warps per chunk, after chunk_scan_kernel (per-warp counts in shared
// memory): warp w owns pairs 128w..128w+127 of the chunk.  (A) each warp counts its pairs
// per expert; (B) the CTA scans the padded expert totals into offsets (CTA 0 stores them)
// and, per expert, takes an exclusive prefix over the warps on top of offset + the chunk's
// base; (C) each warp ranks its pairs from its own bases, 8 serial steps per warp.  Stable
// (t, s) order.  Shared memory: 9E + 8 words (147 KB at 4096 experts, one CTA per SM).
constexpr int kRankWarps = 8;
inline size_t rank_multi_smem(int E) { return ((size_t)(kRankWarps + 1) * E + kRankWarps) * sizeof(int32_t); }
__global__ void __launch_bounds__(kRankWarps * 32) rank_multi_kernel(const int32_t* __restrict__ idx, int64_t npairs,
                                                                     int E, int align, const int32_t* __restrict__ bases,
                                                                     const int32_t* __restrict__ totals,
                                                                     int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ row_id_map, bool ids_wait) {
  extern __shared__ int32_t s_cnt[];  // [kRankWarps][E] | off[E] | warp sums[kRankWarps]
  int32_t* s_off = s_cnt + kRankWarps * E;
  int32_t* s_wsum = s_off + E;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  constexpr int kPer = kChunk / kRankWarps / 32;  // iterations per warp
  const int64_t p0 = (int64_t)blockIdx.x * kChunk + w * (kChunk / kRankWarps);
  int32_t ids[kPer];
  if (ids_wait) pdl_wait_for(idx);  // the ids were written inside this call (see route_ranks)
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t p = p0 + i * 32 + lane;
    ids[i] = p < npairs ? ld_g(idx + p) : -1;
  }
  pdl_trigger();
  for (int e = tid; e < kRankWarps * E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  int32_t* mine = s_cnt + w * E;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t p = p0 + i * 32 + lane;
    const int32_t e = ids[i];
    const bool ok = p < npairs && e >= 0 && e < E;
    const unsigned same = __match_any_sync(0xFFFFFFFFu, ok ? e : -1 - lane);
    if (ok && lane == __ffs(same) - 1) mine[e] += __popc(same);
    __syncwarp();
  }
  pdl_wait_for(bases, totals);  // the chunk bases and expert totals
  // eight loads in flight per thread in both passes (E up to 4096: 16 per thread)
  constexpr int kB = 8, kT = kRankWarps * 32;
  for (int eb = tid; eb < E; eb += kB * kT) {
    int32_t v[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) v[u] = eb + u * kT < E ? ld_g(totals + eb + u * kT) : 0;
#pragma unroll
    for (int u = 0; u < kB; ++u)
      if (eb + u * kT < E) s_off[eb + u * kT] = v[u];
  }
  __syncthreads();
  block_pad_offsets(s_off, s_wsum, E, align, blockIdx.x == 0 ? offsets : nullptr);
  const int32_t* my_bases = bases + (int64_t)blockIdx.x * E;
  for (int eb = tid; eb < E; eb += kB * kT) {
    int32_t b[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) b[u] = eb + u * kT < E ? ld_g(my_bases + eb + u * kT) : 0;
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int e = eb + u * kT;
      if (e >= E) break;
      int32_t run = s_off[e] + b[u];
#pragma unroll
      for (int ww = 0; ww < kRankWarps; ++ww) {
        const int32_t c = s_cnt[ww * E + e];
        s_cnt[ww * E + e] = run;
        run += c;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t p = p0 + i * 32 + lane;
    const bool live = p < npairs;
    const int32_t e = ids[i];
    const bool ok = live && e >= 0 && e < E;
    const unsigned same = __match_any_sync(0xFFFFFFFFu, ok ? e : -1 - lane);
    const int rank = __popc(same & ((1u << lane) - 1u));
    const int base = ok ? mine[e] : 0;
    __syncwarp();
    if (ok) {
      row_id_map[p] = base + rank;
      if (lane == __ffs(same) - 1) mine[e] = base + __popc(same);
    } else if (live) {
      row_id_map[p] = -1;
    }
    __syncwarp();
  }
}

// Rank with the scan folded in, for small routings (see route_pairs): the same stable
// ranking as rank_multi_kernel, but each CTA derives its own bases from the per-chunk
// histograms instead of reading them from chunk_scan_kernel.  A warp per group sums the group's
// counts over all chunks (its total) and over the chunks before this one (this chunk's
// prefix), lanes striding over the chunks; an exclusive scan of the padded totals over the
// groups gives the offsets.  CTA 0 also writes offsets[0..E] and the totals, which the
// payload's padding CTAs read.  The chain becomes histogram -> rank -> payload.
__global__ void __launch_bounds__(kRankWarps * 32) rank_fused_kernel(const int32_t* __restrict__ idx, int64_t npairs,
                                                                     int E, int align, const int32_t* __restrict__ counts,
                                                                     int64_t C, int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ totals,
                                                                     int32_t* __restrict__ row_id_map, bool ids_wait) {
  extern __shared__ int32_t s_cnt[];  // [kRankWarps][E] | pre[E] | tot[E] | warp sums[kRankWarps]
  int32_t* s_pre = s_cnt + kRankWarps * E;
  int32_t* s_tot = s_pre + E;
  int32_t* s_wsum = s_tot + E;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  constexpr int kPer = kChunk / kRankWarps / 32;
  const int64_t p0 = (int64_t)blockIdx.x * kChunk + w * (kChunk / kRankWarps);
  int32_t ids[kPer];
  if (ids_wait) pdl_wait_for(idx);  // the ids were written inside this call (see route_ranks)
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t p = p0 + i * 32 + lane;
    ids[i] = p < npairs ? ld_g(idx + p) : -1;
  }
  pdl_trigger();
  for (int e = tid; e < kRankWarps * E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  int32_t* mine = s_cnt + w * E;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t p = p0 + i * 32 + lane;
    const int32_t e = ids[i];
    const bool ok = p < npairs && e >= 0 && e < E;
    const unsigned same = __match_any_sync(0xFFFFFFFFu, ok ? e : -1 - lane);
    if (ok && lane == __ffs(same) - 1) mine[e] += __popc(same);
    __syncwarp();
  }
  pdl_wait_for(counts);  // the histograms
  // warp w: groups w, w + 8, ... two at a time; lanes stride over the chunks, four strides
  // at a time, so eight count loads are in flight per lane
  for (int e0 = w; e0 < E; e0 += 2 * kRankWarps) {
    int32_t tot[2] = {0, 0}, pre[2] = {0, 0};
    for (int64_t c0 = lane; c0 < C; c0 += 4 * 32) {
      int32_t v[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + j * kRankWarps;
          const int64_t c = c0 + u * 32;
          v[j][u] = e < E && c < C ? ld_g(counts + c * E + e) : 0;
        }
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          tot[j] += v[j][u];
          pre[j] += c0 + u * 32 < (int64_t)blockIdx.x ? v[j][u] : 0;
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        tot[j] += __shfl_xor_sync(0xFFFFFFFFu, tot[j], o);
        pre[j] += __shfl_xor_sync(0xFFFFFFFFu, pre[j], o);
      }
      const int e = e0 + j * kRankWarps;
      if (lane == 0 && e < E) {
        s_tot[e] = tot[j];
        s_pre[e] = pre[j];
      }
    }
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e < E; e += blockDim.x) totals[e] = s_tot[e];
  block_pad_offsets(s_tot, s_wsum, E, align, blockIdx.x == 0 ? offsets : nullptr);  // s_tot now holds offsets
  for (int e = tid; e < E; e += blockDim.x) {
    int32_t r = s_tot[e] + s_pre[e];
#pragma unroll
    for (int ww = 0; ww < kRankWarps; ++ww) {
      const int32_t v = s_cnt[ww * E + e];
      s_cnt[ww * E + e] = r;
      r += v;
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int64_t p = p0 + i * 32 + lane;
    const bool live = p < npairs;
    const int32_t e = ids[i];
    const bool ok = live && e >= 0 && e < E;
    const unsigned same = __match_any_sync(0xFFFFFFFFu, ok ? e : -1 - lane);
    const int rank = __popc(same & ((1u << lane) - 1u));
    const int base = ok ? mine[e] : 0;
    __syncwarp();
    if (ok) {
      row_id_map[p] = base + rank;
      if (lane == __ffs(same) - 1) mine[e] = base + __popc(same);
    } else if (live) {
      row_id_map[p] = -1;
    }
    __syncwarp();
  }
}

// Tiles of x (token t, column block j) in row-major order: 8 lanes per tile, 16 bf16 per
// lane (8 from each half of the tile), four tiles per warp per slot.  Each tile is read
// and quantized once and its codes written to the token's top-k destination rows.
__global__ void __launch_bounds__(kSThreads) scatter_quant_kernel(const uint4* __restrict__ x, int64_t tokens, int ncb,
                                                                  const int32_t* __restrict__ row_id_map, int topk,
                                                                  uint2* __restrict__ q, uint8_t* __restrict__ sf,
                                                                  int64_t scatter_ctas, int pad_slots,
                                                                  const int32_t* __restrict__ offsets,
                                                                  const int32_t* __restrict__ totals,
                                                                  int64_t max_rows) {
  if ((int64_t)blockIdx.x >= scatter_ctas) {
    pdl_wait_for(offsets, totals);  // the offsets
    pad_rows((int64_t)blockIdx.x - scatter_ctas, pad_slots, offsets, totals, (int64_t)ncb * 128,
             reinterpret_cast<uint8_t*>(q), sf, max_rows);
    return;
  }
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int64_t n_tiles = tokens * ncb;
  const int64_t warp = ((int64_t)blockIdx.x * kSThreads + threadIdx.x) >> 5;
  int64_t tile[kSUnroll];
  uint4 v0[kSUnroll], v1[kSUnroll];
#pragma unroll
  for (int u = 0; u < kSUnroll; ++u) {
    tile[u] = (warp * kSUnroll + u) * 4 + (lane >> 3);
    if (tile[u] < n_tiles) {
      v0[u] = ld_stream(x + tile[u] * 16 + sub);
      v1[u] = ld_stream(x + tile[u] * 16 + 8 + sub);
    } else {
      v0[u] = v1[u] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  uint2 lo[kSUnroll], hi[kSUnroll];
  int e[kSUnroll];
#pragma unroll
  for (int u = 0; u < kSUnroll; ++u) {
    uint32_t m = maxabs_bf16x2(maxabs_bf16x2(maxabs_bf16x2(v0[u].x, v0[u].y), maxabs_bf16x2(v0[u].z, v0[u].w)),
                               maxabs_bf16x2(maxabs_bf16x2(v1[u].x, v1[u].y), maxabs_bf16x2(v1[u].z, v1[u].w)));
    m = maxabs_bf16x2(m, __byte_perm(m, 0u, 0x1032)) & 0x7FFFu;
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    e[u] = bf16_tile_exponent(m);
    const float s = exp2_neg(e[u]);
    lo[u] = make_uint2(encode4(v0[u].x, v0[u].y, s), encode4(v0[u].z, v0[u].w, s));
    hi[u] = make_uint2(encode4(v1[u].x, v1[u].y, s), encode4(v1[u].z, v1[u].w, s));
  }
  pdl_wait_for(row_id_map);  // the row ids: everything above overlaps the routing
#pragma unroll
  for (int u = 0; u < kSUnroll; ++u) {
    if (tile[u] >= n_tiles) continue;
    const int64_t t = tile[u] / ncb;
    const int j = (int)(tile[u] - t * ncb);
    for (int k = 0; k < topk; ++k) {
      const int32_t row = ld_g(row_id_map + t * topk + k);
      if (row < 0 || row >= max_rows) continue;  // (never out of range for a consistent routing)
      uint2* dst = q + ((int64_t)row * ncb + j) * 16;
      dst[sub] = lo[u];
      dst[8 + sub] = hi[u];
      if (sub == 0) sf[(int64_t)row * ncb + j] = (uint8_t)(e[u] + 127);
    }
  }
}

// FP8-input payload: tiles (token t, column block j) in row-major order, 8 lanes per
// tile (16 codes each, so each load instruction reads whole 128-byte lines), four tiles
// per warp per slot, all loads issued first; each tile's codes and scale byte are
// written to the token's top-k destination rows.
__global__ void __launch_bounds__(kSThreads) scatter_copy_kernel(const uint4* __restrict__ xq,
                                                                 const uint8_t* __restrict__ xsf, int64_t tokens,
                                                                 int ncb, const int32_t* __restrict__ row_id_map,
                                                                 int topk, uint4* __restrict__ q,
                                                                 uint8_t* __restrict__ sf, int64_t scatter_ctas,
                                                                 int pad_slots, const int32_t* __restrict__ offsets,
                                                                 const int32_t* __restrict__ totals, int64_t max_rows) {
  if ((int64_t)blockIdx.x >= scatter_ctas) {
    pdl_wait_for(offsets, totals);  // the offsets
    pad_rows((int64_t)blockIdx.x - scatter_ctas, pad_slots, offsets, totals, (int64_t)ncb * 128,
             reinterpret_cast<uint8_t*>(q), sf, max_rows);
    return;
  }
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int64_t n_tiles = tokens * ncb;
  const int64_t warp = ((int64_t)blockIdx.x * kSThreads + threadIdx.x) >> 5;
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
    for (int k = 0; k < topk; ++k) {
      const int32_t row = ld_g(row_id_map + t * topk + k);
      if (row < 0 || row >= max_rows) continue;  // (never out of range for a consistent routing)
      q[((int64_t)row * ncb + j) * 8 + sub] = v[u];
      if (sub == 0) sf[(int64_t)row * ncb + j] = e[u];
    }
  }
}

}  // namespace

size_t permute_workspace_bytes(int64_t tokens, int32_t topk, int32_t num_experts) {
  const int64_t C = num_chunks(tokens, topk);
  return (size_t)(2 * C * num_experts + num_experts) * sizeof(int32_t) + 16;
}

// Steps (1)-(3): offsets, per-chunk bases, row ids (workspace: counts, bases, totals).
fp8q_status route_pairs(const DeviceInfo& dev, int64_t rows, const int32_t* idx, int32_t slots, int32_t E,
                        int32_t align, bool allow_drop, int32_t* offsets, int32_t* row_id_map, void* workspace,
                        cudaStream_t stream) {
  const int64_t npairs = rows * slots;
  const int64_t C = num_chunks(rows, slots);
  int32_t* counts = static_cast<int32_t*>(workspace);
  const size_t hist_smem = (size_t)E * sizeof(int32_t);
  if (launch_after(count_kernel, dim3((unsigned)C), 256, hist_smem, stream, idx, npairs, (int)E, allow_drop, counts,
                   dev.status) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  return route_ranks(dev, rows, idx, slots, E, align, offsets, row_id_map, workspace, false, stream);
}

// Steps (2)-(3) after the per-chunk histograms are in the workspace's counts.  The rank
// kernels load their chunk's ids before waiting on their predecessor; that is safe when
// the ids existed before the call (after route_pairs' histogram kernel, which waits before
// it lets them start).  ids_wait makes them wait first, for ids written by the kernel
// just before.
fp8q_status route_ranks(const DeviceInfo& dev, int64_t rows, const int32_t* idx, int32_t slots, int32_t E,
                        int32_t align, int32_t* offsets, int32_t* row_id_map, void* workspace, bool ids_wait,
                        cudaStream_t stream) {
  (void)dev;
  const int64_t npairs = rows * slots;
  const int64_t C = num_chunks(rows, slots);
  int32_t* counts = static_cast<int32_t*>(workspace);
  int32_t* bases = counts + C * E;
  int32_t* totals = bases + C * E;
  // Small routings (at most 32 count loads per lane in the fused kernel's reduction) fold
  // the chunk scan into the rank kernel: one dependent launch fewer.
  if (E <= 512 && (int64_t)((E + kRankWarps - 1) / kRankWarps) * ((C + 31) / 32) <= 32) {
    const size_t smem = ((size_t)(kRankWarps + 2) * E + kRankWarps) * sizeof(int32_t);
    return launch_after(rank_fused_kernel, (unsigned)C, kRankWarps * 32, smem, stream, idx, npairs, E, (int)align,
                        (const int32_t*)counts, C, offsets, totals, row_id_map, ids_wait) == cudaSuccess
               ? FP8Q_OK
               : FP8Q_ERR_CUDA;
  }
  if (launch_after(chunk_scan_kernel, (unsigned)((E + 31) / 32), 1024, 0, stream, (const int32_t*)counts, C, E, bases,
                   totals) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  const size_t smem = rank_multi_smem(E);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(rank_multi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  return launch_after(rank_multi_kernel, (unsigned)C, kRankWarps * 32, smem, stream, idx, npairs, E, (int)align,
                      (const int32_t*)bases, (const int32_t*)totals, offsets, row_id_map, ids_wait) == cudaSuccess
             ? FP8Q_OK
             : FP8Q_ERR_CUDA;
}

const int32_t* route_totals(const void* workspace, int64_t rows, int32_t slots, int32_t E) {
  return static_cast<const int32_t*>(workspace) + 2 * num_chunks(rows, slots) * E;
}

namespace {

// xq/xsf != nullptr: FP8-input payload; else quantize x.
fp8q_status permute_pad(const DeviceInfo& dev, const void* x, const uint8_t* xq, const uint8_t* xsf, int64_t tokens,
                        int64_t hidden, const int32_t* topk_idx, int32_t topk, int32_t num_experts, int32_t align,
                        uint8_t* q, uint8_t* sf, int64_t max_rows, int32_t* expert_offsets, int32_t* row_id_map,
                        void* workspace, cudaStream_t stream) {
  const int E = num_experts;
  if (tokens == 0) {
    return cudaMemsetAsync(expert_offsets, 0, (size_t)(E + 1) * sizeof(int32_t), stream) == cudaSuccess
               ? FP8Q_OK
               : FP8Q_ERR_CUDA;
  }
  const fp8q_status rs =
      route_pairs(dev, tokens, topk_idx, topk, E, align, false, expert_offsets, row_id_map, workspace, stream);
  if (rs != FP8Q_OK) return rs;
  const int32_t* totals = route_totals(workspace, tokens, topk, E);
  if (hidden == 0) return FP8Q_OK;  // routing only: offsets and row ids, no payload
  const int ncb = (int)(hidden / 128);
  const int64_t n_tiles = tokens * ncb;
  const int64_t tiles_per_block = (kSThreads / 32) * kSUnroll * 4;
  const int64_t scatter_ctas = (n_tiles + tiles_per_block - 1) / tiles_per_block;
  const int pad_slots = (align - 1 + kPadRowsPerCta - 1) / kPadRowsPerCta;  // 0 when align == 1
  const int64_t blocks = scatter_ctas + (int64_t)E * pad_slots;
  if (blocks > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const int32_t* rmap = row_id_map;
  const int32_t* offs = expert_offsets;
  const int32_t* tots = totals;
  if (xq)
    return launch_scatter_copy(xq, xsf, tokens, hidden, rmap, topk, E, align, q, sf, max_rows, offs, tots, stream);
  const cudaError_t rc = launch_after(scatter_quant_kernel, (unsigned)blocks, kSThreads, 0, stream,
                                      static_cast<const uint4*>(x), tokens, ncb, rmap, (int)topk,
                                      reinterpret_cast<uint2*>(q), sf, scatter_ctas, pad_slots, offs, tots, max_rows);
  return rc == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace

fp8q_status launch_scatter_copy(const uint8_t* xq, const uint8_t* xsf, int64_t rows, int64_t hidden,
                                const int32_t* row_id_map, int32_t slots, int32_t E, int32_t align, uint8_t* q,
                                uint8_t* sf, int64_t max_rows, const int32_t* offsets, const int32_t* totals,
                                cudaStream_t stream) {
  const int ncb = (int)(hidden / 128);
  const int64_t n_tiles = rows * ncb;
  const int64_t tiles_per_block = (kSThreads / 32) * kSUnroll * 4;
  const int64_t scatter_ctas = (n_tiles + tiles_per_block - 1) / tiles_per_block;
  const int pad_slots = (align - 1 + kPadRowsPerCta - 1) / kPadRowsPerCta;  // 0 when align == 1
  const int64_t blocks = scatter_ctas + (int64_t)E * pad_slots;
  if (blocks > 0x7FFFFFFF) return FP8Q_ERR_SHAPE;
  const cudaError_t rc = launch_after(scatter_copy_kernel, (unsigned)blocks, kSThreads, 0, stream,
                                      reinterpret_cast<const uint4*>(xq), xsf, rows, ncb, row_id_map, (int)slots,
                                      reinterpret_cast<uint4*>(q), sf, scatter_ctas, pad_slots, offsets, totals,
                                      max_rows);
  return rc == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

fp8q_status launch_permute_pad_quant(const DeviceInfo& dev, const void* x, int64_t tokens, int64_t hidden,
                                     const int32_t* topk_idx, int32_t topk, int32_t num_experts, int32_t align,
                                     uint8_t* q, uint8_t* sf, int64_t max_out_rows, int32_t* expert_offsets,
                                     int32_t* row_id_map, void* workspace, cudaStream_t stream) {
  return permute_pad(dev, x, nullptr, nullptr, tokens, hidden, topk_idx, topk, num_experts, align, q, sf,
                     max_out_rows, expert_offsets, row_id_map, workspace, stream);
}

fp8q_status launch_permute_pad_fp8(const DeviceInfo& dev, const uint8_t* xq, const uint8_t* xsf, int64_t tokens,
                                   int64_t hidden, const int32_t* topk_idx, int32_t topk, int32_t num_experts,
                                   int32_t align, uint8_t* q, uint8_t* sf, int64_t max_out_rows,
                                   int32_t* expert_offsets, int32_t* row_id_map, void* workspace,
                                   cudaStream_t stream) {
  return permute_pad(dev, nullptr, xq, xsf, tokens, hidden, topk_idx, topk, num_experts, align, q, sf,
                     max_out_rows, expert_offsets, row_id_map, workspace, stream);
}

}  // namespace fp8q
