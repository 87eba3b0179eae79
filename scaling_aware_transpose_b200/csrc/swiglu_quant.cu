// swiglu_quant.cu — fused SwiGLU + row-wise FP8 quantization (+ direct transpose).
//
// FP8-Flow-MoE review, 核心方法 (Fused SwiGLU+Quantization): the activation output is
// produced directly in FP8 at the activation boundary instead of a BF16 tensor followed
// by a separate quantize.  Here a CTA works on one 128x128 block at a time: it reads
// gate and up (bf16) once, computes y = silu(gate) * up in fp32, quantizes each 1x128
// row tile with a power-of-two scale, writes the row-wise codes and scales, and, when
// asked, converts the block to the column-wise layout with the scaling-aware shift
// before any byte leaves the SM.
//
// Arithmetic spec of y (every step one IEEE fp32 operation, round to nearest even, no
// contraction; identical on every implementation of this spec):
//   exp(a):  a > 89 -> +inf, a < -104 -> +0; otherwise (Cody & Waite, "Software Manual
//            for the Elementary Functions", 1980) n = rint(a * L2E) (ties to even),
//            r = fma(-n, LN2_HI, a), r = fma(-n, LN2_LO, r), p = Horner over 1/k!, k=7..0,
//            result = (p * 2^floor(n/2)) * 2^(n - floor(n/2));
//   silu(g) = g / (1 + exp(-g));   y = silu(g) * u.
// Constants (each derived from its definition): L2E = fp32(log2 e); LN2_HI = ln 2 cut
// to the top 15 mantissa bits; LN2_LO = fp32(ln 2 - LN2_HI); 1/k! rounded to fp32.
//
// silu(g) depends on g alone and g is BF16, so it takes at most 65536 values.  Outside
// one magnitude range the spec reduces to a single IEEE operation (each fact checked on
// every BF16 input against the CPU spec):
//   |g| < BF16 0x33C1 (about 9e-8): 1 + exp(-g) rounds to exactly 2, silu(g) = RN(g * 0.5);
//   g >= 89:  exp(-g) <= 2^-24, 1 + exp(-g) rounds to 1, silu(g) = g (true from 16.75 on);
//   g <= -89: exp(-g) = +inf (the exp clamp), silu(g) = g / inf = -0;
// the last two together are max(g, -0).  The 2 x 3825 values in between are computed by
// the spec itself into a shared-memory table, and the element loop looks them up: both
// BF16 values of a word at once (their magnitudes clamped into the range with 16-bit-lane
// min/max, the sign picking the half of the table), with a warp vote sending the rare
// warp that saw an input outside the range through the closed forms.  The lookup
// replaces ~40 instructions per element (the exp, the IEEE divide); every value is still
// the spec's, bit for bit.  The table is evaluated once per device: CTA 0 of the first
// launch that finds no published table writes the one it computed to device memory and
// then sets a ready word (release); every CTA that reads the word as set (acquire) copies
// the 31 KB from there (L2) instead of evaluating the spec again.
//
// Block loop: three persistent 256-thread CTAs per SM (80 registers a thread); CTA i takes
// blocks i, i + gridDim.x, ... (column blocks fastest).  A block is four passes of 32 rows;
// each thread holds two passes of gate/up in registers and, as it consumes one, loads the
// pass two ahead (crossing into its next block), so one pass of loads is in flight per
// thread while it computes the other.
#include "common.cuh"
#include "launch.h"

namespace fp8q {
namespace {

constexpr float kL2E = 0x1.715476p+0f;
constexpr float kLn2Hi = 0x1.62e4p-1f;
constexpr float kLn2Lo = 0x1.7f7d1cp-20f;
constexpr float kC0 = 0x1p+0f, kC1 = 0x1p+0f, kC2 = 0x1p-1f, kC3 = 0x1.555556p-3f;  // 1/k!
constexpr float kC4 = 0x1.555556p-5f, kC5 = 0x1.111112p-7f, kC6 = 0x1.6c16c2p-10f, kC7 = 0x1.a01a02p-13f;

// rint(t) for |t| < 2^22 is (t + 1.5*2^23) - 1.5*2^23 with both additions rounded to
// nearest even (the first sum lies in [2^23, 2^24), whose ulp is 1); the integer n is read
// off the bits of the first sum.  Same result as rintf, without the conversion unit.
// The spec's two range rules need no select here: after the clamp, a = 89 evaluates to
// p * 2^128 with p = e^0.277... > 1, which overflows to +inf, and a = -104 to p * 2^-150
// with p = e^-0.027... < 1, which rounds to +0 - exactly the values the rules assign to
// a > 89 and a < -104 (checked on every fp32 input against the CPU spec).
__device__ __forceinline__ float exp_spec(float a) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const float ac = fminf(fmaxf(a, -104.0f), 89.0f);  // keeps n in [-150, 128]
  const float tm = __fadd_rn(__fmul_rn(ac, kL2E), kMagic);
  const float n = __fadd_rn(tm, -kMagic);
  float r = __fmaf_rn(-n, kLn2Hi, ac);
  r = __fmaf_rn(-n, kLn2Lo, r);
  float p = kC7;
  p = __fmaf_rn(p, r, kC6);
  p = __fmaf_rn(p, r, kC5);
  p = __fmaf_rn(p, r, kC4);
  p = __fmaf_rn(p, r, kC3);
  p = __fmaf_rn(p, r, kC2);
  p = __fmaf_rn(p, r, kC1);
  p = __fmaf_rn(p, r, kC0);
  const int ni = __float_as_int(tm) - 0x4B400000;
  const int n1 = ni >> 1;  // floor(n / 2)
  const int n2 = ni - n1;
  return __fmul_rn(__fmul_rn(p, __int_as_float((n1 + 127) << 23)), __int_as_float((n2 + 127) << 23));
}

__device__ __forceinline__ float silu_spec(float g) { return __fdiv_rn(g, __fadd_rn(1.0f, exp_spec(-g))); }
__device__ __forceinline__ float swiglu_spec(float g, float u) { return __fmul_rn(silu_spec(g), u); }

// The silu table: BF16 magnitudes kSiluLo..kSiluHi-1, positive g at 0..kTabN-1, negative g
// at kNegBase..kNegBase+kTabN-1 (entries between are unused).
constexpr uint32_t kSiluLo = 0x33C1u;
constexpr uint32_t kSiluHi = 0x42B2u;  // 89
constexpr uint32_t kTabN = kSiluHi - kSiluLo;
constexpr uint32_t kNegBase = 4096;
constexpr int kTab = (int)(kNegBase + kTabN);
constexpr int kTabPad = (kTab + 3) & ~3;  // whole 16-byte pieces

__device__ __forceinline__ void build_silu_table(float* tab) {
  for (int i = threadIdx.x; i < kTab; i += blockDim.x) {
    const uint32_t ui = (uint32_t)i;
    if (ui >= kTabN && ui < kNegBase) continue;  // unused gap
    const uint32_t h = ui < kTabN ? kSiluLo + ui : 0x8000u | (kSiluLo + ui - kNegBase);
    tab[i] = silu_spec(__uint_as_float(h << 16));
  }
}

// The device's copy of the table and its ready word (zero until the table is published).
__device__ __align__(16) float g_silu_tab[kTabPad];
__device__ uint32_t g_silu_ready;
constexpr uint32_t kSiluReady = 0x5117AB1Eu;

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Fills the CTA's table (kTabPad floats of shared memory): copied from device memory when
// every thread's acquire load sees the ready word, else evaluated here; CTA 0 then
// publishes it (all entries written and fenced before the release store).  Concurrent
// first launches may publish at once; they write identical values.  Ends with a barrier.
__device__ __forceinline__ void fill_silu_table(float* tab) {
  const bool ready = ld_acquire_gpu(&g_silu_ready) == kSiluReady;
  if (__syncthreads_and(ready)) {
    const uint4* src = reinterpret_cast<const uint4*>(g_silu_tab);
    uint4* dst = reinterpret_cast<uint4*>(tab);
    for (int i = threadIdx.x; i < kTabPad / 4; i += blockDim.x) dst[i] = src[i];
    __syncthreads();
    return;
  }
  build_silu_table(tab);
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < kTab; i += blockDim.x)
      if ((uint32_t)i < kTabN || (uint32_t)i >= kNegBase) g_silu_tab[i] = tab[i];  // the gap stays zero
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) st_release_gpu(&g_silu_ready, kSiluReady);
  }
}

__device__ __forceinline__ uint32_t umin16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t umax16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float sel_f32(bool p, float a, float b) {
  float r;
  asm("{.reg .pred q; setp.ne.u32 q, %1, 0; selp.f32 %0, %2, %3, q;}" : "=f"(r) : "r"((uint32_t)p), "f"(a), "f"(b));
  return r;
}

// Both BF16 values of a word at once: magnitudes clamped into the table's range (16-bit
// lanes), then one byte offset per lane, 4 * (magnitude - kSiluLo) + 4 * 4096 * sign (at
// most 31680, so neither lane carries into the other).  acc collects any clamped-away bits.
__device__ __forceinline__ void silu_lookup2(const float* tab, uint32_t w, float& lo, float& hi, uint32_t& acc) {
  const uint32_t m2 = w & 0x7FFF7FFFu;
  const uint32_t c2 = umin16x2(umax16x2(m2, kSiluLo * 0x10001u), (kSiluHi - 1) * 0x10001u);
  acc |= m2 ^ c2;
  const uint32_t off2 = ((c2 - kSiluLo * 0x10001u) << 2) + ((w >> 1) & 0x40004000u);
  const char* tb = reinterpret_cast<const char*>(tab);
  lo = *reinterpret_cast<const float*>(tb + (off2 & 0xFFFFu));
  hi = *reinterpret_cast<const float*>(tb + (off2 >> 16));
}

__device__ __forceinline__ float silu_fix(float v, uint32_t h, float g) {
  const uint32_t d = (h & 0x7FFFu) - kSiluLo;  // wraps to >= 2^31 below the range
  const float out = sel_f32((int)d < 0, __fmul_rn(g, 0.5f), fmaxf(g, -0.0f));
  return sel_f32(d < kTabN, v, out);
}

// max(|a|, |b|, |c|) in one instruction.
__device__ __forceinline__ float max3abs(float a, float b, float c) {
  float r;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// (x0, x1) *= (m0, m1): two IEEE round-to-nearest products in one packed instruction.
__device__ __forceinline__ void mul2_rn(float& x0, float& x1, float m0, float m1) {
  asm("{.reg .b64 x, m; mov.b64 x, {%0, %1}; mov.b64 m, {%2, %3}; mul.rn.f32x2 x, x, m; mov.b64 {%0, %1}, x;}"
      : "+f"(x0), "+f"(x1) : "f"(m0), "f"(m1));
}

constexpr int kThreads = 256;
constexpr int kPasses = 4;  // 4 passes x 32 rows x (8 threads x 16 elements)
constexpr int kDepth = 2;   // passes held in registers
constexpr int kMinBlocks = 3;

__device__ __forceinline__ uint32_t swizzled_chunk(int row, int chunk) { return (uint32_t)(chunk ^ ((row >> 2) & 7)); }

struct BlockIn {
  uint4 g[kDepth][2], u[kDepth][2];
};

// gate/up of pass p (rows p*32 + rsub) of one 128x128 block, 16 elements per thread, into
// register slot p % kDepth.
__device__ __forceinline__ void load_pass(BlockIn& in, int p, const uint16_t* __restrict__ gate,
                                          const uint16_t* __restrict__ up, int64_t rows, int cols, int64_t r0, int c0,
                                          int rsub, int sub) {
  const int64_t r = r0 + p * 32 + rsub;
  if (r < rows) {
    const int64_t base = r * cols + c0 + sub * 16;
    in.g[p % kDepth][0] = ld_stream(reinterpret_cast<const uint4*>(gate + base));
    in.g[p % kDepth][1] = ld_stream(reinterpret_cast<const uint4*>(gate + base + 8));
    in.u[p % kDepth][0] = ld_stream(reinterpret_cast<const uint4*>(up + base));
    in.u[p % kDepth][1] = ld_stream(reinterpret_cast<const uint4*>(up + base + 8));
  } else {
    in.g[p % kDepth][0] = in.g[p % kDepth][1] = in.u[p % kDepth][0] = in.u[p % kDepth][1] = make_uint4(0u, 0u, 0u, 0u);
  }
}

__global__ void __launch_bounds__(kThreads, kMinBlocks) swiglu_quant_kernel(const uint16_t* __restrict__ gate,
                                                                         const uint16_t* __restrict__ up, int64_t rows,
                                                                         int cols, int nblk,
                                                                         uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                                                                         uint8_t* __restrict__ qt,
                                                                         uint8_t* __restrict__ sft) {
  __shared__ __align__(16) float silu_tab[kTabPad];
  __shared__ __align__(16) uint8_t tile[128 * 128];
  __shared__ __align__(16) uint8_t e_row[128];
  __shared__ int e_max_sh;
  pdl_wait_for(gate, up);
  pdl_trigger();
  const int tid = threadIdx.x;
  const int ncb = cols >> 7;
  const int sub = tid & 7;      // 16-element chunk of the row tile
  const int rsub = tid >> 3;    // row within a pass (0..31)

  int blk = blockIdx.x;
  BlockIn in;
#pragma unroll
  for (int p = 0; p < kDepth; ++p)
    load_pass(in, p, gate, up, rows, cols, (int64_t)(blk / ncb) * 128, (blk % ncb) * 128, rsub, sub);
  fill_silu_table(silu_tab);
  for (;;) {
    const int64_t r0 = (int64_t)(blk / ncb) * 128;
    const int c0 = (blk % ncb) * 128;
    const int next = blk + (int)gridDim.x;
    const int64_t nr0 = (int64_t)(next / ncb) * 128;
    const int nc0 = (next % ncb) * 128;
    // ---- y, row-wise quantization
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const int rl = p * 32 + rsub;
      const int64_t r = r0 + rl;
      float y[16];
      const int bi = p % kDepth;
      const uint32_t gw[8] = {in.g[bi][0].x, in.g[bi][0].y, in.g[bi][0].z, in.g[bi][0].w,
                              in.g[bi][1].x, in.g[bi][1].y, in.g[bi][1].z, in.g[bi][1].w};
      const uint32_t uw[8] = {in.u[bi][0].x, in.u[bi][0].y, in.u[bi][0].z, in.u[bi][0].w,
                              in.u[bi][1].x, in.u[bi][1].y, in.u[bi][1].z, in.u[bi][1].w};
      uint32_t acc = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) silu_lookup2(silu_tab, gw[k], y[2 * k], y[2 * k + 1], acc);
      if (__any_sync(0xFFFFFFFFu, acc != 0u)) {  // an input outside the table in this warp
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          y[2 * k] = silu_fix(y[2 * k], gw[k] & 0xFFFFu, __uint_as_float(gw[k] << 16));
          y[2 * k + 1] = silu_fix(y[2 * k + 1], gw[k] >> 16, __uint_as_float(gw[k] & 0xFFFF0000u));
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)  // y = silu(g) * u
        mul2_rn(y[2 * k], y[2 * k + 1], __uint_as_float(uw[k] << 16), __uint_as_float(uw[k] & 0xFFFF0000u));
      float amax;  // finite y: the largest magnitude, by three-input max instructions
      {
        const float a0 = max3abs(y[0], y[1], y[2]), a1 = max3abs(y[3], y[4], y[5]), a2 = max3abs(y[6], y[7], y[8]);
        const float a3 = max3abs(y[9], y[10], y[11]), a4 = max3abs(y[12], y[13], y[14]);
        amax = fmaxf(max3abs(a0, a1, a2), max3abs(a3, a4, y[15]));
      }
#pragma unroll
      for (int o = 4; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      const int e = tile_exponent(amax);
      const float s = exp2_neg(e);
      uint4 codes;
#pragma unroll
      for (int k = 0; k < 8; ++k) mul2_rn(y[2 * k], y[2 * k + 1], s, s);
      codes.x = cvt_e4m3x2_f32(y[0], y[1]) | (cvt_e4m3x2_f32(y[2], y[3]) << 16);
      codes.y = cvt_e4m3x2_f32(y[4], y[5]) | (cvt_e4m3x2_f32(y[6], y[7]) << 16);
      codes.z = cvt_e4m3x2_f32(y[8], y[9]) | (cvt_e4m3x2_f32(y[10], y[11]) << 16);
      codes.w = cvt_e4m3x2_f32(y[12], y[13]) | (cvt_e4m3x2_f32(y[14], y[15]) << 16);
      if (r < rows) {
        *reinterpret_cast<uint4*>(q + r * cols + c0 + sub * 16) = codes;
        if (sub == 0) sf[r * ncb + (c0 >> 7)] = (uint8_t)(e + 127);
      }
      if (qt != nullptr) {
        *reinterpret_cast<uint4*>(tile + rl * 128 + (swizzled_chunk(rl, sub) << 4)) = codes;
        if (sub == 0) e_row[rl] = (uint8_t)(e + 127);
      }
      if (p + kDepth < kPasses)  // refill the slot just consumed, kDepth passes ahead
        load_pass(in, p + kDepth, gate, up, rows, cols, r0, c0, rsub, sub);
      else if (next < nblk)
        load_pass(in, p + kDepth - kPasses, gate, up, rows, cols, nr0, nc0, rsub, sub);
    }

    if (qt != nullptr) {  // uniform across the CTA
      // ---- direct transpose of the block (rows % 128 == 0 is guaranteed by the host)
      __syncthreads();
      if (tid < 32) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(e_row)[tid];
        int m = (int)max(max(w & 0xFFu, (w >> 8) & 0xFFu), max((w >> 16) & 0xFFu, w >> 24));
        m = (int)__reduce_max_sync(0xFFFFFFFFu, (unsigned)m);
        if (tid == 0) e_max_sh = m;
      }
      __syncthreads();
      const int emax = e_max_sh;
      const int lane = tid & 31, c = tid >> 5;  // token quad = lane, 16-byte column chunk = warp
      const uint32_t ew = reinterpret_cast<const uint32_t*>(e_row)[lane];
      uint32_t w[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rl = 4 * lane + i;
        const uint4 v = *reinterpret_cast<const uint4*>(tile + rl * 128 + (swizzled_chunk(rl, c) << 4));
        w[i][0] = v.x;
        w[i][1] = v.y;
        w[i][2] = v.z;
        w[i][3] = v.w;
        shift_row16_warp(w[i], emax - (int)((ew >> (8 * i)) & 0xFFu));
      }
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t o0, o1, o2, o3;
        transpose4x4(w[0][qq], w[1][qq], w[2][qq], w[3][qq], o0, o1, o2, o3);
        const int64_t ch = c0 + 16 * c + 4 * qq;
        uint8_t* dst = qt + ch * rows + r0 + 4 * lane;
        *reinterpret_cast<uint32_t*>(dst) = o0;
        *reinterpret_cast<uint32_t*>(dst + rows) = o1;
        *reinterpret_cast<uint32_t*>(dst + 2 * rows) = o2;
        *reinterpret_cast<uint32_t*>(dst + 3 * rows) = o3;
      }
      if (tid < 128) sft[(int64_t)(c0 + tid) * (rows >> 7) + (r0 >> 7)] = (uint8_t)emax;
      __syncthreads();  // tile, e_row and e_max_sh are reused by the next block
    }
    if (next >= nblk) break;
    blk = next;
  }
}

// Test hooks: the device exp and SwiGLU spec on raw inputs, for cross-checks against the
// CPU implementation of the same spec.  exp over the fp32 bit patterns first..first+n-1.
__global__ void exp_spec_range_kernel(uint32_t first, int64_t n, float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = exp_spec(__uint_as_float(first + (uint32_t)i));
}
__global__ void swiglu_spec_kernel(const float* __restrict__ g, const float* __restrict__ u, int64_t n,
                                   float* __restrict__ y) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = swiglu_spec(g[i], u[i]);
}

// Test hook: silu of BF16 inputs through the kernel's own table path (the same table fill,
// so the device's published table once there is one; word-pair lookup, warp vote, closed
// forms), for an exhaustive check against the CPU spec.  Each warp
// takes 32 consecutive words per step; lanes past the end look up 1.0 (inside the table).
__global__ void __launch_bounds__(kThreads) silu_table_kernel(const uint32_t* __restrict__ g2, int64_t nwords,
                                                              float2* __restrict__ out) {
  __shared__ __align__(16) float silu_tab[kTabPad];
  fill_silu_table(silu_tab);
  const int lane = threadIdx.x & 31;
  const int64_t step = (int64_t)gridDim.x * kThreads;
  for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x - lane; base < nwords; base += step) {
    const int64_t i = base + lane;
    const uint32_t w = i < nwords ? g2[i] : 0x3F803F80u;
    float lo, hi;
    uint32_t acc = 0;
    silu_lookup2(silu_tab, w, lo, hi, acc);
    if (__any_sync(0xFFFFFFFFu, acc != 0u)) {
      lo = silu_fix(lo, w & 0xFFFFu, __uint_as_float(w << 16));
      hi = silu_fix(hi, w >> 16, __uint_as_float(w & 0xFFFF0000u));
    }
    if (i < nwords) out[i] = make_float2(lo, hi);
  }
}

}  // namespace

fp8q_status launch_swiglu_quant(const DeviceInfo& dev, const void* gate, const void* up, int64_t rows, int64_t cols,
                                uint8_t* q, uint8_t* sf, uint8_t* qt, uint8_t* sft, cudaStream_t stream) {
  if (rows == 0 || cols == 0) return FP8Q_OK;
  const int64_t nblk = (rows + 127) / 128 * (cols / 128);
  if (nblk > 0x7FFFFFFF - 0x10000) return FP8Q_ERR_SHAPE;  // block indices are int32
  const int64_t slots = (int64_t)dev.num_sms * kMinBlocks;
  const int64_t grid = nblk < slots ? nblk : slots;
  return launch_after(swiglu_quant_kernel, dim3((unsigned)grid), kThreads, 0, stream, static_cast<const uint16_t*>(gate),
                      static_cast<const uint16_t*>(up), rows, (int)cols, (int)nblk, q, sf, qt, sft) == cudaSuccess
             ? FP8Q_OK
             : FP8Q_ERR_CUDA;
}

fp8q_status launch_debug_exp_spec_range(uint32_t first, int64_t n, float* out, cudaStream_t stream) {
  if (n <= 0) return FP8Q_OK;
  exp_spec_range_kernel<<<1184, 256, 0, stream>>>(first, n, out);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

fp8q_status launch_debug_swiglu_spec(const float* g, const float* u, int64_t n, float* y, cudaStream_t stream) {
  if (n <= 0) return FP8Q_OK;
  swiglu_spec_kernel<<<1184, 256, 0, stream>>>(g, u, n, y);
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

fp8q_status launch_debug_silu_bf16(const void* g, int64_t n, float* y, cudaStream_t stream) {
  if (n <= 0) return FP8Q_OK;
  silu_table_kernel<<<296, kThreads, 0, stream>>>(static_cast<const uint32_t*>(g), n / 2, reinterpret_cast<float2*>(y));
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

}  // namespace fp8q
