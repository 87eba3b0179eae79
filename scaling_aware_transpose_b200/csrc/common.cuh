// common.cuh — device helpers shared by the libfp8q kernels (sm_100a).
//
// E4M3 codes use the OCP E4M3FN layout (low-precision format table: 1/4/3 bits, max
// 448, no Inf).  Scales are power-of-two exponents e stored as UE8M0 bytes e + 127
// (DeepSeek FP8 §8; FP8-Flow-MoE review, 关键观察 2).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fp8q.h"

namespace fp8q {

constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // bounded mbarrier waits: 1 s

// First error wins; later ones are dropped so the reported code is the root cause.
__device__ __forceinline__ void record_status(int* status, int code) { atomicCAS(status, 0, code); }

// ------------------------------------------------------------ dependent launches
// Every kernel of the library is launched with the programmatic-stream-serialization
// attribute (launch_after), so its CTAs may be scheduled while the previous kernel in the
// stream is still finishing.  pdl_wait() returns once that previous grid has completed
// and its writes are visible (a hardware dependency, not a spin loop); pdl_trigger() lets
// the next kernel in the stream be scheduled.  A kernel that begins a call waits before
// its first global access and triggers after that wait, so whatever a later kernel of the
// call reads before its own wait was complete before the call began.  Inside a call's
// chain (routing -> payload) a kernel may trigger early and wait only where it first
// reads its predecessor's output.  In a launch without the attribute, or after a kernel
// that never triggers, both are no-ops and the launch is ordered as usual.
//
// The wait orders memory accesses only if the compiler keeps them after it.  A load the
// compiler may treat as invariant (a plain load through a const __restrict__ pointer it
// turns into a read-only one) is free to move above an asm statement, so every load after
// a wait goes through a pointer passed through pdl_wait_for(): each pointer becomes the
// output of an empty volatile asm placed after the wait, a value the compiler cannot see
// through, and every address formed from it depends on that output.  (The read-only path
// itself is not used at all; see ld_g.)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
template <typename P>
__device__ __forceinline__ void make_opaque(P& p) {  // p: any pointer variable
  asm volatile("" : "+l"(p));
}
template <typename... P>
__device__ __forceinline__ void pdl_wait_for(P&... ptrs) {
  pdl_wait();
  (make_opaque(ptrs), ...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kernel)(KArgs...), dim3 grid, unsigned block, size_t smem, cudaStream_t stream,
                         Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
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

// ------------------------------------------------------------------ conversions
// Two fp32 -> two E4M3 codes, round to nearest even, saturating to +-448; `lo` lands
// in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two E4M3 codes (low byte first) -> f16x2, exact.
__device__ __forceinline__ uint32_t cvt_f16x2_e4m3x2(uint32_t two_codes) {
  uint32_t r;
  uint16_t v = (uint16_t)two_codes;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}
// f16x2 -> two E4M3 codes, round to nearest even, saturating.
__device__ __forceinline__ uint32_t cvt_e4m3x2_f16x2(uint32_t v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(v));
  return r;
}
__device__ __forceinline__ uint32_t mul_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// ------------------------------------------------------------------ scale rule
// e = the smallest integer with amax <= 448 * 2^e (S = 2^ceil(log2(amax/448))), e = 0
// for amax == 0, clamped below at -127.  Exact: with amax = mu * 2^p, mu in [1, 2),
// 448 = 1.75 * 2^8 gives e = p - 8 when mu <= 1.75 and p - 7 otherwise.
// `amax` is a finite, non-negative fp32.
__device__ __forceinline__ int tile_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  if (b == 0u) return 0;
  const int E = (int)(b >> 23);
  uint32_t mant = b & 0x7FFFFFu;
  int p;
  if (E == 0) {  // fp32 subnormal: renormalize
    const int L = 31 - __clz((int)mant);
    p = L - 149;
    mant = (mant << (23 - L)) & 0x7FFFFFu;
  } else {
    p = E - 127;
  }
  const int e = p - 8 + (mant > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : e;
}
// 2^-e as fp32 for e in [-127, 120] (the exponents this library produces): the
// exponent field 127 - e lies in [7, 254], so the value is always a normal number.
__device__ __forceinline__ float exp2_neg(int e) { return __uint_as_float((uint32_t)(127 - e) << 23); }

// ------------------------------------------------------------------ bf16 tiles
// Two bf16x2 words -> the larger magnitude per half (sign bits meaningless).
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Scale exponent of a tile from its BF16 amax bit pattern (sign clear): e = the smallest
// integer with amax <= 448 * 2^e, 0 for amax == 0, clamped below at -127.  With
// amax = (1 + m/128) * 2^(E-127): e = E - 135, plus one when the 7-bit mantissa exceeds
// 0x60 (mu > 1.75 = 448 / 2^8).  BF16 subnormals (E == 0) are all far below the clamp.
// zero_e is what an all-zero tile takes: 0 (S = 1), or -127 under the zero-tile option.
__device__ __forceinline__ int bf16_tile_exponent(uint32_t amax16, int zero_e = 0) {
  const int e = (int)(amax16 >> 7) - 135 + ((amax16 & 0x7Fu) > 0x60u ? 1 : 0);
  return amax16 == 0u ? zero_e : max(e, -127);
}

// Four bf16 (two words) times s -> four E4M3 codes, element 0 in the low byte.  The
// product by a power of two is exact except below 2^-126, where E4M3 rounds to +-0
// either way.
__device__ __forceinline__ uint32_t encode4(uint32_t a, uint32_t b, float s) {
  float2 p0 = make_float2(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u));
  float2 p1 = make_float2(__uint_as_float(b << 16), __uint_as_float(b & 0xFFFF0000u));
  uint64_t r0, r1;
  const uint64_t ss = ((uint64_t)__float_as_uint(s) << 32) | __float_as_uint(s);
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r0) : "l"(*reinterpret_cast<uint64_t*>(&p0)), "l"(ss));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r1) : "l"(*reinterpret_cast<uint64_t*>(&p1)), "l"(ss));
  const uint32_t c01 = cvt_e4m3x2_f32(__uint_as_float((uint32_t)r0), __uint_as_float((uint32_t)(r0 >> 32)));
  const uint32_t c23 = cvt_e4m3x2_f32(__uint_as_float((uint32_t)r1), __uint_as_float((uint32_t)(r1 >> 32)));
  return __byte_perm(c01, c23, 0x5410);
}

// ------------------------------------------------------------------ scaling-aware shift
// Shift E4M3 codes of one row by k >= 0 binades: q' = RNE_e4m3(decode(q) * 2^-k)
// (FP8-Flow-MoE review, 核心方法).
//  * General form, used for every word: decode exactly to f16 (every E4M3 value is an
//    f16 value), multiply by 2^-k in f16 and re-encode with round-to-nearest-even.
//    While the result stays normal this is the exponent-field subtract; where it turns
//    subnormal the hardware re-rounds the mantissa.  The f16 product is exact unless it
//    falls below 2^-20, and every such value rounds to +-0 in E4M3 either way (the
//    smallest E4M3 rounding threshold is 2^-10), so the result equals the exact RNE of
//    decode(q) * 2^-k.  For k > 24 the scale is 0 (result +-0, sign kept).
//  * SWAR form (all four exponent fields > k, or k == 0): a per-byte subtract of 8k.
//    The test (b | 0x80) - 8(k+1) keeps bit 7 set iff the byte's 7-bit magnitude is
//    >= 8(k+1), with no borrow between bytes.
__device__ __forceinline__ bool shift_fast_ok(const uint32_t (&w)[4], int k) {
  const uint32_t thr = (k == 0) ? 0u : (uint32_t)min(k + 1, 16) * 0x08080808u;
  uint32_t acc = 0x80808080u;
#pragma unroll
  for (int i = 0; i < 4; ++i) acc &= (w[i] | 0x80808080u) - thr;
  return (acc & 0x80808080u) == 0x80808080u;
}
__device__ __forceinline__ uint32_t f16_pow2_neg(int k) {  // f16 bits of 2^-k, 0 for k > 24
  return k <= 14 ? (uint32_t)(15 - k) << 10 : (k <= 24 ? 1u << (24 - k) : 0u);
}
__device__ __forceinline__ uint32_t f16x2_pow2_neg(int k) {
  const uint32_t s = f16_pow2_neg(k);
  return s | (s << 16);
}
// Four codes (one row) times the f16x2 scale s2 = {2^-k, 2^-k}, re-encoded.
__device__ __forceinline__ uint32_t shift_word_general(uint32_t w, uint32_t s2) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h, ol, oh;\n\t.reg .b32 fl, fh;\n\t"
      "mov.b32 {l, h}, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 fl, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 fh, h;\n\t"
      "mul.rn.f16x2 fl, fl, %2;\n\t"
      "mul.rn.f16x2 fh, fh, %2;\n\t"
      "cvt.rn.satfinite.e4m3x2.f16x2 ol, fl;\n\t"
      "cvt.rn.satfinite.e4m3x2.f16x2 oh, fh;\n\t"
      "mov.b32 %0, {ol, oh};\n\t}"
      : "=r"(r)
      : "r"(w), "r"(s2));
  return r;
}
// One 16-byte row chunk per lane, the form chosen once per warp: the SWAR subtract when
// it is exact for every lane's 16 bytes, else the general form on every lane.  A per-lane choice
// makes a warp that mixes the two run both; on real activations most warps hold some
// lane that needs the general form.  Every lane of the warp must call it.
__device__ __forceinline__ void shift_row16_warp(uint32_t (&w)[4], int k) {
  if (__all_sync(0xFFFFFFFFu, shift_fast_ok(w, k))) {
    const uint32_t kk = (uint32_t)k * 0x08080808u;
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] -= kk;
  } else {
    const uint32_t s2 = f16x2_pow2_neg(k);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = shift_word_general(w[i], s2);
  }
}

// 4x4 byte transpose: out[c] = (r0.byte c, r1.byte c, r2.byte c, r3.byte c).
__device__ __forceinline__ void transpose4x4(uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3, uint32_t& o0,
                                             uint32_t& o1, uint32_t& o2, uint32_t& o3) {
  const uint32_t a = __byte_perm(r0, r1, 0x5140), b = __byte_perm(r2, r3, 0x5140);
  const uint32_t c = __byte_perm(r0, r1, 0x7362), d = __byte_perm(r2, r3, 0x7362);
  o0 = __byte_perm(a, b, 0x5410);
  o1 = __byte_perm(a, b, 0x7632);
  o2 = __byte_perm(c, d, 0x5410);
  o3 = __byte_perm(c, d, 0x7632);
}

// ------------------------------------------------------------------ mbarrier (bounded waits)
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete; gives up after timeout_ns, or
// after 2^26 polls should the global timer ever stall.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; it < (1u << 26); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return false;
}

// ------------------------------------------------------------------ groups
// Expert groups are contiguous row ranges (DeepSeek FP8 §5.6, M-grouped contiguous):
// off[0..G], group g = rows off[g]..off[g+1].  Finds the group holding row r and
// checks everything an address computation relies on: off[g] <= r < off[g+1] <= limit,
// both ends multiples of 128.  Inconsistent offsets make it return false (the caller
// records FP8Q_ERR_SHAPE and skips the block), never an out-of-range group.
__device__ __forceinline__ bool find_group(const int32_t* off, int G, int64_t r, int64_t limit, int64_t& o,
                                           int64_t& M) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)off[mid] <= r) lo = mid; else hi = mid;
  }
  const int64_t a = off[lo], b = off[lo + 1];
  o = a;
  M = b - a;
  return a <= r && r < b && b <= limit && (a & 127) == 0 && (b & 127) == 0;
}
// Full consistency check of the offset vector by one CTA (threads stride over the
// groups): non-decreasing, every group a multiple of 128.  Records FP8Q_ERR_SHAPE.
// Address safety does not depend on it (find_group bounds every block); it makes
// inconsistent offsets visible in the status word.
__device__ __forceinline__ void validate_groups_cta(const int32_t* off, int G, int* status) {
  bool bad = false;
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const int64_t a = off[g], b = off[g + 1];
    bad |= b < a || ((b - a) & 127) != 0;
  }
  if (bad) record_status(status, FP8Q_ERR_SHAPE);
}
// Rows covered by the groups: off[G] when it is a valid end (multiple of 128 within
// [0, capacity]), else 0 with FP8Q_ERR_SHAPE recorded.
__device__ __forceinline__ int64_t grouped_rows(const int32_t* off, int G, int64_t capacity, int* status) {
  const int64_t first = off[0], last = off[G];
  if (first != 0 || last < 0 || last > capacity || (last & 127)) {
    if (status != nullptr) record_status(status, FP8Q_ERR_SHAPE);
    return 0;
  }
  return last;
}

// ------------------------------------------------------------------ memory
// Global loads are ordinary coherent loads (ld_g) or evict-first ones (ld_stream), never
// the read-only path (ld.global.nc, __ldg): with dependent launches a kernel's lifetime
// overlaps its predecessor's, which may still be writing what the kernel reads after its
// wait, and the read-only path requires data that stays unchanged for the reading
// kernel's whole lifetime.
template <typename T>
__device__ __forceinline__ T ld_g(const T* p) {
  return *p;
}
__device__ __forceinline__ uint4 ld_stream(const uint4* p) { return __ldcs(p); }
// 8-byte store marked evict-first (written once, not read again by this kernel).
__device__ __forceinline__ void st_stream8(void* p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

}  // namespace fp8q
