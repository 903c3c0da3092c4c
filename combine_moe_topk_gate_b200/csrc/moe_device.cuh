// moe_device.cuh -- device helpers shared by the sm_100a kernels of libmoe.
//
// Every floating-point step whose result decides an integer (a top-k choice,
// an FP8 code) or must be reproducible bit for bit uses an explicitly
// rounded intrinsic (__fmul_rn, __fadd_rn, __fmaf_rn, __fdiv_rn), so the
// compiler cannot contract or reassociate it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr unsigned kFullMask = 0xffffffffu;

// ---------------------------------------------------------------- exp
// e^y = 2^n * e^r, n = nearest integer to y*log2(e), r = y - n*ln2 removed in
// two fused steps (ln2 = head + tail, head = floor(ln2 * 2^16) / 2^16 so that
// n*head is exact), e^r by its Taylor series to r^7/7! (Horner), 2^n built
// from the exponent field.  y is clamped to [-87, 88] so 2^n stays normal.
__device__ __forceinline__ float fixed_exp(float y) {
  constexpr float kLog2e = 1.44269504088896340736f;
  constexpr float kLn2Head = 0.693145751953125f;          // 45426 / 65536
  constexpr float kLn2Tail = 1.42860682030941723212e-6f;  // ln2 - head
  constexpr float kInv2 = 0.5f, kInv6 = 1.0f / 6.0f, kInv24 = 1.0f / 24.0f;
  constexpr float kInv120 = 1.0f / 120.0f, kInv720 = 1.0f / 720.0f;
  constexpr float kInv5040 = 1.0f / 5040.0f;
  y = fminf(fmaxf(y, -87.0f), 88.0f);
  const float n = rintf(__fmul_rn(y, kLog2e));
  float r = __fmaf_rn(-n, kLn2Head, y);
  r = __fmaf_rn(-n, kLn2Tail, r);
  float p = kInv5040;
  p = __fmaf_rn(p, r, kInv720);
  p = __fmaf_rn(p, r, kInv120);
  p = __fmaf_rn(p, r, kInv24);
  p = __fmaf_rn(p, r, kInv6);
  p = __fmaf_rn(p, r, kInv2);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float two_n = __int_as_float((static_cast<int>(n) + 127) << 23);
  return __fmul_rn(p, two_n);
}

// 1 / (1 + e^-x), each operation rounded once.
__device__ __forceinline__ float logistic(float x) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, fixed_exp(-x)));
}

// ---------------------------------------------------------------- bf16
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// two floats -> packed bf16x2 (lo in bits 0..15), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo, .y = hi
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- e4m3
// Saturating round-to-nearest-even encoding (OCP E4M3).  Values beyond +-448
// (and infinities) are clamped to +-448 before the hardware conversion,
// which rounds to nearest even; the clamp gives the same code RNE-then-
// saturate would.  NaN maps to the NaN code with its sign.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  const bool nan_lo = lo != lo, nan_hi = hi != hi;
  const float clo = fminf(fmaxf(lo, -448.0f), 448.0f);
  const float chi = fminf(fmaxf(hi, -448.0f), 448.0f);
  uint16_t r;
  // cvt packs its first source into the upper byte, the second into the lower
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(chi), "f"(clo));
  uint32_t v = r;
  if (nan_lo) v = (v & 0xff00u) | ((__float_as_uint(lo) >> 24) & 0x80u) | 0x7fu;
  if (nan_hi) v = (v & 0x00ffu) | ((((__float_as_uint(hi) >> 24) & 0x80u) | 0x7fu) << 8);
  return v;
}

// ---------------------------------------------------------------- memory
// Read-once streaming load of 16 bytes: not kept in L1 (the rows of x in
// dispatch and y in combine are touched by exactly one warp).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Streaming store: evict-first in L2, so written rows drain to DRAM while the
// kernel still runs instead of piling up as dirty lines for the next kernel.
__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// Lanes of the warp holding the same key (the bits of key above nbits must be
// zero): one ballot per key bit, intersected.  On B200 this is far cheaper
// than __match_any_sync.
__device__ __forceinline__ unsigned warp_match(unsigned key, int nbits) {
  unsigned peers = kFullMask;
  for (int i = 0; i < nbits; ++i) {
    const bool bit = (key >> i) & 1u;
    const unsigned m = __ballot_sync(kFullMask, bit);
    peers &= bit ? m : ~m;
  }
  return peers;
}

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialisation attribute may start while its predecessor finishes;
// pdl_wait() blocks until the predecessor's grid has completed and its writes
// are visible, so it must come before the first global read or write.
// pdl_trigger() lets the successor start launching.  Both are no-ops for a
// kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void report_bad_index(int32_t* d_status) {
  if (d_status) *reinterpret_cast<volatile int32_t*>(d_status) = MOE_ERR_BAD_INDEX;
}

__device__ __forceinline__ void report_timeout(int32_t* d_status) {
  if (d_status) *reinterpret_cast<volatile int32_t*>(d_status) = MOE_ERR_TIMEOUT;
}

// ---------------------------------------------------------------- mbarrier + bulk copy
// 1-D bulk copies (cp.async.bulk, no tensor map, no multicast) complete on an
// mbarrier in the issuing CTA's shared memory.  Every wait is bounded.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete; gives up
// (returns false) after kWaitLimitNs of wall time.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned), counted against `bar`'s transaction bytes.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Launch with the programmatic stream-serialisation attribute (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace moe
