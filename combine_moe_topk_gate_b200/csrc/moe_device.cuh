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
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "moe.h"

namespace moe {

constexpr unsigned kFullMask = 0xffffffffu;

// ---------------------------------------------------------------- exp
// e^y = 2^n * e^r, n = nearest integer to y*log2(e), r = y - n*ln2 removed in
// two fused steps (ln2 = head + tail, head = floor(ln2 * 2^16) / 2^16 so that
// n*head is exact), e^r by its Taylor series to r^7/7! (Horner), 2^n built
// from the exponent field.  y is clamped to [-87, 88] so 2^n stays normal;
// the hardware max returns its other operand for any NaN, quiet or
// signalling, so every NaN becomes -87 (as the definition's comparisons do;
// checked on all 2^32 patterns).
// The nearest integer (ties to even) comes from adding 1.5 * 2^23: the sum's
// unit in the last place is 1, so the addition itself rounds y*log2(e) to an
// integer, which then sits in the low mantissa bits (|y*log2(e)| <= 127).
// fixed_exp for y already in [-87, 88] (the clamp would leave it unchanged)
__device__ __forceinline__ float fixed_exp_in_range(float y) {
  constexpr float kLog2e = 1.44269504088896340736f;
  constexpr float kLn2Head = 0.693145751953125f;          // 45426 / 65536
  constexpr float kLn2Tail = 1.42860682030941723212e-6f;  // ln2 - head
  constexpr float kInv2 = 0.5f, kInv6 = 1.0f / 6.0f, kInv24 = 1.0f / 24.0f;
  constexpr float kInv120 = 1.0f / 120.0f, kInv720 = 1.0f / 720.0f;
  constexpr float kInv5040 = 1.0f / 5040.0f;
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float t = __fadd_rn(__fmul_rn(y, kLog2e), kRound);
  const float n = __fsub_rn(t, kRound);
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
  // t's bits are 0x4B400000 + n, whose low 9 bits shifted up by 23 are n's
  // exponent field; one multiply-add builds 2^n = (n + 127) << 23
  const float two_n = __uint_as_float((__float_as_uint(t) << 23) + 0x3F800000u);
  return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float fixed_exp(float y) {
  y = fminf(fmaxf(y, -87.0f), 88.0f);  // the GPU's max returns -87 for every NaN
  return fixed_exp_in_range(y);
}

// 1 / (1 + e^-x), each operation rounded once (the correctly rounded
// reciprocal is the correctly rounded quotient 1 / d).
__device__ __forceinline__ float logistic(float x) {
  return __frcp_rn(__fadd_rn(1.0f, fixed_exp(-x)));
}

// ---------------------------------------------------------------- silu
// silu(g) = g / (1 + e^-g), each operation rounded once, e^-g the fixed exp.
__device__ __forceinline__ float silu_exact(float g) {
  return __fdiv_rn(g, __fadd_rn(1.0f, fixed_exp(-g)));
}

// g / d rounded once, by one correction of the quotient (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): from y ~ 1/d and q = g*y, the
// residual r = d*q - g is exact in one fused multiply-add, and q - r*y,
// rounded once, is the quotient.  r is taken as d*q - g rather than g - d*q
// so that g = -0 keeps its sign.  Used where d is in [1, 2^126) (y normal,
// no flush to zero) and g is finite.
__device__ __forceinline__ float div_corrected(float g, float d) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d));
  const float q = __fmul_rn(g, y);
  const float r = __fmaf_rn(d, q, -g);
  return __fmaf_rn(-r, y, q);
}

// silu for |g| <= 87: -g is then inside the exp's clamp range and
// 1 + e^-g <= 1 + e^87 < 2^126, so the clamp is skipped and the division is
// div_corrected.  Equal to silu_exact on every bf16 g with |g| <= 87, the
// only inputs the SwiGLU kernels give it (all of them checked on the GPU);
// on other fp32 inputs one correction from an approximate reciprocal can be
// one unit in the last place off (the same sweep finds such inputs).
__device__ __forceinline__ float silu_in_range(float g) {
  return div_corrected(g, __fadd_rn(1.0f, fixed_exp_in_range(-g)));
}

// max(m, |g|), NaN if either is NaN
__device__ __forceinline__ float max_abs_nan(float m, float g) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(m), "f"(fabsf(g)));
  return r;
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
// Saturating round-to-nearest-even encoding (OCP E4M3) by the hardware
// conversion: .rn rounds to nearest even, .satfinite takes finite values
// beyond +-448 and infinities to +-448 (checked against the OCP-derived
// oracle on all 2^32 fp32 inputs).  NaN maps to the NaN code with its sign.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  const bool nan_lo = lo != lo, nan_hi = hi != hi;
  uint16_t r;
  // cvt packs its first source into the upper byte, the second into the lower
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  uint32_t v = r;
  if (nan_lo) v = (v & 0xff00u) | ((__float_as_uint(lo) >> 24) & 0x80u) | 0x7fu;
  if (nan_hi) v = (v & 0x00ffu) | ((((__float_as_uint(hi) >> 24) & 0x80u) | 0x7fu) << 8);
  return v;
}

// ---------------------------------------------------------------- scales
// floor(log2(a)) for a > 0 finite, exact from the bits (subnormals too)
__device__ __forceinline__ int floor_log2_pos(float a) {  // a > 0, finite; exact
  const uint32_t u = __float_as_uint(a);
  const int ex = static_cast<int>((u >> 23) & 0xffu);
  return ex ? ex - 127 : (31 - __clz(u & 0x7fffffu)) - 149;
}

// Receive-scale layouts (moe_scale_layout_t): element of scale (row s, block b)
// for B blocks per row.  MN-major: column b is contiguous over the rows with
// leading dimension ld (the row count padded to 16 bytes).  MMA-tiled (E8M0):
// 128-row x 4-block atoms of 512 bytes, row-major over atoms, row s / block b
// at byte (s % 32) * 16 + ((s % 128) / 32) * 4 + b % 4 inside the atom -- the
// order the block-scaled tensor-core MMA takes scale factors in.
template <int SL>
__device__ __forceinline__ size_t scale_at(long long s, int b, int B, long long ld) {
  if constexpr (SL == MOE_SCALE_MN_MAJOR) {
    return static_cast<size_t>(b) * ld + s;
  } else if constexpr (SL == MOE_SCALE_MMA_TILED) {
    const size_t atom = static_cast<size_t>(s >> 7) * (B >> 2) + (b >> 2);
    return atom * 512 + (s & 31) * 16 + ((s >> 5) & 3) * 4 + (b & 3);
  } else if constexpr (SL == MOE_SCALE_MN_MAJOR_PACK4) {
    // 32-bit words of 4 consecutive blocks, MN-major; ld = rows rounded up to 4
    return static_cast<size_t>(b >> 2) * 4 * ld + static_cast<size_t>(s) * 4 + (b & 3);
  } else {
    return static_cast<size_t>(s) * B + b;
  }
}

// e4m3x2 for inputs that are never NaN (the codes of finite values and of
// +-infinity equal e4m3x2's; a NaN input gives an unspecified code).
__device__ __forceinline__ uint32_t e4m3x2_nonan(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- e2m1
// Eight floats -> eight FP4 E2M1 codes packed in a word, value i in bits
// 4i..4i+3 (so the even channel of each byte sits in its low nibble).  Round
// to nearest even; .satfinite takes values beyond +-6 (infinities too) to
// +-6.  cvt puts its first source in the upper nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float* c) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]), "f"(c[4]), "f"(c[5]), "f"(c[6]), "f"(c[7]));
  return r;
}

// value of a non-negative e4m3 code (no NaN), exact
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : __fmul_rn(static_cast<float>(m), 0x1p-9f);
}

// ---------------------------------------------------------------- L2 policy
// Scale tables written in pieces (MN-major, tiled): keep their lines in L2
// (evict-last) until every piece has arrived, so that the stream of payload
// stores does not push half-written sectors out to DRAM.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void st_keep_b32(void* ptr, uint32_t v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.b32 [%0], %1, %2;" ::"l"(ptr), "r"(v), "l"(pol));
}
__device__ __forceinline__ void st_keep_b8(void* ptr, uint32_t v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.b8 [%0], %1, %2;" ::"l"(ptr), "r"(v), "l"(pol));
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

// Bounds-checked build (compiled with -DMOE_BOUNDS_CHECK): a receive-row
// index a kernel derives itself -- from the layout's own counts and offsets,
// not read from a caller's array (those are always checked) -- is also tested
// against the buffer's rows before it is written; one outside [0, rows) is
// skipped and reported as MOE_ERR_BAD_INDEX.  In the default build the test
// compiles to nothing: the indices follow from counts of the same entries.
__device__ __forceinline__ bool derived_row_ok(long long row, long long rows, int32_t* d_status) {
#ifdef MOE_BOUNDS_CHECK
  if (row < 0 || row >= rows) {
    report_bad_index(d_status);
    return false;
  }
#else
  (void)row;
  (void)rows;
  (void)d_status;
#endif
  return true;
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

// Asks L2 to fetch [src, src + bytes) (bulk prefetch: no data returns to the
// SM, nothing waits on it; src and bytes multiples of 16).
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// CTA blockIdx.x of gridDim.x prefetches its share of [base, base + bytes)
// into L2 (thread 0 issues it in pieces of at most 64 KiB).  base 16-byte
// aligned; bytes is rounded down to a multiple of 16.
__device__ __forceinline__ void prefetch_share_l2(const char* base, unsigned long long bytes) {
  if (base == nullptr || threadIdx.x != 0) return;
  bytes &= ~15ull;
  const unsigned long long per = ((bytes + gridDim.x - 1) / gridDim.x + 15) & ~15ull;
  unsigned long long b = per * blockIdx.x;
  const unsigned long long e = b + per < bytes ? b + per : bytes;
  for (; b < e; b += 65536) {
    const unsigned long long n = e - b < 65536 ? e - b : 65536;
    prefetch_l2_bulk(base + b, static_cast<uint32_t>(n));
  }
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

// Launch trace: with MOE_DEBUG set in the environment (to anything but "" or
// "0"), every launch through launch_pdl / launch_pdl_cluster prints the
// kernel's name and launch configuration on stderr.  The variable is read once
// per process.
inline bool debug_launches() {
  static const bool on = [] {
    const char* v = getenv("MOE_DEBUG");
    return v != nullptr && v[0] != '\0' && strcmp(v, "0") != 0;
  }();
  return on;
}

inline void trace_launch(const void* kernel, dim3 grid, dim3 block, size_t smem, unsigned cluster_x) {
  if (!debug_launches()) return;
  const char* name = nullptr;
  if (cudaFuncGetName(&name, kernel) != cudaSuccess || name == nullptr) {
    (void)cudaGetLastError();
    name = "(unknown kernel)";
  }
  fprintf(stderr, "[moe] launch %s grid=(%u,%u,%u) block=(%u,%u,%u) smem=%zu cluster=%u pdl=1\n", name,
          grid.x, grid.y, grid.z, block.x, block.y, block.z, smem, cluster_x);
}

// Launch with the programmatic stream-serialisation attribute (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  trace_launch(reinterpret_cast<const void*>(kernel), grid, block, smem, 1);
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

// Same launch with a thread-block cluster of cluster_x CTAs along x (the
// grid's x extent a multiple of it).  A driver that refuses the two
// attributes together gets the cluster launch alone.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t stream, unsigned cluster_x, Args... args) {
  trace_launch(reinterpret_cast<const void*>(kernel), grid, block, smem, cluster_x);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  if (err == cudaErrorNotSupported || err == cudaErrorInvalidValue) {
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  }
  return err;
}

// ---------------------------------------------------------------- clusters
// Barrier over all threads of all CTAs of the cluster (hardware barrier, no
// spin loop): arrive with release semantics, wait with acquire semantics.
// Every thread of every CTA of the cluster must execute both.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// fp32 at the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ float ld_peer_shared_f32(const void* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(local))), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

}  // namespace moe
