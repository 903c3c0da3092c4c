// quant_channel.cu -- per-(expert, channel) FP8 of the receive buffer, for
// the weight-gradient GEMM of each expert.
//
// DeepSeek Tile-Kernels news, "Funktionen der DeepSeek-Tile-Kernel": FP8
// quantisation "pro Kanal" and batched transposes.  An expert's receive rows
// are the contracted dimension of dW_e = X_e^T dY_e, so one scale per
// (expert, channel) factors out of that GEMM.  Per expert e and channel c,
// over the landed rows [expert_offset[e], expert_offset[e] + expert_count[e]):
//   amax = max |x|, scale[e][c] = amax / 448, code = e4m3(x * (448 / amax)),
// zeros keeping their sign.  Codes go out row-major [S, H] (read MN-major by
// the GEMM) or transposed [H, S] (K-major); padding rows are not touched.
//
// Work list built on the device from the actual expert counts (no host
// synchronisation): a unit is one expert and a slab of SW channels, SW a
// power of two from 16 to 256 chosen per expert so that the unit's rows
// (count x SW x 2 bytes) stay near kUnitBytes -- hot experts get narrow slabs
// and therefore many units, cold ones wide slabs.  A persistent grid walks
// the units (CTA b takes units b, b + G, ...).  Each unit is two passes over
// its rows: pass 1 takes the per-channel amax (loads marked evict-last in L2),
// pass 2 reads the rows again -- from L2 -- and writes the codes.  Only G
// units are in flight at once, and G is lowered when the largest unit is big,
// so the rows between the two passes fit in L2 (about kL2Budget bytes): the
// data leaves DRAM once.  A max is exact in any order, so the slab width
// changes no bit of the result.
//
// Lane mapping for a slab of SW channels: 8 channels (16 bytes) per lane,
// LPR = SW / 8 lanes per row, RPW = 32 / LPR rows per warp instruction.
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kMaxSlab = 256;
constexpr int kMinSlab = 16;
constexpr int kCtasPerSm = 2;  // 16 loads in flight per lane in pass 1 need the registers
constexpr long long kUnitBytes = 96 << 10;       // target rows x slab bytes of one unit
constexpr long long kL2Budget = 56ll << 20;      // rows kept in L2 between the two passes
constexpr int kMaxExperts = MOE_MAX_EXPERTS;

// L2 eviction policies: pass 1 marks the unit's lines evict-last so that pass
// 2 finds them in L2 despite the stream of other CTAs' loads and stores;
// pass 2 and the code stores are evict-first (nothing reads them again here).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ld_hint(const void* ptr, uint64_t pol) {
  uint4 r;  // not volatile: independent loads may be scheduled together
  asm("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(ptr), "l"(pol));
  return r;
}
__device__ __forceinline__ void st_hint_v2(void* ptr, uint2 v, uint64_t pol) {
  // no memory clobber: the codes are never read back here, so loads of x may
  // move ahead of these stores
  asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;" ::"l"(ptr), "r"(v.x), "r"(v.y),
               "l"(pol));
}

// log2 of the slab width for an expert of n rows: the widest slab whose unit
// (n rows x SW channels x 2 bytes) stays within kUnitBytes, at least kMinSlab
// channels, at most kMaxSlab and at most what divides H.
__device__ __forceinline__ int slab_log2(long long n, int max_log2) {
  int l = max_log2;
  while ((1 << l) > kMinSlab && 2 * n * (1ll << l) > kUnitBytes) --l;
  return l;
}

template <bool TRANSPOSE>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    quant_fp8_channel_kernel(const uint16_t* __restrict__ x, long long S, int H, int E,
                             const int32_t* __restrict__ expert_offset,
                             const int32_t* __restrict__ expert_count, uint8_t* __restrict__ out,
                             float* __restrict__ scale, int32_t* d_status) {
  __shared__ int uoff[kMaxExperts + 1];       // first unit of each expert
  __shared__ unsigned char slog[kMaxExperts];  // log2 of each expert's slab width
  __shared__ long long row0[kMaxExperts];
  __shared__ int nrows[kMaxExperts];
  __shared__ int wsum[kWarpsPerCta];
  __shared__ long long max_unit;
  __shared__ float part[kWarpsPerCta][kMaxSlab];
  __shared__ float inv_s[kMaxSlab];
  __shared__ uint8_t tile[TRANSPOSE ? kMaxSlab : 1][33];  // transposed: 32 rows per channel (+1: banks)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int max_log2 = (H % 256 == 0) ? 8 : 7;  // H % 128 == 0
  pdl_wait();
  pdl_trigger();

  // ---- the work list: units per expert, prefix over experts (every CTA
  // computes the same list from the same counts)
  if (tid == 0) max_unit = 0;
  __syncthreads();
  long long my_max = 0;
  for (int e = tid; e < E; e += kThreads) {
    const long long r0 = expert_offset[e];
    long long n = expert_count[e];
    if (r0 < 0 || n < 0 || r0 + n > S) {  // a corrupted layout: the expert is skipped
      if (blockIdx.x == 0) report_bad_index(d_status);
      n = -1;
    }
    const int l = n < 0 ? max_log2 : slab_log2(n, max_log2);
    row0[e] = r0;
    nrows[e] = static_cast<int>(n);
    slog[e] = static_cast<unsigned char>(l);
    uoff[e] = n < 0 ? 0 : (H >> l);
    my_max = max(my_max, n < 0 ? 0 : 2 * n << l);
  }
  if (my_max > 0) atomicMax(reinterpret_cast<unsigned long long*>(&max_unit), static_cast<unsigned long long>(my_max));
  __syncthreads();
  // exclusive scan of uoff[0..E) (E <= 1024: four entries per thread)
  {
    int v[4], s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid * 4 + i;
      v[i] = e < E ? uoff[e] : 0;
      s += v[i];
    }
    int incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFullMask, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wsum[w];
    int run = base + incl - s;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid * 4 + i;
      if (e < E) uoff[e] = run;
      run += v[i];
    }
    if (tid == kThreads - 1) uoff[E] = run;
  }
  __syncthreads();
  const int U = uoff[E];
  // CTAs in flight: all of them unless the largest unit is big; then as many
  // as keep kL2Budget of rows between the passes (at least one per SM)
  long long g = max_unit > 0 ? kL2Budget / max_unit : gridDim.x;
  g = g < 148 ? 148 : g;
  const int G = static_cast<int>(g < gridDim.x ? g : gridDim.x);
  if (static_cast<int>(blockIdx.x) >= G) return;

  const uint64_t keep = l2_policy_evict_last(), done = l2_policy_evict_first();
  for (int u = blockIdx.x; u < U; u += G) {
    // the unit's expert: largest e with uoff[e] <= u (experts without units are skipped)
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (uoff[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int l = slog[e];
    const int SW = 1 << l;
    const int LPR = SW >> 3, RPW = 32 / LPR;
    const int c0 = (u - uoff[e]) * SW;       // first channel of the slab
    const long long r0 = row0[e], n = nrows[e];
    const int sub = lane & (LPR - 1), rr = lane / LPR;
    const int cl = sub * 8;                  // the lane's first channel inside the slab
    const uint16_t* col = x + c0 + cl;
    const long long step = static_cast<long long>(kWarpsPerCta) * RPW;  // rows per CTA instruction

    // pass 1: amax of the lane's 8 channels over its rows, on packed bf16
    // pairs (|x| and max are exact in bf16, so this is the fp32 amax)
    __nv_bfloat162 m2[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) m2[j] = __floats2bfloat162_rn(0.0f, 0.0f);
    auto fold = [&](uint4 v) {
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        m2[j] = __hmax2(m2[j], __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[j])));
    };
    {
      long long s = warp * RPW + rr;  // row index inside the expert
      for (; s + 15 * step < n; s += 16 * step) {
        uint4 v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = ld_hint(col + static_cast<size_t>(r0 + s + q * step) * H, keep);
#pragma unroll
        for (int q = 0; q < 16; ++q) fold(v[q]);
      }
      for (; s < n; s += step) fold(ld_hint(col + static_cast<size_t>(r0 + s) * H, keep));
    }
    // lanes of a warp with the same channels (same sub) differ in the row bits
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t o = __shfl_xor_sync(kFullMask, *reinterpret_cast<uint32_t*>(&m2[j]), off);
        m2[j] = __hmax2(m2[j], *reinterpret_cast<const __nv_bfloat162*>(&o));
      }
    }
    if (rr == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        part[warp][cl + 2 * j] = __low2float(m2[j]);
        part[warp][cl + 2 * j + 1] = __high2float(m2[j]);
      }
    }
    __syncthreads();
    if (tid < SW) {
      float a = part[0][tid];
#pragma unroll
      for (int w = 1; w < kWarpsPerCta; ++w) a = fmaxf(a, part[w][tid]);
      inv_s[tid] = __fdiv_rn(448.0f, a);
      scale[static_cast<size_t>(e) * H + c0 + tid] = __fdiv_rn(a, 448.0f);
    }
    __syncthreads();
    float inv[8];
    bool finite = true;  // every 448/amax of the lane finite: products keep zero signs
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      inv[i] = inv_s[cl + i];
      finite = finite && inv[i] <= 3.402823466e38f;
    }

    // pass 2: codes of one row's 8 channels (x * inv of finite bf16 is never
    // NaN, so the encoder without NaN handling gives the same codes)
    auto codes_of_v = [&](uint4 v) -> uint2 {
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      float p[8];
      if (finite) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          p[2 * j] = __fmul_rn(bf16_lo(w[j]), inv[2 * j]);
          p[2 * j + 1] = __fmul_rn(bf16_hi(w[j]), inv[2 * j + 1]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float lo = bf16_lo(w[j]), hi = bf16_hi(w[j]);
          p[2 * j] = (lo == 0.0f) ? lo : __fmul_rn(lo, inv[2 * j]);
          p[2 * j + 1] = (hi == 0.0f) ? hi : __fmul_rn(hi, inv[2 * j + 1]);
        }
      }
      return make_uint2(e4m3x2_nonan(p[0], p[1]) | (e4m3x2_nonan(p[2], p[3]) << 16),
                        e4m3x2_nonan(p[4], p[5]) | (e4m3x2_nonan(p[6], p[7]) << 16));
    };
    if constexpr (!TRANSPOSE) {
      long long s = warp * RPW + rr;
      for (; s + 7 * step < n; s += 8 * step) {  // eight rows' loads in flight
        uint4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = ld_hint(col + static_cast<size_t>(r0 + s + q * step) * H, done);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          st_hint_v2(out + static_cast<size_t>(r0 + s + q * step) * H + c0 + cl, codes_of_v(v[q]), done);
      }
      for (; s < n; s += step)
        st_hint_v2(out + static_cast<size_t>(r0 + s) * H + c0 + cl,
                   codes_of_v(ld_hint(col + static_cast<size_t>(r0 + s) * H, done)), done);
    } else {
      // 32 rows at a time through the tile: the CTA fills tile[channel][row],
      // then warp w writes channels w, w + 8, ...: lane = row, 32 bytes each
      for (long long s0 = 0; s0 < n; s0 += 32) {
        for (int rt = warp * RPW + rr; rt < 32; rt += step) {
          const long long s = s0 + rt;
          const uint2 q = s < n ? codes_of_v(ld_hint(col + static_cast<size_t>(r0 + s) * H, done))
                                : make_uint2(0, 0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            tile[cl + i][rt] = static_cast<uint8_t>(q.x >> (8 * i));
            tile[cl + 4 + i][rt] = static_cast<uint8_t>(q.y >> (8 * i));
          }
        }
        __syncthreads();
        const long long s = s0 + lane;
        for (int c = warp; c < SW; c += kWarpsPerCta)
          if (s < n) out[static_cast<size_t>(c0 + c) * S + r0 + s] = tile[c][lane];
        __syncthreads();
      }
    }
    __syncthreads();  // part / inv_s are rewritten by the next unit
  }
}

}  // namespace

cudaError_t launch_quant_fp8_channel(const void* x, long long num_rows, int H, int E,
                                     const int32_t* expert_offset, const int32_t* expert_count,
                                     bool transpose, void* out, float* scale, int32_t* d_status,
                                     cudaStream_t stream) {
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* o = static_cast<uint8_t*>(out);
  // one CTA per resident slot; the kernel walks all units with them
  const unsigned grid = 148u * kCtasPerSm;
  if (transpose)
    return launch_pdl(quant_fp8_channel_kernel<true>, grid, kThreads, 0, stream, xs, num_rows, H, E,
                      expert_offset, expert_count, o, scale, d_status);
  return launch_pdl(quant_fp8_channel_kernel<false>, grid, kThreads, 0, stream, xs, num_rows, H, E,
                    expert_offset, expert_count, o, scale, d_status);
}

}  // namespace moe
