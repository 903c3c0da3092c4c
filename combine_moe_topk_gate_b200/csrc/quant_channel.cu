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
// One CTA per (expert, slab of SW channels), SW = 256 or 128, 8 warps, each
// lane owning 8 channels (one 16-byte load per row; a warp instruction
// covers 512 contiguous bytes, or two rows of 256).  Pass 1 reduces the
// slab's amax over the expert's rows, eight loads in flight per lane; pass 2
// reads the same rows again -- from L2, the slab of one expert is small --
// and writes the codes: 8 bytes per lane and row (row-major), or through a
// shared-memory tile of 32 rows so that each warp store covers 32
// consecutive rows of one channel (transposed).  The host narrows the slab
// to 128 channels when a wave of resident CTAs would hold more rows between
// its two passes than L2 keeps.
//
// With few experts (thousands of rows each) one CTA per (expert, slab) is
// too little parallelism, so Q > 1 CTAs form a thread-block cluster per
// (expert, slab), each taking a 32-row-aligned share of the expert's rows:
// every CTA reduces its share's per-channel amax, the cluster combines them
// through distributed shared memory between two hardware cluster barriers,
// and each CTA writes the codes of its own rows.  A max is exact in any
// order, so every Q gives the same bits.
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kMinSlabLog2 = 7;                 // 128 channels: 256-byte row pieces
constexpr long long kResidentCtas = 148 * 4;     // CTAs one wave holds (4 per SM)
constexpr long long kWaveBytes = 96ll << 20;     // rows a wave may keep in L2 between its passes

// L2 eviction policies: pass 1 marks the slab's lines evict-last so that pass
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

template <bool TRANSPOSE, bool CLUSTER, int LSW>
__global__ void __launch_bounds__(kThreads)
    quant_fp8_channel_kernel(const uint16_t* __restrict__ x, long long S, int H, int E,
                             const int32_t* __restrict__ expert_offset,
                             const int32_t* __restrict__ expert_count, uint8_t* __restrict__ out,
                             float* __restrict__ scale, int32_t* d_status) {
  constexpr int SW = 1 << LSW;      // channels per slab
  constexpr int LPR = SW / 8;       // lanes per row (8 channels, 16 bytes each)
  constexpr int RPW = 32 / LPR;     // rows per warp instruction
  constexpr int STEP = kWarpsPerCta * RPW;  // rows per CTA instruction
  __shared__ float part[kWarpsPerCta][SW];
  __shared__ float inv_s[SW];
  __shared__ float cta_amax[CLUSTER ? SW : 1];  // this CTA's share, read by the cluster
  __shared__ uint8_t tile[TRANSPOSE ? SW : 1][33];  // transposed: 32 rows per channel (+1: banks)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // cluster: x = slab * Q + rank, the Q CTAs of a cluster share (expert, slab)
  const int Q = CLUSTER ? static_cast<int>(gridDim.x / (H / SW)) : 1;
  const int q = CLUSTER ? static_cast<int>(cluster_rank()) : 0;
  const int slab = CLUSTER ? static_cast<int>(blockIdx.x) / Q : static_cast<int>(blockIdx.x);
  const int e = blockIdx.y;
  const int sub = lane % LPR, rr = lane / LPR;  // channel group and row of the lane
  const int cl = sub * 8;                       // the lane's first channel inside the slab
  const int c0 = slab * SW + cl;
  pdl_wait();
  pdl_trigger();
  const long long r0 = expert_offset[e];
  const long long n = expert_count[e];
  if (r0 < 0 || n < 0 || r0 + n > S) {  // a corrupted layout: skip the expert (the
    if (tid == 0 && slab == 0) report_bad_index(d_status);  // whole cluster returns:
    return;                                                   // e is the same for all)
  }
  const long long share = CLUSTER ? ((n + Q - 1) / Q + 31) / 32 * 32 : n;  // rows per CTA
  const long long rb = r0 + q * share < r0 + n ? r0 + q * share : r0 + n;  // this CTA's rows
  const long long r1 = rb + share < r0 + n ? rb + share : r0 + n;
  const uint16_t* col = x + c0;
  const uint64_t keep = l2_policy_evict_last(), done = l2_policy_evict_first();

  // pass 1: amax of the lane's 8 channels over its rows, on packed bf16
  // pairs (|x| and max are exact in bf16, so the result is the fp32 amax)
  __nv_bfloat162 m2[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) m2[j] = __floats2bfloat162_rn(0.0f, 0.0f);
  auto fold = [&](uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m2[j] = __hmax2(m2[j], __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[j])));
  };
  {
    long long s = rb + warp * RPW + rr;
    for (; s + 7 * STEP < r1; s += 8 * STEP) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = ld_hint(col + static_cast<size_t>(s + u * STEP) * H, keep);
#pragma unroll
      for (int u = 0; u < 8; ++u) fold(v[u]);
    }
    for (; s < r1; s += STEP) fold(ld_hint(col + static_cast<size_t>(s) * H, keep));
  }
  // lanes of a warp holding the same channels differ in their row bits
#pragma unroll
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
  {
    const int c = tid;  // channel of this thread, c < SW
    float a = 0.0f;
    if (c < SW) {
      a = part[0][c];
#pragma unroll
      for (int w = 1; w < kWarpsPerCta; ++w) a = fmaxf(a, part[w][c]);
    }
    if constexpr (CLUSTER) {
      if (c < SW) cta_amax[c] = a;
      cluster_arrive();  // every CTA's share published ...
      cluster_wait();
      if (c < SW) {
        a = 0.0f;
        for (int r = 0; r < Q; ++r) a = fmaxf(a, ld_peer_shared_f32(&cta_amax[c], static_cast<uint32_t>(r)));
      }
      cluster_arrive();  // ... and read; the matching wait comes before the exit
    }
    if (c < SW) {
      inv_s[c] = __fdiv_rn(448.0f, a);
      if (q == 0) scale[static_cast<size_t>(e) * H + slab * SW + c] = __fdiv_rn(a, 448.0f);
    }
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
    long long s = rb + warp * RPW + rr;
    for (; s + 3 * STEP < r1; s += 4 * STEP) {  // four rows' loads in flight
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ld_hint(col + static_cast<size_t>(s + u * STEP) * H, done);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        st_hint_v2(out + static_cast<size_t>(s + u * STEP) * H + c0, codes_of_v(v[u]), done);
    }
    for (; s < r1; s += STEP)
      st_hint_v2(out + static_cast<size_t>(s) * H + c0,
                 codes_of_v(ld_hint(col + static_cast<size_t>(s) * H, done)), done);
  } else {
    for (long long s0 = rb; s0 < r1; s0 += 32) {
      // the CTA fills rows s0 .. s0 + 31 of the tile, RPW rows per warp instruction
      for (int rt = warp * RPW + rr; rt < 32; rt += STEP) {
        const long long s = s0 + rt;
        const uint2 v = s < r1 ? codes_of_v(ld_hint(col + static_cast<size_t>(s) * H, done)) : make_uint2(0, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          tile[cl + i][rt] = static_cast<uint8_t>(v.x >> (8 * i));
          tile[cl + 4 + i][rt] = static_cast<uint8_t>(v.y >> (8 * i));
        }
      }
      __syncthreads();
      // warp w writes channels w, w + 8, ...: lane = row, 32 consecutive bytes
      const long long s = s0 + lane;
      for (int c = warp; c < SW; c += kWarpsPerCta)
        if (s < r1) out[static_cast<size_t>(slab * SW + c) * S + s] = tile[c][lane];
      __syncthreads();
    }
  }
  if constexpr (CLUSTER) cluster_wait();  // no CTA leaves while a peer may still read its share
}

template <bool TRANSPOSE, int LSW>
cudaError_t launch_channel(bool cluster, int Q, const uint16_t* xs, long long num_rows, int H, int E,
                           const int32_t* expert_offset, const int32_t* expert_count, uint8_t* o,
                           float* scale, int32_t* d_status, cudaStream_t stream) {
  const int slabs = H >> LSW;
  if (cluster)
    return launch_pdl_cluster(quant_fp8_channel_kernel<TRANSPOSE, true, LSW>, dim3(slabs * Q, E), kThreads, 0,
                              stream, Q, xs, num_rows, H, E, expert_offset, expert_count, o, scale, d_status);
  return launch_pdl(quant_fp8_channel_kernel<TRANSPOSE, false, LSW>, dim3(slabs, E), kThreads, 0, stream, xs,
                    num_rows, H, E, expert_offset, expert_count, o, scale, d_status);
}

template <bool TRANSPOSE>
cudaError_t launch_channel_sw(int lsw, bool cluster, int Q, const uint16_t* xs, long long num_rows, int H,
                              int E, const int32_t* expert_offset, const int32_t* expert_count, uint8_t* o,
                              float* scale, int32_t* d_status, cudaStream_t stream) {
  switch (lsw) {
    case 8: return launch_channel<TRANSPOSE, 8>(cluster, Q, xs, num_rows, H, E, expert_offset, expert_count, o,
                                                scale, d_status, stream);
    case 7: return launch_channel<TRANSPOSE, 7>(cluster, Q, xs, num_rows, H, E, expert_offset, expert_count, o,
                                                scale, d_status, stream);
    case 6: return launch_channel<TRANSPOSE, 6>(cluster, Q, xs, num_rows, H, E, expert_offset, expert_count, o,
                                                scale, d_status, stream);
    default: return launch_channel<TRANSPOSE, 5>(cluster, Q, xs, num_rows, H, E, expert_offset, expert_count, o,
                                                 scale, d_status, stream);
  }
}

}  // namespace

cudaError_t launch_quant_fp8_channel(const void* x, long long num_rows, int H, int E,
                                     const int32_t* expert_offset, const int32_t* expert_count,
                                     bool transpose, void* out, float* scale, int32_t* d_status,
                                     cudaStream_t stream) {
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* o = static_cast<uint8_t*>(out);
  // CTAs per (expert, slab): about 512 rows each on average, at most 8 (the
  // portable cluster size); 1 keeps the plain launch
  const long long avg_rows = E > 0 ? num_rows / E : 0;
  const int Q = avg_rows >= 4096 ? 8 : avg_rows >= 2048 ? 4 : avg_rows >= 1024 ? 2 : 1;
  // Slab width: the rows one wave of resident CTAs holds between its two
  // passes should fit in L2, or the second pass re-reads DRAM; a narrower
  // slab gives smaller CTAs and more waves, and spreads a hot expert over
  // more CTAs.  Measured on B200 (256 / 128 / 64 / 32 channels): 256 is best
  // up to the 4096-token prefill shape, 128 on the Zipf-skewed and the
  // Mixtral shapes, narrower never (the per-CTA overhead wins).
  const long long share = (avg_rows + Q - 1) / Q;
  int lsw = (H % 256 == 0) ? 8 : 7;
  if (lsw > kMinSlabLog2 && kResidentCtas * share * (2ll << lsw) > kWaveBytes) --lsw;
  if (transpose)
    return launch_channel_sw<true>(lsw, Q > 1, Q, xs, num_rows, H, E, expert_offset, expert_count, o, scale,
                                   d_status, stream);
  return launch_channel_sw<false>(lsw, Q > 1, Q, xs, num_rows, H, E, expert_offset, expert_count, o, scale,
                                  d_status, stream);
}

}  // namespace moe
