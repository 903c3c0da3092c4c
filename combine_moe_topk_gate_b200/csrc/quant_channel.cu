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
//
// With a caller's workspace and experts of a few hundred rows on average
// (where one CTA per (expert, slab) leaves a hot expert's lone CTAs on the
// critical path), a persistent grid takes (expert, slab, part) tasks from a
// counter instead: each expert is cut into parts of at most kPartRows rows,
// and the parts of one (expert, slab) combine their amax through the
// workspace (see quant_fp8_channel_queue_kernel).
#include <algorithm>

#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kMinSlabLog2 = 7;                 // 128 channels: 256-byte row pieces
constexpr long long kResidentCtas = 148 * 4;     // CTAs one wave holds (4 per SM)
constexpr long long kWaveBytes = 96ll << 20;     // rows a wave may keep in L2 between its passes
constexpr int kPartRows = 256;                  // rows per task of the queue kernel (a multiple of 32)
constexpr int kMaxParts = 64;                   // parts per (expert, slab): fewer than the grid's CTAs

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

// Pass 1 of a slab over rows [rb, r1): the per-channel amax of this CTA's
// rows, returned on thread c for channel c < SW (0 on the others).  Lanes
// reduce packed bf16 pairs (|x| and max are exact in bf16, so the result is
// the fp32 amax), eight loads in flight per lane; part[] is left for the
// caller to reuse after its next __syncthreads.
template <int LSW>
__device__ __forceinline__ float slab_amax(const uint16_t* __restrict__ col, int H, long long rb,
                                           long long r1, uint64_t keep, float (*part)[1 << LSW]) {
  constexpr int SW = 1 << LSW, LPR = SW / 8, RPW = 32 / LPR, STEP = kWarpsPerCta * RPW;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rr = lane / LPR, cl = (lane % LPR) * 8;
  __nv_bfloat162 m2[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) m2[j] = __floats2bfloat162_rn(0.0f, 0.0f);
  auto fold = [&](uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m2[j] = __hmax2(m2[j], __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[j])));
  };
  long long s = rb + warp * RPW + rr;
  for (; s + 7 * STEP < r1; s += 8 * STEP) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = ld_hint(col + static_cast<size_t>(s + u * STEP) * H, keep);
#pragma unroll
    for (int u = 0; u < 8; ++u) fold(v[u]);
  }
  for (; s < r1; s += STEP) fold(ld_hint(col + static_cast<size_t>(s) * H, keep));
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
  float a = 0.0f;
  if (tid < SW) {
    a = part[0][tid];
#pragma unroll
    for (int w = 1; w < kWarpsPerCta; ++w) a = fmaxf(a, part[w][tid]);
  }
  return a;
}

// Pass 2 of a slab over rows [rb, r1): codes x * inv_s[c] of every channel,
// row-major (8 bytes per lane and row) or transposed through a shared-memory
// tile of 32 rows (each warp store then covers 32 consecutive rows of one
// channel).  x * inv of finite bf16 is never NaN, so the encoder without NaN
// handling gives the same codes.  inv_s must be visible to the whole CTA.
template <bool TRANSPOSE, int LSW>
__device__ __forceinline__ void slab_codes(const uint16_t* __restrict__ col, uint8_t* __restrict__ out,
                                           long long S, int H, int slab, long long rb, long long r1,
                                           const float* inv_s, uint64_t done, uint8_t (*tile)[33]) {
  constexpr int SW = 1 << LSW, LPR = SW / 8, RPW = 32 / LPR, STEP = kWarpsPerCta * RPW;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rr = lane / LPR, cl = (lane % LPR) * 8, c0 = slab * SW + cl;
  float inv[8];
  bool finite = true;  // every 448/amax of the lane finite: products keep zero signs
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    inv[i] = inv_s[cl + i];
    finite = finite && inv[i] <= 3.402823466e38f;
  }
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
}

// Cluster version (no workspace): one CTA, or a cluster of Q CTAs, per
// (expert, slab); the Q CTAs combine their amax through distributed shared
// memory between two hardware cluster barriers.
template <bool TRANSPOSE, bool CLUSTER, int LSW>
__global__ void __launch_bounds__(kThreads)
    quant_fp8_channel_kernel(const uint16_t* __restrict__ x, long long S, int H, int E,
                             const int32_t* __restrict__ expert_offset,
                             const int32_t* __restrict__ expert_count, uint8_t* __restrict__ out,
                             float* __restrict__ scale, int32_t* d_status) {
  constexpr int SW = 1 << LSW;
  __shared__ float part[kWarpsPerCta][SW];
  __shared__ float inv_s[SW];
  __shared__ float cta_amax[CLUSTER ? SW : 1];  // this CTA's share, read by the cluster
  __shared__ uint8_t tile[TRANSPOSE ? SW : 1][33];  // transposed: 32 rows per channel (+1: banks)
  const int tid = threadIdx.x;
  // cluster: x = slab * Q + rank, the Q CTAs of a cluster share (expert, slab)
  const int Q = CLUSTER ? static_cast<int>(gridDim.x / (H / SW)) : 1;
  const int q = CLUSTER ? static_cast<int>(cluster_rank()) : 0;
  const int slab = CLUSTER ? static_cast<int>(blockIdx.x) / Q : static_cast<int>(blockIdx.x);
  const int e = blockIdx.y;
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
  const uint16_t* col = x + slab * SW;
  const uint64_t keep = l2_policy_evict_last(), done = l2_policy_evict_first();

  float a = slab_amax<LSW>(col + ((tid & 31) % (SW / 8)) * 8, H, rb, r1, keep, part);
  if constexpr (CLUSTER) {
    if (tid < SW) cta_amax[tid] = a;
    cluster_arrive();  // every CTA's share published ...
    cluster_wait();
    if (tid < SW) {
      a = 0.0f;
      for (int r = 0; r < Q; ++r) a = fmaxf(a, ld_peer_shared_f32(&cta_amax[tid], static_cast<uint32_t>(r)));
    }
    cluster_arrive();  // ... and read; the matching wait comes before the exit
  }
  if (tid < SW) {
    inv_s[tid] = __fdiv_rn(448.0f, a);
    if (q == 0) scale[static_cast<size_t>(e) * H + slab * SW + tid] = __fdiv_rn(a, 448.0f);
  }
  __syncthreads();
  slab_codes<TRANSPOSE, LSW>(col + ((tid & 31) % (SW / 8)) * 8, out, S, H, slab, rb, r1, inv_s, done, tile);
  if constexpr (CLUSTER) cluster_wait();  // no CTA leaves while a peer may still read its share
}

// ---------------------------------------------------------------- task queue
// Workspace (32-bit words, all zero between calls): [0] next task, [1] CTAs
// finished, then two counters per (expert, 128-channel slab) -- parts that
// published their amax, parts that have read the combined one -- then the
// combined amax of every (expert, channel) as fp32 bits (a max of
// non-negative floats is the max of their bit patterns).
constexpr int kWsHeaderWords = 64;

__host__ __device__ inline long long ws_counter_base() { return kWsHeaderWords; }
__host__ __device__ inline long long ws_amax_base(int E, int H) {
  return kWsHeaderWords + 2ll * E * (H >> kMinSlabLog2);
}

// parts an expert of n rows is cut into (a bad count: one part, which only reports it)
__device__ __forceinline__ int parts_of(long long n) {
  if (n <= kPartRows) return 1;
  const long long p = (n + kPartRows - 1) / kPartRows;
  return p < kMaxParts ? static_cast<int>(p) : kMaxParts;
}

// Persistent CTAs take tasks (expert e, slab, part p) from a counter in the
// workspace, in the order e, slab, p, so the parts of one (expert, slab) run
// side by side and its rows are read twice within a short time (the second
// time from L2).  A part publishes its amax with atomic max, counts itself
// in, and waits (bounded) until every part of its (expert, slab) has done the
// same; the parts were taken before any later task, and pass 1 waits on
// nothing, so the wait ends as long as the grid has more CTAs than an
// expert has parts.  The last part to read the combined amax zeroes the
// scratch of its (expert, slab); the last CTA to finish zeroes the queue.
template <bool TRANSPOSE, int LSW>
__global__ void __launch_bounds__(kThreads)
    quant_fp8_channel_queue_kernel(const uint16_t* __restrict__ x, long long S, int H, int E,
                                   const int32_t* __restrict__ expert_offset,
                                   const int32_t* __restrict__ expert_count, uint8_t* __restrict__ out,
                                   float* __restrict__ scale, int32_t* d_status, uint32_t* ws) {
  constexpr int SW = 1 << LSW;
  __shared__ float part[kWarpsPerCta][SW];
  __shared__ float inv_s[SW];
  __shared__ uint8_t tile[TRANSPOSE ? SW : 1][33];
  __shared__ int first_task[MOE_MAX_EXPERTS + 1];  // tasks of experts < e
  __shared__ int scan[kThreads];
  __shared__ int s_task, s_last;
  const int tid = threadIdx.x;
  const int slabs = H >> LSW;
  pdl_wait();
  pdl_trigger();

  // first_task[e] = slabs * sum over e' < e of parts_of(n_e'): thread i sums
  // the experts of its contiguous run, then a block scan of the run totals
  {
    const int per = (E + kThreads - 1) / kThreads;
    const int e0 = tid * per, e1 = e0 + per < E ? e0 + per : E;
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += parts_of(expert_count[e]) * slabs;
    scan[tid] = sum;
    __syncthreads();
    for (int off = 1; off < kThreads; off <<= 1) {
      const int v = tid >= off ? scan[tid - off] : 0;
      __syncthreads();
      scan[tid] += v;
      __syncthreads();
    }
    int run = scan[tid] - sum;  // exclusive prefix of this thread's run
    for (int e = e0; e < e1; ++e) {
      first_task[e] = run;
      run += parts_of(expert_count[e]) * slabs;
    }
    if (tid == kThreads - 1) first_task[E] = scan[kThreads - 1];
    __syncthreads();
  }
  const int total = first_task[E];
  const uint64_t keep = l2_policy_evict_last(), done = l2_policy_evict_first();
  uint32_t* const counters = ws + ws_counter_base();
  uint32_t* const amax_ws = ws + ws_amax_base(E, H);

  if (tid == 0) s_task = static_cast<int>(atomicAdd(&ws[0], 1u));
  __syncthreads();
  for (;;) {
    const int t = s_task;
    __syncthreads();  // s_task may be overwritten from here on
    if (t >= total) break;
    // the expert whose tasks hold t: the last e with first_task[e] <= t
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (first_task[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const long long r0 = expert_offset[e];
    const long long n = expert_count[e];
    const int P = parts_of(n);
    const int j = t - first_task[e];
    const int slab = j / P, p = j - slab * P;
    if (r0 < 0 || n < 0 || r0 + n > S) {  // a corrupted layout: skip the expert
      if (tid == 0) {
        if (j == 0) report_bad_index(d_status);
        s_task = static_cast<int>(atomicAdd(&ws[0], 1u));
      }
      __syncthreads();
      continue;
    }
    const long long share = P == 1 ? n : ((n + P - 1) / P + 31) / 32 * 32;
    const long long rb = r0 + p * share < r0 + n ? r0 + p * share : r0 + n;
    const long long r1 = rb + share < r0 + n ? rb + share : r0 + n;
    const uint16_t* col = x + slab * SW + ((tid & 31) % (SW / 8)) * 8;

    float a = slab_amax<LSW>(col, H, rb, r1, keep, part);
    if (P > 1) {
      uint32_t* const unit_amax = amax_ws + static_cast<size_t>(e) * H + slab * SW;
      uint32_t* const cnt = counters + 2 * (static_cast<size_t>(e) * (H >> kMinSlabLog2) + slab);
      if (tid < SW) atomicMax(&unit_amax[tid], __float_as_uint(a));
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        atomicAdd(&cnt[0], 1u);
        const unsigned long long t0 = globaltimer_ns();
        while (atomicAdd(&cnt[0], 0u) < static_cast<uint32_t>(P)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            report_timeout(d_status);
            break;
          }
          __nanosleep(64);
        }
        __threadfence();
      }
      __syncthreads();
      if (tid < SW) a = __uint_as_float(atomicAdd(&unit_amax[tid], 0u));
      __syncthreads();  // every thread holds the combined amax
      if (tid == 0) {
        __threadfence();
        s_last = atomicAdd(&cnt[1], 1u) == static_cast<uint32_t>(P - 1);
      }
      __syncthreads();
      if (s_last) {  // every part has read it: leave the scratch zeroed
        if (tid < SW) unit_amax[tid] = 0u;
        if (tid == 0) {
          cnt[0] = 0u;
          cnt[1] = 0u;
        }
      }
    }
    // this task waits on nothing from here on: take the next one now, so that
    // the counter's round trip overlaps pass 2 (a CTA never waits while it
    // holds a task it has not started)
    uint32_t next = 0;
    if (tid == 0) next = atomicAdd(&ws[0], 1u);
    if (tid < SW) {
      inv_s[tid] = __fdiv_rn(448.0f, a);
      if (p == 0) scale[static_cast<size_t>(e) * H + slab * SW + tid] = __fdiv_rn(a, 448.0f);
    }
    __syncthreads();
    slab_codes<TRANSPOSE, LSW>(col, out, S, H, slab, rb, r1, inv_s, done, tile);
    if (tid == 0) s_task = static_cast<int>(next);
    __syncthreads();  // the next task is known; inv_s and part are free again
  }
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&ws[1], 1u) == gridDim.x - 1) {  // the last CTA: every task is taken
      ws[0] = 0u;
      ws[1] = 0u;
    }
  }
}

template <bool TRANSPOSE, int LSW>
cudaError_t launch_channel(bool cluster, int Q, const uint16_t* xs, long long num_rows, int H, int E,
                           const int32_t* expert_offset, const int32_t* expert_count, uint8_t* o,
                           float* scale, int32_t* d_status, uint32_t* ws, cudaStream_t stream) {
  const int slabs = H >> LSW;
  if (ws) {
    auto* kernel = quant_fp8_channel_queue_kernel<TRANSPOSE, LSW>;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t err;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0)) != cudaSuccess)
      return err;
    // no more CTAs than tasks can exist; never fewer than an expert's parts + 1
    const long long tasks = ((num_rows + kPartRows - 1) / kPartRows + E) * slabs;
    long long grid = static_cast<long long>(sms) * (per_sm > 0 ? per_sm : 1);
    if (grid > tasks) grid = tasks;
    if (grid < kMaxParts + 1 && tasks > grid) grid = kMaxParts + 1;
    return launch_pdl(kernel, static_cast<unsigned>(grid), kThreads, 0, stream, xs, num_rows, H, E,
                      expert_offset, expert_count, o, scale, d_status, ws);
  }
  if (cluster)
    return launch_pdl_cluster(quant_fp8_channel_kernel<TRANSPOSE, true, LSW>, dim3(slabs * Q, E), kThreads, 0,
                              stream, Q, xs, num_rows, H, E, expert_offset, expert_count, o, scale, d_status);
  return launch_pdl(quant_fp8_channel_kernel<TRANSPOSE, false, LSW>, dim3(slabs, E), kThreads, 0, stream, xs,
                    num_rows, H, E, expert_offset, expert_count, o, scale, d_status);
}

template <bool TRANSPOSE>
cudaError_t launch_channel_sw(int lsw, bool cluster, int Q, const uint16_t* xs, long long num_rows, int H,
                              int E, const int32_t* expert_offset, const int32_t* expert_count, uint8_t* o,
                              float* scale, int32_t* d_status, uint32_t* ws, cudaStream_t stream) {
  switch (lsw) {
    case 8: return launch_channel<TRANSPOSE, 8>(cluster, Q, xs, num_rows, H, E, expert_offset, expert_count, o,
                                                scale, d_status, ws, stream);
    default: return launch_channel<TRANSPOSE, 7>(cluster, Q, xs, num_rows, H, E, expert_offset, expert_count, o,
                                                 scale, d_status, ws, stream);
  }
}

}  // namespace

// The task queue (workspace) where the cluster path would give every
// (expert, slab) one CTA although the average expert already fills a part:
// there a hot expert's lone CTAs are the critical path (Zipf-skewed shape:
// 297 against 369 us).  Below that the hardware's own scheduling of the
// small (expert, slab) CTAs is faster than the persistent loop (prefill
// shape: 128 against 144 us; decode: 27 against 41 us), and from 1024 rows
// on the clusters already spread every expert (Mixtral shape: 103 against
// 108 us).
bool quant_fp8_channel_takes_workspace(long long num_rows, int E) {
  const long long avg_rows = E > 0 ? num_rows / E : 0;
  return avg_rows >= kPartRows && avg_rows < 1024;
}

size_t quant_fp8_channel_workspace_bytes(int E, int H) {
  return 4 * static_cast<size_t>(ws_amax_base(E, H) + static_cast<long long>(E) * H);
}

cudaError_t launch_quant_fp8_channel(const void* x, long long num_rows, int H, int E,
                                     const int32_t* expert_offset, const int32_t* expert_count,
                                     bool transpose, void* out, float* scale, int32_t* d_status,
                                     void* workspace, cudaStream_t stream) {
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* o = static_cast<uint8_t*>(out);
  const long long avg_rows = E > 0 ? num_rows / E : 0;
  uint32_t* ws = quant_fp8_channel_takes_workspace(num_rows, E) ? static_cast<uint32_t*>(workspace) : nullptr;
  // Without it: CTAs per (expert, slab) from the average rows, about 512 rows
  // each, at most 8 (the portable cluster size); 1 keeps the plain launch.
  const int Q = ws ? 1 : avg_rows >= 4096 ? 8 : avg_rows >= 2048 ? 4 : avg_rows >= 1024 ? 2 : 1;
  // Slab width: the rows one wave of resident CTAs holds between its two
  // passes should fit in L2, or the second pass re-reads DRAM; a narrower
  // slab gives smaller CTAs and more waves, and spreads a hot expert over
  // more CTAs.  Measured on B200 (256 / 128 / 64 / 32 channels): 256 is best
  // up to the 4096-token prefill shape, 128 on the Zipf-skewed and the
  // Mixtral shapes, narrower never (the per-CTA overhead wins).  With the
  // workspace a task holds at most kPartRows rows of its slab.
  const long long share = ws ? std::min<long long>(avg_rows, kPartRows) : (avg_rows + Q - 1) / Q;
  int lsw = (H % 256 == 0) ? 8 : 7;
  if (lsw > kMinSlabLog2 && kResidentCtas * share * (2ll << lsw) > kWaveBytes) --lsw;
  if (transpose)
    return launch_channel_sw<true>(lsw, Q > 1, Q, xs, num_rows, H, E, expert_offset, expert_count, o, scale,
                                   d_status, ws, stream);
  return launch_channel_sw<false>(lsw, Q > 1, Q, xs, num_rows, H, E, expert_offset, expert_count, o, scale,
                                  d_status, ws, stream);
}

}  // namespace moe
