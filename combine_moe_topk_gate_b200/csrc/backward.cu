// backward.cu -- backward of combine (the backward of dispatch is the combine
// kernel with unit weights, see combine.cu).
//
// DeepEP V2 summary, "training / prefill / decoding usage patterns": the
// backward pass of combine is a dispatch.  For out[t] = sum_j w_j y[s_j]:
//   grad_y[s_j, c] = bf16_rne(fp32(w_j * grad_out[t, c]))    (a weighted dispatch)
//   grad_w[t, j]   = sum_c grad_out[t, c] * y[s_j, c]         (fp32)
//
// Same pipeline as combine: persistent warp-specialised CTAs, work item =
// (group of T = max(1, 8/k) tokens, segment of channels).  The producer warp
// bulk-copies (cp.async.bulk, 1-D, completing on the stage's mbarrier) the
// item's T*k rows of y and the T rows of grad_out into a shared-memory ring.
// 8 consumer warps (8 channels per thread) add the exact bf16 x bf16 products
// into per-row partial dots kept in registers across the group's segments,
// and store the scaled grad_y rows.  After a group's last segment the
// partials are reduced -- over the lanes by an xor-shuffle tree, then over the
// warps in warp order -- so grad_w is deterministic.  Each CTA owns whole
// token groups, so no dot is split between CTAs.  Only additions round: any
// order is within (H - 1) * 2^-24 * sum |terms| of the exact value.
// Every mbarrier wait is bounded (1 s, then MOE_ERR_TIMEOUT).  Segment width,
// consumer warps and the stage budget were chosen by timing variants on B200.
#include <algorithm>

#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;  // x 8 channels = kMaxSeg
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxSeg = 2048;
constexpr int kRowsBudgetBytes = 64 * 1024;       // bytes staged per item (narrower segments for large k)
constexpr int kHeaderBytes = 512;               // weights[32], valid mask, slots[32]
constexpr int kStageTarget = 64 * 1024;
constexpr int kMaxStages = 8;

struct Layout {
  int T, seg, nstage;
  size_t stage_bytes, hdr_off, data_off, total;
};

__host__ __device__ inline Layout smem_layout(int k) {
  Layout L;
  L.T = k >= 8 ? 1 : 8 / k;
  const int rows = L.T * k + L.T;  // y rows + grad_out rows
  int seg = kRowsBudgetBytes / (rows * 2) / 256 * 256;
  L.seg = seg > kMaxSeg ? kMaxSeg : (seg < 256 ? 256 : seg);
  L.stage_bytes = static_cast<size_t>(rows) * L.seg * 2;
  int ns = static_cast<int>(kStageTarget / L.stage_bytes);
  L.nstage = ns < 2 ? 2 : (ns > kMaxStages ? kMaxStages : ns);
  L.hdr_off = 256;  // 2 * kMaxStages mbarriers, padded
  L.data_off = L.hdr_off + static_cast<size_t>(L.nstage) * kHeaderBytes;
  L.total = L.data_off + static_cast<size_t>(L.nstage) * L.stage_bytes;
  return L;
}

__device__ __forceinline__ void consumer_barrier() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}

// KT > 0: k == KT is known at compile time (1, 2, 4 or 8), so the group holds
// exactly 8 slots and the consumers keep 8 dot partials with constant indices;
// KT == 0 serves any k (up to 32 slots per group).
template <int KT>
__global__ void __launch_bounds__(kThreads)
    combine_backward_bulk_kernel(const uint16_t* __restrict__ grad_out,
                                 const uint16_t* __restrict__ y, int N, int H, int k,
                                 const int32_t* __restrict__ token_slot, long long S,
                                 const float* __restrict__ topk_w, uint16_t* __restrict__ grad_y,
                                 float* __restrict__ grad_w, int32_t* d_status) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float part[kConsumerWarps][32];
  const Layout L = smem_layout(k);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bars = smem_addr(smem);
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 64u + 8u * s; };
  const uint32_t data = smem_addr(smem + L.data_off);
  if (threadIdx.x == 0) {
    for (int s = 0; s < L.nstage; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kConsumerWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  const int T = L.T, TK = L.T * k, seg = L.seg;
  const uint32_t seg_bytes = static_cast<uint32_t>(seg) * 2u;
  const int groups = (N + T - 1) / T;
  const int segs = (H + seg - 1) / seg;
  // whole token groups per CTA
  const int gper = (groups + gridDim.x - 1) / gridDim.x;
  const int g0 = blockIdx.x * gper;
  const int g1 = g0 + gper < groups ? g0 + gper : groups;
  const long long i0 = static_cast<long long>(g0) * segs;
  const long long i1 = g1 > g0 ? static_cast<long long>(g1) * segs : i0;
  const long long NK = static_cast<long long>(N) * k;  // entries of token_slot / topk_w

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool ok = true;
    int cur_g = -1, my_slot = -1;
    float my_w = 0.0f;
    for (long long it = i0; it < i1; ++it) {
      const int g = static_cast<int>(it / segs);
      const int s = static_cast<int>(it - static_cast<long long>(g) * segs);
      if (g != cur_g) {
        cur_g = g;
        const long long f = static_cast<long long>(g) * TK + lane;
        my_slot = -1;
        my_w = 0.0f;
        if (lane < TK && f < NK) {
          my_slot = token_slot[f];
          my_w = topk_w[f];
        }
        if (my_slot < -1 || my_slot >= S) report_bad_index(d_status);
      }
      if (!mbar_wait(empty_bar(stage), phase ^ 1u)) {
        report_timeout(d_status);
        ok = false;
        break;
      }
      const int seg_ch = H - s * seg < seg ? H - s * seg : seg;
      const uint32_t row_bytes = static_cast<uint32_t>(seg_ch) * 2u;
      const bool valid = lane < TK && my_slot >= 0 && my_slot < S;
      const uint32_t vmask = __ballot_sync(kFullMask, valid);
      const int ntok = N - g * T < T ? N - g * T : T;  // tokens of this group
      float* hw = reinterpret_cast<float*>(smem + L.hdr_off + static_cast<size_t>(stage) * kHeaderBytes);
      if (lane < TK) {
        hw[lane] = my_w;
        reinterpret_cast<int32_t*>(hw)[64 + lane] = my_slot;
      }
      if (lane == 0) reinterpret_cast<uint32_t*>(hw)[32] = vmask;
      __syncwarp();
      if (lane == 0)
        mbar_arrive_expect_tx(full_bar(stage), (__popc(vmask) + ntok) * row_bytes);
      __syncwarp();
      const uint32_t st0 = data + static_cast<uint32_t>(stage * L.stage_bytes);
      if (valid)
        bulk_g2s(st0 + lane * seg_bytes,
                 y + static_cast<size_t>(my_slot) * H + static_cast<size_t>(s) * seg, row_bytes,
                 full_bar(stage));
      if (lane < ntok)  // grad_out rows follow the y rows
        bulk_g2s(st0 + (TK + lane) * seg_bytes,
                 grad_out + static_cast<size_t>(g * T + lane) * H + static_cast<size_t>(s) * seg,
                 row_bytes, full_bar(stage));
      ++issued;
      if (++stage == L.nstage) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) {
      const long long n = issued < L.nstage ? issued : L.nstage;
      for (long long q = issued - n; q < issued; ++q)
        mbar_wait(full_bar(static_cast<int>(q % L.nstage)), static_cast<uint32_t>((q / L.nstage) & 1));
    }
  } else {
    // ------------------------------------------------------------ consumers
    int stage = 0;
    uint32_t phase = 0;
    const int c = threadIdx.x * 8;
    constexpr int kDots = KT > 0 ? (KT >= 8 ? KT : 8) : 32;  // >= TK
    float dot[kDots];
#pragma unroll
    for (int q = 0; q < kDots; ++q) dot[q] = 0.0f;
    bool failed = false;
    for (long long it = i0; it < i1; ++it) {
      const int g = static_cast<int>(it / segs);
      const int s = static_cast<int>(it - static_cast<long long>(g) * segs);
      if (!failed && !mbar_wait(full_bar(stage), phase)) {
        report_timeout(d_status);
        failed = true;  // keep the barrier schedule, skip the work
      }
      const int seg_ch = H - s * seg < seg ? H - s * seg : seg;
      const float* hw =
          reinterpret_cast<const float*>(smem + L.hdr_off + static_cast<size_t>(stage) * kHeaderBytes);
      const uint32_t vmask = reinterpret_cast<const uint32_t*>(hw)[32];
      if (!failed && c < seg_ch) {
        const uint32_t st0 = data + static_cast<uint32_t>(stage * L.stage_bytes) + c * 2;
        // slot q of the group (token q / k): dot partial of grad_out . y, and
        // grad_y = w * grad_out
        auto slot_work = [&](int q, const float(&gf)[8]) {
          const uint4 yv = ld_shared_v4(st0 + q * seg_bytes);
          const uint32_t y4[4] = {yv.x, yv.y, yv.z, yv.w};
          float d = dot[q];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            d = __fmaf_rn(gf[2 * i], bf16_lo(y4[i]), d);
            d = __fmaf_rn(gf[2 * i + 1], bf16_hi(y4[i]), d);
          }
          dot[q] = d;
          const float wq = hw[q];
          const int slot = reinterpret_cast<const int32_t*>(hw)[64 + q];
          uint4 o;
          o.x = pack_bf16x2(__fmul_rn(wq, gf[0]), __fmul_rn(wq, gf[1]));
          o.y = pack_bf16x2(__fmul_rn(wq, gf[2]), __fmul_rn(wq, gf[3]));
          o.z = pack_bf16x2(__fmul_rn(wq, gf[4]), __fmul_rn(wq, gf[5]));
          o.w = pack_bf16x2(__fmul_rn(wq, gf[6]), __fmul_rn(wq, gf[7]));
          st_stream_v4(grad_y + static_cast<size_t>(slot) * H + static_cast<size_t>(s) * seg + c, o);
        };
        auto grad_row = [&](int u, float(&gf)[8]) {
          const uint4 gv = ld_shared_v4(st0 + (TK + u) * seg_bytes);
          const uint32_t g4[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            gf[2 * i] = bf16_lo(g4[i]);
            gf[2 * i + 1] = bf16_hi(g4[i]);
          }
        };
        if constexpr (KT > 0) {
          constexpr int TT = kDots / KT;  // == L.T
#pragma unroll
          for (int u = 0; u < TT; ++u) {
            if (g * TT + u >= N) break;
            float gf[8];
            grad_row(u, gf);
#pragma unroll
            for (int j = 0; j < KT; ++j)
              if ((vmask >> (u * KT + j)) & 1u) slot_work(u * KT + j, gf);
          }
        } else {
          for (int u = 0; u < T; ++u) {
            if (g * T + u >= N) break;
            float gf[8];
            grad_row(u, gf);
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              if (q >= TK) break;
              if (q / k != u || !((vmask >> q) & 1u)) continue;
              slot_work(q, gf);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(stage));
      if (++stage == L.nstage) {
        stage = 0;
        phase ^= 1u;
      }
      if (s == segs - 1) {
        // the group's last segment: reduce the partial dots and write grad_w
#pragma unroll
        for (int q = 0; q < kDots; ++q) {
          if (q >= TK) break;
          float d = dot[q];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) d = __fadd_rn(d, __shfl_xor_sync(kFullMask, d, o));
          if (lane == 0) part[warp][q] = d;
          dot[q] = 0.0f;
        }
        consumer_barrier();
        if (threadIdx.x < TK) {
          const long long f = static_cast<long long>(g) * TK + threadIdx.x;
          if (f < NK) {
            float acc = part[0][threadIdx.x];
            for (int w = 1; w < kConsumerWarps; ++w) acc = __fadd_rn(acc, part[w][threadIdx.x]);
            grad_w[f] = (!failed && ((vmask >> threadIdx.x) & 1u)) ? acc : 0.0f;
          }
        }
        consumer_barrier();
      }
    }
  }
}

template <int KT>
cudaError_t launch_bulk(const void* grad_out, const void* y, int N, int H, int k,
                        const int32_t* token_slot, long long num_rows, const float* topk_w,
                        void* grad_y, float* grad_w, int32_t* d_status, cudaStream_t stream) {
  const Layout L = smem_layout(k);
  cudaError_t err = cudaFuncSetAttribute(combine_backward_bulk_kernel<KT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L.total));
  if (err != cudaSuccess) return err;
  // keep the shared-memory side of the L1/shared split large enough for the
  // CTAs per SM the stage budget is sized for
  err = cudaFuncSetAttribute(combine_backward_bulk_kernel<KT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 0, per_sm = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_backward_bulk_kernel<KT>,
                                                           kThreads, L.total)) != cudaSuccess)
    return err;
  if (per_sm < 1) per_sm = 1;
  const long long groups = (N + L.T - 1) / L.T;
  const long long grid = std::min<long long>(groups, static_cast<long long>(sms) * per_sm);
  return launch_pdl(combine_backward_bulk_kernel<KT>, static_cast<unsigned>(grid), kThreads, L.total,
                    stream, static_cast<const uint16_t*>(grad_out), static_cast<const uint16_t*>(y),
                    N, H, k, token_slot, num_rows, topk_w, static_cast<uint16_t*>(grad_y), grad_w,
                    d_status);
}

}  // namespace

cudaError_t launch_combine_backward(const void* grad_out, const void* y, int N, int H, int k,
                                    const int32_t* token_slot, long long num_rows,
                                    const float* topk_w, void* grad_y, float* grad_w,
                                    int32_t* d_status, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  switch (k) {
    case 1: return launch_bulk<1>(grad_out, y, N, H, k, token_slot, num_rows, topk_w, grad_y, grad_w, d_status, stream);
    case 2: return launch_bulk<2>(grad_out, y, N, H, k, token_slot, num_rows, topk_w, grad_y, grad_w, d_status, stream);
    case 4: return launch_bulk<4>(grad_out, y, N, H, k, token_slot, num_rows, topk_w, grad_y, grad_w, d_status, stream);
    case 8: return launch_bulk<8>(grad_out, y, N, H, k, token_slot, num_rows, topk_w, grad_y, grad_w, d_status, stream);
    default: return launch_bulk<0>(grad_out, y, N, H, k, token_slot, num_rows, topk_w, grad_y, grad_w, d_status, stream);
  }
}

}  // namespace moe
