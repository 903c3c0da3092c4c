// combine.cu -- weighted gather-reduce of each token's k expert outputs.
//
// [pplx] "Efficient and portable mixture-of-experts communication",
// Introduction and Combine: the token's output is the average of its
// experts' outputs weighted by the router weights.  DeepEP V2 summary, usage
// patterns: combine reduces the expert outputs back to the token.
//
//   out[t, c] = bf16_rne(acc),  acc = +0, then acc = fmaf(w[t,j], y[slot[t,j], c], acc)
//   for j = 0..k-1 in slot order (masked slots skipped).  With no weights
//   (topk_w == nullptr) every weight is 1 and fmaf(1, v, acc) = acc + v: that
//   is the backward of dispatch (the slot-order sum of a token's gradient rows).
//
// Persistent, warp-specialised CTAs.  Work item = (group of T consecutive
// tokens, 2048-channel segment) with T = max(1, 8 / k), so an item always
// stages about 8 row segments of 4 KB whatever k is.  Each CTA walks a
// contiguous range of items, so consecutive items mostly share a token group
// and its metadata (the group's T*k slots and weights are contiguous).
//   producer warp: per item, waits for a free stage of a shared-memory ring,
//     writes the item's weights and valid-slot mask into the stage header and
//     issues one 1-D bulk copy (cp.async.bulk, global -> shared, completing on
//     the stage's "full" mbarrier) per valid slot row -- lane q copies row q.
//     The next group's slots and weights are loaded one group ahead.
//   8 consumer warps: per item, wait for "full"; each thread folds its 8
//     channels of every token's k staged rows in slot order, stores 16 bytes
//     of bf16 per token, and each warp releases the stage through the
//     "empty" mbarrier.
// Segment size, consumer warps and the ~64 KB stage budget per CTA were
// chosen by timing variants on B200 (prefill and Mixtral shapes).  Waits are
// bounded (1 s, then MOE_ERR_TIMEOUT).
#include <algorithm>

#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kMaxSeg = 2048;           // channels per work item (k <= 8)
constexpr int kConsumerWarps = 8;       // 256 threads x 8 channels = kMaxSeg
constexpr int kStageRowsBytes = 8 * kMaxSeg * 2;  // row segments staged per item
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kHeaderBytes = 256;       // weights[32] + valid mask, per stage
constexpr int kStageTarget = 64 * 1024; // shared bytes in flight per CTA
constexpr int kMaxStages = 8;

struct Layout {
  int T;    // tokens per work item
  int seg;  // channels per work item: 2048, narrower for k > 8 (32 KB per stage)
  int nstage;
  size_t stage_bytes;
  size_t bars_off, hdr_off, data_off, total;
};

__host__ __device__ inline Layout smem_layout(int k) {
  Layout L;
  L.T = k >= 8 ? 1 : 8 / k;
  const int rows = L.T * k;
  L.seg = rows <= 8 ? kMaxSeg : (kStageRowsBytes / (rows * 2)) / 256 * 256;
  L.stage_bytes = static_cast<size_t>(rows) * L.seg * 2;
  int ns = static_cast<int>(kStageTarget / L.stage_bytes);
  L.nstage = ns < 2 ? 2 : (ns > kMaxStages ? kMaxStages : ns);
  L.bars_off = 0;
  L.hdr_off = 128;  // 2 * kMaxStages mbarriers of 8 bytes
  L.data_off = L.hdr_off + static_cast<size_t>(L.nstage) * kHeaderBytes;
  L.total = L.data_off + static_cast<size_t>(L.nstage) * L.stage_bytes;
  return L;
}

// KT > 0: k == KT is known at compile time (1, 2, 4 or 8), so the consumers'
// loops over tokens and slots unroll exactly; KT == 0 serves any k.
template <int KT>
__global__ void __launch_bounds__(kThreads, 3)
    combine_bulk_kernel(const uint16_t* __restrict__ y, int N, int H, int k,
                        const int32_t* __restrict__ token_slot, long long S,
                        const float* __restrict__ topk_w, uint16_t* __restrict__ out,
                        int32_t* d_status) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Layout L = smem_layout(k);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bars = smem_addr(smem + L.bars_off);  // full[s] at bars + 8s, empty[s] at + 64
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
  pdl_wait();  // everything above touched shared memory only
  pdl_trigger();

  const int T = L.T, TK = L.T * k;  // tokens and rows per item (TK <= 32)
  const int seg = L.seg;
  const uint32_t seg_bytes = static_cast<uint32_t>(seg) * 2u;
  const int groups = (N + T - 1) / T;
  const int segs = (H + seg - 1) / seg;
  const long long items = static_cast<long long>(groups) * segs;
  const long long per = (items + gridDim.x - 1) / gridDim.x;
  const long long i0 = static_cast<long long>(blockIdx.x) * per;
  const long long i1 = i0 + per < items ? i0 + per : items;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool ok = true;
    // lane q < TK stands for row q of the group: token g*T + q/k, slot q%k;
    // the group's entries are contiguous in token_slot / topk_w
    const long long NK = static_cast<long long>(N) * k;
    int cur_g = -1, my_slot = -1, next_slot = -1;
    float my_w = 0.0f, next_w = 0.0f;
    if (i0 < i1) {
      const long long f = (i0 / segs) * TK + lane;
      if (lane < TK && f < NK) {
        next_slot = token_slot[f];
        next_w = topk_w ? topk_w[f] : 1.0f;
      }
    }
    for (long long it = i0; it < i1; ++it) {
      const int g = static_cast<int>(it / segs);
      const int s = static_cast<int>(it - static_cast<long long>(g) * segs);
      if (g != cur_g) {
        cur_g = g;
        my_slot = next_slot;
        my_w = next_w;
        const long long f = static_cast<long long>(g + 1) * TK + lane;  // one group ahead
        next_slot = -1;
        next_w = 0.0f;
        if (g + 1 < groups && lane < TK && f < NK) {
          next_slot = token_slot[f];
          next_w = topk_w ? topk_w[f] : 1.0f;
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
      float* hw = reinterpret_cast<float*>(smem + L.hdr_off + static_cast<size_t>(stage) * kHeaderBytes);
      if (lane < TK) hw[lane] = my_w;
      if (lane == 0) reinterpret_cast<uint32_t*>(hw)[32] = vmask;
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(full_bar(stage), __popc(vmask) * row_bytes);
      __syncwarp();
      if (valid)
        bulk_g2s(data + static_cast<uint32_t>(stage * L.stage_bytes) + lane * seg_bytes,
                 y + static_cast<size_t>(my_slot) * H + static_cast<size_t>(s) * seg, row_bytes,
                 full_bar(stage));
      ++issued;
      if (++stage == L.nstage) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) {
      // let the copies already issued land before the CTA may exit
      const long long n = issued < L.nstage ? issued : L.nstage;
      for (long long q = issued - n; q < issued; ++q)  // q-th issue: stage q % ns, parity (q / ns) & 1
        mbar_wait(full_bar(static_cast<int>(q % L.nstage)),
                  static_cast<uint32_t>((q / L.nstage) & 1));
    }
  } else {
    // ------------------------------------------------------------ consumers
    int stage = 0;
    uint32_t phase = 0;
    const int c = threadIdx.x * 8;  // this thread's 8 channels of the segment
    for (long long it = i0; it < i1; ++it) {
      const int g = static_cast<int>(it / segs);
      const int s = static_cast<int>(it - static_cast<long long>(g) * segs);
      if (!mbar_wait(full_bar(stage), phase)) {
        report_timeout(d_status);
        break;
      }
      const int seg_ch = H - s * seg < seg ? H - s * seg : seg;
      if (c < seg_ch) {
        const float* hw =
            reinterpret_cast<const float*>(smem + L.hdr_off + static_cast<size_t>(stage) * kHeaderBytes);
        const uint32_t vmask = reinterpret_cast<const uint32_t*>(hw)[32];
        const uint32_t stage0 = data + static_cast<uint32_t>(stage * L.stage_bytes) + c * 2;
        if constexpr (KT > 0) {
          constexpr int TT = KT >= 8 ? 1 : 8 / KT;  // == L.T
#pragma unroll
          for (int u = 0; u < TT; ++u) {
            const int t = g * TT + u;
            if (t >= N) break;
            const uint32_t row0 = stage0 + static_cast<uint32_t>(u * KT) * seg_bytes;
            uint4 v[KT];
#pragma unroll
            for (int q = 0; q < KT; ++q) v[q] = ld_shared_v4(row0 + q * seg_bytes);
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
            for (int q = 0; q < KT; ++q) {
              if (!((vmask >> (u * KT + q)) & 1u)) continue;  // masked slot: rows not staged
              const float wj = hw[u * KT + q];
              const uint32_t w4[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                acc[2 * i] = __fmaf_rn(wj, bf16_lo(w4[i]), acc[2 * i]);
                acc[2 * i + 1] = __fmaf_rn(wj, bf16_hi(w4[i]), acc[2 * i + 1]);
              }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            st_stream_v4(out + static_cast<size_t>(t) * H + static_cast<size_t>(s) * seg + c, o);
          }
        } else
        for (int u = 0; u < T; ++u) {
          const int t = g * T + u;
          if (t >= N) break;
          const uint32_t row0 = stage0 + static_cast<uint32_t>(u * k) * seg_bytes;
          const uint32_t umask = vmask >> (u * k);
          const float* uw = hw + u * k;
          float acc[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
          for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (j0 + q < k) v[q] = ld_shared_v4(row0 + (j0 + q) * seg_bytes);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int j = j0 + q;
              if (j >= k || !((umask >> j) & 1u)) continue;
              const float wj = uw[j];
              const uint32_t w4[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                acc[2 * i] = __fmaf_rn(wj, bf16_lo(w4[i]), acc[2 * i]);
                acc[2 * i + 1] = __fmaf_rn(wj, bf16_hi(w4[i]), acc[2 * i + 1]);
              }
            }
          }
          uint4 o;
          o.x = pack_bf16x2(acc[0], acc[1]);
          o.y = pack_bf16x2(acc[2], acc[3]);
          o.z = pack_bf16x2(acc[4], acc[5]);
          o.w = pack_bf16x2(acc[6], acc[7]);
          st_stream_v4(out + static_cast<size_t>(t) * H + static_cast<size_t>(s) * seg + c, o);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(stage));
      if (++stage == L.nstage) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

// Small batches (N*k <= kSmallEntries, the decode-sized ones): one warp per
// (token, 256 channels), each lane 8 channels.  The lane loads its 16 bytes of
// all k rows at once -- one memory round trip instead of the pipeline's
// copy-then-fold per item -- and folds them in slot order exactly as the
// pipelined kernel does (acc = fma(w_j, y_j, acc), invalid slots skipped).
constexpr int kSmallEntries = 4096;
constexpr int kSmallWarps = 8;

__global__ void __launch_bounds__(kSmallWarps * 32)
    combine_regs_kernel(const uint16_t* __restrict__ y, int N, int H, int k,
                        const int32_t* __restrict__ token_slot, long long S,
                        const float* __restrict__ topk_w, uint16_t* __restrict__ out,
                        int32_t* d_status) {
  const int lane = threadIdx.x & 31;
  const int segs = (H + 255) / 256;
  const int item = blockIdx.x * kSmallWarps + (threadIdx.x >> 5);  // N*k <= 4096: fits an int
  const int t = item / segs;
  if (t >= N) return;
  const int s = item - t * segs;
  const int c0 = s * 256 + lane * 8;
  const bool active = c0 < H;  // H % 8 == 0
  pdl_wait();
  pdl_trigger();
  int my_slot = -1;
  float my_w = 0.0f;
  if (lane < k) {
    my_slot = token_slot[static_cast<size_t>(t) * k + lane];
    my_w = topk_w ? topk_w[static_cast<size_t>(t) * k + lane] : 1.0f;
    if (s == 0 && (my_slot < -1 || my_slot >= S)) report_bad_index(d_status);
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  for (int j0 = 0; j0 < k; j0 += 8) {
    uint4 v[8];
    int slot[8];
    float w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      slot[q] = __shfl_sync(kFullMask, my_slot, (j0 + q) & 31);
      w[q] = __shfl_sync(kFullMask, my_w, (j0 + q) & 31);
      const bool ok = j0 + q < k && slot[q] >= 0 && slot[q] < S;
      if (!ok) slot[q] = -1;
      v[q] = make_uint4(0, 0, 0, 0);
      if (ok && active) v[q] = ld_stream(y + static_cast<size_t>(slot[q]) * H + c0);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (slot[q] < 0) continue;
      const uint32_t w4[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(w[q], bf16_lo(w4[i]), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(w[q], bf16_hi(w4[i]), acc[2 * i + 1]);
      }
    }
  }
  if (active) {
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    st_stream_v4(out + static_cast<size_t>(t) * H + c0, o);
  }
}

template <int KT>
cudaError_t launch_bulk(const void* y, int N, int H, int k, const int32_t* token_slot,
                        long long num_rows, const float* topk_w, void* out, int32_t* d_status,
                        cudaStream_t stream) {
  const Layout L = smem_layout(k);
  cudaError_t err = cudaFuncSetAttribute(combine_bulk_kernel<KT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L.total));
  if (err != cudaSuccess) return err;
  // keep the shared-memory side of the L1/shared split large enough for the
  // CTAs per SM the stage budget is sized for
  err = cudaFuncSetAttribute(combine_bulk_kernel<KT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 0, per_sm = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_bulk_kernel<KT>, kThreads,
                                                           L.total)) != cudaSuccess)
    return err;
  if (per_sm < 1) per_sm = 1;
  const long long items =
      static_cast<long long>((N + L.T - 1) / L.T) * ((H + L.seg - 1) / L.seg);
  const long long grid = std::min<long long>(items, static_cast<long long>(sms) * per_sm);
  return launch_pdl(combine_bulk_kernel<KT>, static_cast<unsigned>(grid), kThreads, L.total, stream,
                    static_cast<const uint16_t*>(y), N, H, k, token_slot, num_rows, topk_w,
                    static_cast<uint16_t*>(out), d_status);
}

}  // namespace

cudaError_t launch_combine(const void* y, int N, int H, int k, const int32_t* token_slot,
                           long long num_rows, const float* topk_w, void* out, int32_t* d_status,
                           cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  if (static_cast<long long>(N) * k <= kSmallEntries) {
    const int items = N * ((H + 255) / 256);
    return launch_pdl(combine_regs_kernel, static_cast<unsigned>((items + kSmallWarps - 1) / kSmallWarps),
                      kSmallWarps * 32, 0, stream, static_cast<const uint16_t*>(y), N, H, k, token_slot,
                      num_rows, topk_w, static_cast<uint16_t*>(out), d_status);
  }
  switch (k) {
    case 1: return launch_bulk<1>(y, N, H, k, token_slot, num_rows, topk_w, out, d_status, stream);
    case 2: return launch_bulk<2>(y, N, H, k, token_slot, num_rows, topk_w, out, d_status, stream);
    case 4: return launch_bulk<4>(y, N, H, k, token_slot, num_rows, topk_w, out, d_status, stream);
    case 8: return launch_bulk<8>(y, N, H, k, token_slot, num_rows, topk_w, out, d_status, stream);
    default: return launch_bulk<0>(y, N, H, k, token_slot, num_rows, topk_w, out, d_status, stream);
  }
}

}  // namespace moe
