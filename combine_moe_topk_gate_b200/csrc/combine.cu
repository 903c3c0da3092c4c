// combine.cu -- weighted gather-reduce of each token's k expert outputs.
//
// [pplx] "Efficient and portable mixture-of-experts communication",
// Introduction and Combine: the token's output is the average of its
// experts' outputs weighted by the router weights.  DeepEP V2 summary, usage
// patterns: combine reduces the expert outputs back to the token.
//
// Work item = (token, 256-channel segment), one warp each; lane owns 8
// channels.  Up to 8 slot rows are loaded (16 bytes per lane each) before any
// of them is used, so every lane keeps 128 bytes in flight; the partial rows
// live in registers and are folded with fmaf in slot order, then rounded to
// bf16 once:  acc = +0; acc = fmaf(w_j, y_j, acc) for j = 0..k-1.
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kBatch = 8;

__global__ void __launch_bounds__(kWarps * 32)
    combine_kernel(const uint16_t* __restrict__ y, int N, int H, int k,
                   const int32_t* __restrict__ token_slot, const float* __restrict__ topk_w,
                   uint16_t* __restrict__ out, int32_t* d_status) {
  const int lane = threadIdx.x & 31;
  const int segs = (H + 255) / 256;
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(N) * segs) return;
  const int t = static_cast<int>(item / segs);
  const int s = static_cast<int>(item - static_cast<long long>(t) * segs);
  const int c0 = s * 256 + lane * 8;
  const bool active = c0 < H;
  const long long S = static_cast<long long>(N) * k;

  int my_slot = -1;
  float my_w = 0.0f;
  if (lane < k) {
    my_slot = token_slot[static_cast<size_t>(t) * k + lane];
    my_w = topk_w[static_cast<size_t>(t) * k + lane];
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;

  for (int j0 = 0; j0 < k; j0 += kBatch) {
    uint4 v[kBatch];
    float wj[kBatch];
    bool use[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + u;
      const int slot = __shfl_sync(kFullMask, my_slot, j & 31);
      wj[u] = __shfl_sync(kFullMask, my_w, j & 31);
      const bool in_range = slot >= 0 && slot < S;
      if (j < k && (slot < -1 || slot >= S) && lane == 0) report_bad_index(d_status);
      use[u] = j < k && in_range;
      v[u] = make_uint4(0, 0, 0, 0);
      if (use[u] && active) v[u] = ld_stream(y + static_cast<size_t>(slot) * H + c0);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (!use[u]) continue;
      const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(wj[u], bf16_lo(w4[i]), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(wj[u], bf16_hi(w4[i]), acc[2 * i + 1]);
      }
    }
  }
  if (active) {
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    st_v4(out + static_cast<size_t>(t) * H + c0, o);
  }
}

}  // namespace

cudaError_t launch_combine(const void* y, int N, int H, int k, const int32_t* token_slot,
                           const float* topk_w, void* out, int32_t* d_status,
                           cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const long long items = static_cast<long long>(N) * ((H + 255) / 256);
  const unsigned blocks = static_cast<unsigned>((items + kWarps - 1) / kWarps);
  combine_kernel<<<blocks, kWarps * 32, 0, stream>>>(static_cast<const uint16_t*>(y), N, H, k,
                                                     token_slot, topk_w,
                                                     static_cast<uint16_t*>(out), d_status);
  return cudaGetLastError();
}

}  // namespace moe
