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
// One CTA per (expert, 128-channel slab), 8 warps, each lane owning 4
// channels (one 8-byte load per row).  Pass 1 reduces the slab's amax over
// the expert's rows; pass 2 reads the same rows again -- from L2, the slab of
// one expert is small -- and writes the codes: 4 bytes per lane and row
// (row-major), or through a shared-memory tile of 32 rows so that each warp
// store covers 32 consecutive rows of one channel (transposed).
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kSlab = 128;

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

template <bool TRANSPOSE>
__global__ void __launch_bounds__(kThreads)
    quant_fp8_channel_kernel(const uint16_t* __restrict__ x, long long S, int H, int E,
                             const int32_t* __restrict__ expert_offset,
                             const int32_t* __restrict__ expert_count, uint8_t* __restrict__ out,
                             float* __restrict__ scale, int32_t* d_status) {
  __shared__ float part[kWarpsPerCta][kSlab];
  __shared__ float inv_s[kSlab];
  __shared__ uint8_t tile[kSlab][33];  // transposed path: 32 rows per channel (+1 against conflicts)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slab = blockIdx.x, e = blockIdx.y;
  const int c0 = slab * kSlab + lane * 4;
  pdl_wait();
  pdl_trigger();
  long long r0 = expert_offset[e];
  const long long n = expert_count[e];
  if (r0 < 0 || n < 0 || r0 + n > S) {  // a corrupted layout: skip the expert
    if (tid == 0 && slab == 0) report_bad_index(d_status);
    return;
  }
  const long long r1 = r0 + n;

  // pass 1: amax of the lane's 4 channels over the warp's rows
  float m[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 4
  for (long long s = r0 + warp; s < r1; s += kWarpsPerCta) {
    const uint2 v = ld_nc_v2(x + static_cast<size_t>(s) * H + c0);
    m[0] = fmaxf(m[0], fabsf(bf16_lo(v.x)));
    m[1] = fmaxf(m[1], fabsf(bf16_hi(v.x)));
    m[2] = fmaxf(m[2], fabsf(bf16_lo(v.y)));
    m[3] = fmaxf(m[3], fabsf(bf16_hi(v.y)));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) part[warp][lane * 4 + i] = m[i];
  __syncthreads();
  if (tid < kSlab) {
    float a = part[0][tid];
#pragma unroll
    for (int w = 1; w < kWarpsPerCta; ++w) a = fmaxf(a, part[w][tid]);
    inv_s[tid] = __fdiv_rn(448.0f, a);
    scale[static_cast<size_t>(e) * H + slab * kSlab + tid] = __fdiv_rn(a, 448.0f);
  }
  __syncthreads();
  float inv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) inv[i] = inv_s[lane * 4 + i];

  // pass 2: codes
  auto codes_of = [&](long long s) -> uint32_t {
    const uint2 v = ld_nc_v2(x + static_cast<size_t>(s) * H + c0);
    const float f[4] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y)};
    float p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = (f[i] == 0.0f) ? f[i] : __fmul_rn(f[i], inv[i]);
    return e4m3x2(p[0], p[1]) | (e4m3x2(p[2], p[3]) << 16);
  };
  if constexpr (!TRANSPOSE) {
    for (long long s = r0 + warp; s < r1; s += kWarpsPerCta)
      *reinterpret_cast<uint32_t*>(out + static_cast<size_t>(s) * H + c0) = codes_of(s);
  } else {
    for (long long s0 = r0; s0 < r1; s0 += 32) {
      // warp w fills rows s0 + w, s0 + w + 8, ... of the 32-row tile
      for (int rr = warp; rr < 32; rr += kWarpsPerCta) {
        const long long s = s0 + rr;
        const uint32_t q = s < r1 ? codes_of(s) : 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) tile[lane * 4 + i][rr] = static_cast<uint8_t>(q >> (8 * i));
      }
      __syncthreads();
      // warp w writes channels w, w + 8, ...: lane = row, 32 consecutive bytes
      const long long s = s0 + lane;
      for (int c = warp; c < kSlab; c += kWarpsPerCta)
        if (s < r1) out[static_cast<size_t>(slab * kSlab + c) * S + s] = tile[c][lane];
      __syncthreads();
    }
  }
}

}  // namespace

cudaError_t launch_quant_fp8_channel(const void* x, long long num_rows, int H, int E,
                                     const int32_t* expert_offset, const int32_t* expert_count,
                                     bool transpose, void* out, float* scale, int32_t* d_status,
                                     cudaStream_t stream) {
  const dim3 grid(H / kSlab, E);
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* o = static_cast<uint8_t*>(out);
  if (transpose)
    return launch_pdl(quant_fp8_channel_kernel<true>, grid, kThreads, 0, stream, xs, num_rows, H, E,
                      expert_offset, expert_count, o, scale, d_status);
  return launch_pdl(quant_fp8_channel_kernel<false>, grid, kThreads, 0, stream, xs, num_rows, H, E,
                    expert_offset, expert_count, o, scale, d_status);
}

}  // namespace moe
