// swiglu.cu -- SwiGLU between an expert's two GEMMs, fused with the
// quantisation the second GEMM reads.
//
// DeepSeek Tile-Kernels news, "Funktionen der DeepSeek-Tile-Kernel": SwiGLU
// combined with the quantisation operations.  Each receive row
// h = [gate | up] (bf16, 2I channels) becomes a = silu(gate) * up with
// silu(g) = g / (1 + e^-g) (fp32, every operation rounded once, the fixed
// exp of the gate), then a is stored as bf16 or quantised exactly as
// dispatch quantises a row: per-128-block FP8, per-row FP8 or MXFP8, the
// scales in the chosen layout.  Rows with slot_token = -1 (padding of the
// aligned layout) are skipped.
//
// Work item = (row, 512 channels of a): one warp, each lane reading 16 gate
// and 16 up channels (four 16-byte streaming loads) and writing its 16
// outputs with 16-byte stores.  Per-row FP8 needs the row's amax before any
// code: one CTA per row, the row held in registers.
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kRowThreads = 256;

// a for 8 channels from a vector of 8 gate and a vector of 8 up values, on
// every input
__device__ __forceinline__ void swiglu8(uint4 gv, uint4 uv, float* a) {
  const uint32_t g4[4] = {gv.x, gv.y, gv.z, gv.w};
  const uint32_t u4[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] = __fmul_rn(silu_exact(bf16_lo(g4[i])), bf16_lo(u4[i]));
    a[2 * i + 1] = __fmul_rn(silu_exact(bf16_hi(g4[i])), bf16_hi(u4[i]));
  }
}

// The same a when every |g| <= 87 (silu_in_range: no clamp, a corrected
// division); returns max(m, |g| over the 8), NaN if a g is NaN.  The caller
// redoes the channels with swiglu8 when the maximum is above 87 or NaN, which
// real activations almost never reach.
__device__ __forceinline__ float swiglu8_in_range(uint4 gv, uint4 uv, float* a, float m) {
  const uint32_t g4[4] = {gv.x, gv.y, gv.z, gv.w};
  const uint32_t u4[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float g0 = bf16_lo(g4[i]), g1 = bf16_hi(g4[i]);
    m = max_abs_nan(max_abs_nan(m, g0), g1);
    a[2 * i] = __fmul_rn(silu_in_range(g0), bf16_lo(u4[i]));
    a[2 * i + 1] = __fmul_rn(silu_in_range(g1), bf16_hi(u4[i]));
  }
  return m;
}

constexpr float kSiluRange = 87.0f;

// a is never NaN for finite h (silu(g) * u of finite bf16 values), so the
// encoder without NaN handling gives the same codes
__device__ __forceinline__ uint32_t e4m3x4(const float* p) {
  return e4m3x2_nonan(p[0], p[1]) | (e4m3x2_nonan(p[2], p[3]) << 16);
}

// x * f with the sign of a zero kept when f is infinite (an all-zero or
// tiny block); for finite f the product already keeps it
template <int n>
__device__ __forceinline__ void scale_keep_zero(const float* a, float f, float* p) {
  if (f <= 3.402823466e38f) {
#pragma unroll
    for (int i = 0; i < n; ++i) p[i] = __fmul_rn(a[i], f);
  } else {
#pragma unroll
    for (int i = 0; i < n; ++i) p[i] = (a[i] == 0.0f) ? a[i] : __fmul_rn(a[i], f);
  }
}

template <int DT, int SL>
__global__ void __launch_bounds__(kWarps * 32, 6)  // 40 registers, no spill: 48 warps per SM
    swiglu_quant_kernel(const uint16_t* __restrict__ h, long long S, int I,
                        const int32_t* __restrict__ slot_token, void* __restrict__ out,
                        void* __restrict__ out_scale, long long ld) {
  // grid: x = groups of kWarps rows, y = 512-channel segment (no division)
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (row >= S) return;
  const int seg = blockIdx.y;
  const int c0 = seg * 512 + lane * 16;
  const bool active = c0 < I;  // I % 16 == 0: a lane's 16 channels are all in or all out
  pdl_wait();
  pdl_trigger();
  if (slot_token && slot_token[row] < 0) return;  // the whole warp: one row

  float a[16];
  {
    const uint16_t* hr = h + static_cast<size_t>(row) * 2 * I + c0;
    uint4 g0 = make_uint4(0, 0, 0, 0), g1 = g0, u0 = g0, u1 = g0;
    if (active) {
      g0 = ld_stream(hr);
      g1 = ld_stream(hr + 8);
      u0 = ld_stream(hr + I);
      u1 = ld_stream(hr + I + 8);
    }
    float m = swiglu8_in_range(g0, u0, a, 0.0f);
    m = swiglu8_in_range(g1, u1, a + 8, m);
    if (!(m <= kSiluRange)) {
      // rare: the lane reads its 16 channels again (an L2 hit) rather than
      // keeping them live through the common path
      swiglu8(ld_stream(hr), ld_stream(hr + I), a);
      swiglu8(ld_stream(hr + 8), ld_stream(hr + I + 8), a + 8);
    }
  }

  if constexpr (DT == MOE_DTYPE_BF16) {
    if (active) {
      uint16_t* orow = static_cast<uint16_t*>(out) + static_cast<size_t>(row) * I + c0;
      st_stream_v4(orow, make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                    pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7])));
      st_stream_v4(orow + 8, make_uint4(pack_bf16x2(a[8], a[9]), pack_bf16x2(a[10], a[11]),
                                        pack_bf16x2(a[12], a[13]), pack_bf16x2(a[14], a[15])));
    }
  } else {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(a[i]));
    uint8_t* orow = static_cast<uint8_t*>(out) + static_cast<size_t>(row) * I;
    if constexpr (DT == MOE_DTYPE_FP8_E4M3) {
      // 8 lanes = one 128-channel block
      amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 4));
      // the block's 448 / amax and amax / 448 from one division per lane:
      // even lanes take the first, odd lanes the second
      const bool odd = lane & 1;
      const float q = __fdiv_rn(odd ? amax : 448.0f, odd ? 448.0f : amax);
      const float inv = __shfl_sync(kFullMask, q, lane & ~7);
      const float scale = __shfl_sync(kFullMask, q, (lane & ~7) | 1);
      float p[16];
      scale_keep_zero<16>(a, inv, p);
      if (active) {
        st_stream_v4(orow + c0, make_uint4(e4m3x4(p), e4m3x4(p + 4), e4m3x4(p + 8), e4m3x4(p + 12)));
        if ((lane & 7) == 0)
          static_cast<float*>(out_scale)[scale_at<SL>(row, c0 >> 7, I / 128, ld)] = scale;
      }
    } else {
      // MXFP8: 2 lanes = one 32-channel block
      amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
      int e = amax > 0.0f ? floor_log2_pos(amax) - 8 : -127;
      e = e < -127 ? -127 : (e > 127 ? 127 : e);
      const float down = __int_as_float((127 - e) << 23);  // 2^-e, e in [-127, 119]
      float p[16];
      scale_keep_zero<16>(a, down, p);  // down is a finite power of two
      if (active)
        st_stream_v4(orow + c0, make_uint4(e4m3x4(p), e4m3x4(p + 4), e4m3x4(p + 8), e4m3x4(p + 12)));
      const int nblk = I / 32;
      const uint32_t my_byte = static_cast<uint32_t>(e + 127);
      uint8_t* sc = static_cast<uint8_t*>(out_scale);
      if constexpr (SL == MOE_SCALE_MN_MAJOR) {
        if (active && (lane & 1) == 0) sc[scale_at<SL>(row, c0 >> 5, nblk, ld)] = static_cast<uint8_t>(my_byte);
      } else {
        // the warp's 16 block bytes (block j from lane 2j) as 4 words, word i
        // = blocks 4i..4i+3 gathered on lane 8i in two shuffles
        uint32_t word = my_byte | (__shfl_down_sync(kFullMask, my_byte, 2) << 8);
        word |= __shfl_down_sync(kFullMask, word, 4) << 16;
        const int b0 = seg * 16 + (lane >> 1);
        if ((lane & 7) == 0 && b0 < nblk) {
          if constexpr (SL == MOE_SCALE_MMA_TILED) {
            *reinterpret_cast<uint32_t*>(sc + scale_at<SL>(row, b0, nblk, ld)) = word;
          } else {
            // row-major: row*nblk + b0 need not be 4-byte aligned, so byte stores
            uint8_t* dst = sc + static_cast<size_t>(row) * nblk + b0;
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (b0 + u < nblk) dst[u] = static_cast<uint8_t>(word >> (8 * u));
          }
        }
      }
    }
  }
}

// Per-row FP8: one CTA per row, VPT vectors of 8 channels per thread.
template <int VPT>
__global__ void __launch_bounds__(kRowThreads, 1)
    swiglu_fp8_row_kernel(const uint16_t* __restrict__ h, int I,
                          const int32_t* __restrict__ slot_token, uint8_t* __restrict__ out,
                          float* __restrict__ out_scale) {
  __shared__ float warp_max[kRowThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long row = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (slot_token && slot_token[row] < 0) return;  // the whole CTA: one row
  const int nvec = I / 8;
  const uint16_t* hr = h + static_cast<size_t>(row) * 2 * I;
  float a[VPT][8];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = i * kRowThreads + tid;
    uint4 gv = make_uint4(0, 0, 0, 0), uv = gv;
    if (vi < nvec) {
      gv = ld_stream(hr + static_cast<size_t>(vi) * 8);
      uv = ld_stream(hr + I + static_cast<size_t>(vi) * 8);
    }
    if (!(swiglu8_in_range(gv, uv, a[i], 0.0f) <= kSiluRange))
      swiglu8(ld_stream(hr + static_cast<size_t>(vi) * 8), ld_stream(hr + I + static_cast<size_t>(vi) * 8),
              a[i]);
#pragma unroll
    for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(a[i][u]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, o));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < kRowThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);
  const float inv = __fdiv_rn(448.0f, amax);
  const float scale = __fdiv_rn(amax, 448.0f);
  uint8_t* orow = out + static_cast<size_t>(row) * I;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = i * kRowThreads + tid;
    float p[8];
    scale_keep_zero<8>(a[i], inv, p);
    if (vi < nvec)
      *reinterpret_cast<uint2*>(orow + static_cast<size_t>(vi) * 8) = make_uint2(e4m3x4(p), e4m3x4(p + 4));
  }
  if (tid == 0) out_scale[row] = scale;  // row-major and MN-major agree for one block per row
}

template <int DT, int SL>
cudaError_t launch_warp_kernel(const uint16_t* h, long long S, int I, const int32_t* slot_token,
                               void* out, void* out_scale, long long ld, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((S + kWarps - 1) / kWarps), (I + 511) / 512);
  return launch_pdl(swiglu_quant_kernel<DT, SL>, grid, kWarps * 32, 0, stream, h, S, I,
                    slot_token, out, out_scale, ld);
}

}  // namespace

cudaError_t launch_swiglu_quant(const void* h, long long num_rows, int I, const int32_t* slot_token,
                                int dtype, int scale_layout, void* out, void* out_scale,
                                cudaStream_t stream) {
  if (num_rows == 0) return cudaSuccess;
  const uint16_t* hs = static_cast<const uint16_t*>(h);
  const long long ld = scale_ld(num_rows, dtype);
  switch (dtype) {
    case MOE_DTYPE_BF16:
      return launch_warp_kernel<MOE_DTYPE_BF16, MOE_SCALE_ROW_MAJOR>(hs, num_rows, I, slot_token, out,
                                                                   out_scale, ld, stream);
    case MOE_DTYPE_FP8_E4M3:
      if (scale_layout == MOE_SCALE_MN_MAJOR)
        return launch_warp_kernel<MOE_DTYPE_FP8_E4M3, MOE_SCALE_MN_MAJOR>(hs, num_rows, I, slot_token,
                                                                         out, out_scale, ld, stream);
      return launch_warp_kernel<MOE_DTYPE_FP8_E4M3, MOE_SCALE_ROW_MAJOR>(hs, num_rows, I, slot_token,
                                                                        out, out_scale, ld, stream);
    case MOE_DTYPE_MXFP8_E4M3:
      if (scale_layout == MOE_SCALE_MN_MAJOR)
        return launch_warp_kernel<MOE_DTYPE_MXFP8_E4M3, MOE_SCALE_MN_MAJOR>(hs, num_rows, I, slot_token,
                                                                           out, out_scale, ld, stream);
      if (scale_layout == MOE_SCALE_MMA_TILED)
        return launch_warp_kernel<MOE_DTYPE_MXFP8_E4M3, MOE_SCALE_MMA_TILED>(hs, num_rows, I, slot_token,
                                                                            out, out_scale, ld, stream);
      return launch_warp_kernel<MOE_DTYPE_MXFP8_E4M3, MOE_SCALE_ROW_MAJOR>(hs, num_rows, I, slot_token,
                                                                          out, out_scale, ld, stream);
    default: {  // per-row FP8
      const int vpt = (I / 8 + kRowThreads - 1) / kRowThreads;
      uint8_t* o8 = static_cast<uint8_t*>(out);
      float* sc = static_cast<float*>(out_scale);
      const unsigned rows = static_cast<unsigned>(num_rows);
      if (vpt <= 1)
        return launch_pdl(swiglu_fp8_row_kernel<1>, rows, kRowThreads, 0, stream, hs, I, slot_token, o8, sc);
      if (vpt <= 2)
        return launch_pdl(swiglu_fp8_row_kernel<2>, rows, kRowThreads, 0, stream, hs, I, slot_token, o8, sc);
      if (vpt <= 4)
        return launch_pdl(swiglu_fp8_row_kernel<4>, rows, kRowThreads, 0, stream, hs, I, slot_token, o8, sc);
      return launch_pdl(swiglu_fp8_row_kernel<8>, rows, kRowThreads, 0, stream, hs, I, slot_token, o8, sc);
    }
  }
}

}  // namespace moe
