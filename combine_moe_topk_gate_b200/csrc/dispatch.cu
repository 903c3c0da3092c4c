// dispatch.cu -- scatter each token's hidden row to its k receive rows,
// optionally quantising it to FP8 e4m3 with one fp32 scale per 128 channels.
//
// [pplx] "Efficient and portable mixture-of-experts communication",
// Dispatch: a token's activations, with block scaling factors when quantised,
// go to every expert it was routed to, unpacked into a contiguous buffer per
// expert.  DeepEP V2 summary, usage patterns: BF16 and FP8 dispatch.
// DeepSeek Tile-Kernels news: per-block FP8 quantisation.
//
// Work item = (token, segment).  One warp per item reads the segment of the
// row once (16-byte streaming loads), converts it in registers and stores it
// k times (16-byte stores, 512 contiguous bytes per warp and slot).  The
// segments of one token sit in neighbouring warps of one CTA, so a CTA writes
// long contiguous runs of every destination row.
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kWarps = 8;

// FP8: lane owns 16 channels (two 16-byte loads), 8 lanes = one 128-block,
// a warp covers 512 channels.
// ceil(log2(q)) for q > 0 finite, exact from the bits (subnormals too)
__device__ __forceinline__ int ceil_log2_pos(float q) {
  const uint32_t u = __float_as_uint(q);
  const uint32_t m = u & 0x7fffffu;
  const int ex = static_cast<int>((u >> 23) & 0xffu);
  if (ex) return ex - 127 + (m != 0u);
  const int fl = (31 - __clz(m)) - 149;
  return fl + ((m & (m - 1u)) != 0u);
}

// UE8M0 = true: power-of-two scale 2^e per 128-block with e = ceil(log2(amax /
// 448)) of the fp32 quotient, stored as the byte e + 127; codes e4m3(x * 2^-e)
// (exact scaling, so a zero keeps its sign without a select).
// SPW = segments per warp: with SPW = 2 a warp owns two neighbouring
// 512-channel segments of its token and issues both segments' loads before
// working on the first, twice the bytes in flight per warp -- for small k,
// where reading x is most of the traffic and load latency sets the pace.
template <int SL, bool UE8M0 = false, int SPW = 1>
__global__ void __launch_bounds__(kWarps * 32)
    dispatch_fp8_kernel(const uint16_t* __restrict__ x, int N, int H, int k,
                        const int32_t* __restrict__ token_slot, long long S,
                        uint8_t* __restrict__ recv_x, float* __restrict__ recv_scale,
                        long long ld, int32_t* d_status) {
  const int lane = threadIdx.x & 31;
  const int segs = (H + 511) / 512;
  const int groups = (segs + SPW - 1) / SPW;  // work items per token
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(N) * groups) return;
  const int t = static_cast<int>(item / groups);
  const int s0 = static_cast<int>(item - static_cast<long long>(t) * groups) * SPW;
  const int nblk = H / 128;
  pdl_wait();
  pdl_trigger();

  const int my_slot = lane < k ? token_slot[static_cast<size_t>(t) * k + lane] : -1;
  uint4 av[SPW], bv[SPW];
#pragma unroll
  for (int u = 0; u < SPW; ++u) {
    const int c0 = (s0 + u) * 512 + lane * 16;
    av[u] = make_uint4(0, 0, 0, 0);
    bv[u] = make_uint4(0, 0, 0, 0);
    if (c0 < H) {  // H % 128 == 0: whole 8-lane blocks are in or out
      const uint16_t* src = x + static_cast<size_t>(t) * H + c0;
      av[u] = ld_stream(src);
      bv[u] = ld_stream(src + 8);
    }
  }
#pragma unroll
  for (int u = 0; u < SPW; ++u) {
    const int s = s0 + u;
    if (s >= segs) break;  // warp-uniform
    const int c0 = s * 512 + lane * 16;
    const bool active = c0 < H;
    const uint4 a = av[u], b = bv[u];
    float f[16];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[2 * i] = bf16_lo(w[i]);
      f[2 * i + 1] = bf16_hi(w[i]);
    }
    // A warp whose values are all finite (the usual case) takes the encoder
    // without NaN fix-ups: no input NaN, and no inf * 0 in the scaling.  The
    // maximum with NaN propagation doubles as the block amax there.
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = max_abs_nan(amax, f[i]);
    const bool special = __any_sync(kFullMask, !(amax <= 3.402823466e38f));
    if (special) {  // warp-uniform: the amax ignores NaN, as the definition does
      amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 4));
    float inv, scale = 0.0f;
    uint32_t sword = 0;  // UE8M0: the warp's 4 block bytes (block i in byte i)
    if constexpr (UE8M0) {
      int e = amax > 0.0f ? ceil_log2_pos(__fdiv_rn(amax, 448.0f)) : -127;
      e = e < -127 ? -127 : (e > 127 ? 127 : e);
      // 2^-e exactly: a normal float for e <= 126 (every finite bf16 block:
      // e <= 120), the subnormal 2^-127 for an infinite amax (e = 127)
      inv = e < 127 ? __int_as_float((127 - e) << 23) : __int_as_float(0x00400000);
      const uint32_t byte = static_cast<uint32_t>(e + 127);
#pragma unroll
      for (int i = 0; i < 4; ++i) sword |= (__shfl_sync(kFullMask, byte, 8 * i) & 0xffu) << (8 * i);
    } else {
      // the block's 448 / amax and amax / 448 from one division per lane:
      // even lanes take the first, odd lanes the second
      const bool odd = lane & 1;
      const float qd = __fdiv_rn(odd ? amax : 448.0f, odd ? 448.0f : amax);
      inv = __shfl_sync(kFullMask, qd, lane & ~7);
      scale = __shfl_sync(kFullMask, qd, (lane & ~7) | 1);
    }
    // a finite factor keeps the sign of a zero by itself; an infinite one (an
    // all-zero or tiny block) needs the select
    float p[16];
    if (UE8M0 || inv <= 3.402823466e38f) {
#pragma unroll
      for (int i = 0; i < 16; ++i) p[i] = __fmul_rn(f[i], inv);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) p[i] = f[i] != 0.0f ? __fmul_rn(f[i], inv) : f[i];  // zero keeps its sign
    }
    uint32_t q[4];
    if (special) {
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = e4m3x2(p[4 * i], p[4 * i + 1]) | (e4m3x2(p[4 * i + 2], p[4 * i + 3]) << 16);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        q[i] = e4m3x2_nonan(p[4 * i], p[4 * i + 1]) | (e4m3x2_nonan(p[4 * i + 2], p[4 * i + 3]) << 16);
    }
    const uint4 qv = make_uint4(q[0], q[1], q[2], q[3]);
    for (int j = 0; j < k; ++j) {
      const int slot = __shfl_sync(kFullMask, my_slot, j);
      if (slot == -1) continue;
      if (slot < -1 || slot >= S) {
        if (lane == 0 && u == 0) report_bad_index(d_status);
        continue;
      }
      if (active) st_stream_v4(recv_x + static_cast<size_t>(slot) * H + c0, qv);
      if constexpr (!UE8M0) {
        if (active && (lane & 7) == 0) {
          if constexpr (SL == MOE_SCALE_ROW_MAJOR)
            recv_scale[scale_at<SL>(slot, c0 >> 7, nblk, ld)] = scale;
          else
            st_keep_b32(recv_scale + scale_at<SL>(slot, c0 >> 7, nblk, ld), __float_as_uint(scale),
                        l2_evict_last_policy());
        }
      } else {
        uint8_t* sb = reinterpret_cast<uint8_t*>(recv_scale);
        if constexpr (SL == MOE_SCALE_MN_MAJOR_PACK4) {
          // the warp's 4 blocks are exactly word s of the row
          if (lane == 0) *reinterpret_cast<uint32_t*>(sb + scale_at<SL>(slot, 4 * s, nblk, ld)) = sword;
        } else if (SL == MOE_SCALE_ROW_MAJOR && (nblk & 3) == 0) {
          if (lane == 0) *reinterpret_cast<uint32_t*>(sb + static_cast<size_t>(slot) * nblk + 4 * s) = sword;
        } else if (active && (lane & 7) == 0) {
          sb[scale_at<SL>(slot, c0 >> 7, nblk, ld)] = static_cast<uint8_t>(sword >> (lane & 24));
        }
      }
    }
  }
}

// MXFP8 (OCP Microscaling): 32-element blocks share X = 2^e with
// e = floor(log2(amax)) - 8, stored as the E8M0 byte e + 127; elements are
// e4m3(x * 2^-e), saturating (x * 2^-e can reach 511.x).  Same work split as
// the per-block kernel: lane owns 16 channels, 2 lanes = one block, a warp
// covers 512 channels and gathers its 16 scale bytes into one 16-byte store.

template <int SL, int SPW = 1>  // SPW: segments per warp, as in the FP8 kernel
__global__ void __launch_bounds__(kWarps * 32)
    dispatch_mxfp8_kernel(const uint16_t* __restrict__ x, int N, int H, int k,
                          const int32_t* __restrict__ token_slot, long long S,
                          uint8_t* __restrict__ recv_x, uint8_t* __restrict__ recv_e8m0,
                          long long ld, int32_t* d_status) {
  const int lane = threadIdx.x & 31;
  const int segs = (H + 511) / 512;
  const int groups = (segs + SPW - 1) / SPW;  // work items per token
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(N) * groups) return;
  const int t = static_cast<int>(item / groups);
  const int s0 = static_cast<int>(item - static_cast<long long>(t) * groups) * SPW;
  const int nblk = H / 32;
  pdl_wait();
  pdl_trigger();

  const int my_slot = lane < k ? token_slot[static_cast<size_t>(t) * k + lane] : -1;
  uint4 av[SPW], bv[SPW];
#pragma unroll
  for (int u = 0; u < SPW; ++u) {
    const int cu = (s0 + u) * 512 + lane * 16;
    av[u] = make_uint4(0, 0, 0, 0);
    bv[u] = make_uint4(0, 0, 0, 0);
    if (cu < H) {  // H % 32 == 0: whole 2-lane blocks are in or out
      const uint16_t* src = x + static_cast<size_t>(t) * H + cu;
      av[u] = ld_stream(src);
      bv[u] = ld_stream(src + 8);
    }
  }
#pragma unroll
  for (int u = 0; u < SPW; ++u) {
  const int s = s0 + u;
  if (s >= segs) break;  // warp-uniform
  const int c0 = s * 512 + lane * 16;
  const bool active = c0 < H;
  const uint4 a = av[u], b = bv[u];
  float f[16];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = bf16_lo(w[i]);
    f[2 * i + 1] = bf16_hi(w[i]);
  }
  // all-finite warps take the encoder without NaN fix-ups (as in the FP8
  // kernel; the scaling by a finite power of two makes no NaN)
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = max_abs_nan(amax, f[i]);
  const bool special = __any_sync(kFullMask, !(amax <= 3.402823466e38f));
  if (special) {  // warp-uniform: the amax ignores NaN, as the definition does
    amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
  amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
  int e = amax > 0.0f ? floor_log2_pos(amax) - 8 : -127;
  e = e < -127 ? -127 : (e > 127 ? 127 : e);
  // 2^-e, e in [-127, 127]: a finite power of two, so every product keeps a
  // zero's sign and scales exactly (short of underflow)
  const float down = __int_as_float((127 - e) << 23);
  uint32_t q[4];
  {
    float p[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i] = __fmul_rn(f[i], down);
    if (special) {
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = e4m3x2(p[4 * i], p[4 * i + 1]) | (e4m3x2(p[4 * i + 2], p[4 * i + 3]) << 16);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        q[i] = e4m3x2_nonan(p[4 * i], p[4 * i + 1]) | (e4m3x2_nonan(p[4 * i + 2], p[4 * i + 3]) << 16);
    }
  }
  const uint4 qv = make_uint4(q[0], q[1], q[2], q[3]);
  // the warp's 16 scale bytes (block j from lane 2j) as 4 words, word i =
  // blocks 4i..4i+3 gathered on lane 8i in two shuffles
  const uint32_t my_byte = static_cast<uint32_t>(e + 127);
  uint32_t word = my_byte | (__shfl_down_sync(kFullMask, my_byte, 2) << 8);
  word |= __shfl_down_sync(kFullMask, word, 4) << 16;
  const bool whole16 = (H % 512) == 0;  // full 16 scale bytes per warp
  for (int j = 0; j < k; ++j) {
    const int slot = __shfl_sync(kFullMask, my_slot, j);
    if (slot == -1) continue;
    if (slot < -1 || slot >= S) {
      if (lane == 0 && u == 0) report_bad_index(d_status);
      continue;
    }
    if (active) st_stream_v4(recv_x + static_cast<size_t>(slot) * H + c0, qv);
    if constexpr (SL == MOE_SCALE_ROW_MAJOR) {
      uint8_t* srow = recv_e8m0 + static_cast<size_t>(slot) * nblk;
      if (whole16) {  // nblk % 16 == 0: the 4 words are 4-byte aligned
        if ((lane & 7) == 0) *reinterpret_cast<uint32_t*>(srow + s * 16 + (lane >> 1)) = word;
      } else if (active && (lane & 1) == 0) {
        srow[c0 >> 5] = static_cast<uint8_t>(my_byte);
      }
    } else if constexpr (SL == MOE_SCALE_MMA_TILED) {
      // blocks 4i..4i+3 are 4 consecutive bytes of one atom (nblk % 4 == 0):
      // lane 8i stores word i of the warp's 16 blocks
      const int b0 = s * 16 + (lane >> 1);
      if ((lane & 7) == 0 && b0 < nblk)
        st_keep_b32(recv_e8m0 + scale_at<SL>(slot, b0, nblk, ld), word, l2_evict_last_policy());
    } else {
      if (active && (lane & 1) == 0)
        st_keep_b8(recv_e8m0 + scale_at<SL>(slot, c0 >> 5, nblk, ld), my_byte, l2_evict_last_policy());
    }
  }
  }  // segments of the warp
}

// FP8 with one scale per token: one 128-thread CTA per token.  One thread
// copies the row into shared memory with a 1-D bulk copy (no tensor map, no
// multicast) completing on an mbarrier; the CTA reduces the row amax from
// shared memory and codes its VPT 8-channel vectors per thread with the
// block rule: scale = amax/448, codes e4m3(x * (448/amax)).  The row does not
// occupy registers, so many tokens are in flight per SM.  The copy's wait is
// bounded (MOE_ERR_TIMEOUT), the give-up decision taken by one thread.
constexpr int kTokenThreads = 128;

template <int VPT>
__global__ void __launch_bounds__(kTokenThreads)
    dispatch_fp8_token_kernel(const uint16_t* __restrict__ x, int N, int H, int k,
                              const int32_t* __restrict__ token_slot, long long S,
                              uint8_t* __restrict__ recv_x, float* __restrict__ recv_scale,
                              int32_t* d_status) {
  extern __shared__ __align__(128) unsigned char smem[];  // mbarrier at 0, the row from 128
  __shared__ float warp_max[kTokenThreads / 32];
  __shared__ int slots[MOE_MAX_TOPK];
  __shared__ int copy_ok;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = blockIdx.x;
  const int nvec = H / 8;
  const uint32_t bar = smem_addr(smem);
  const uint32_t row = smem_addr(smem + 128);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(H) * 2u);
    bulk_g2s(row, x + static_cast<size_t>(t) * H, static_cast<uint32_t>(H) * 2u, bar);
  }
  if (tid < k) {
    const int sl = token_slot[static_cast<size_t>(t) * k + tid];
    slots[tid] = sl;
    if (sl < -1 || sl >= S) report_bad_index(d_status);
  }
  if (tid == 0) {
    copy_ok = mbar_wait(bar, 0) ? 1 : 0;
    if (!copy_ok) {
      report_timeout(d_status);
      mbar_wait(bar, 0);  // bounded again: the copy must land before the CTA may exit
    }
  }
  __syncthreads();
  if (!copy_ok) return;
  mbar_wait(bar, 0);  // the phase has completed: returns at once (and is bounded regardless)

  // the row amax with NaN propagation; a row whose values are all finite
  // (the usual case) takes the encoder without NaN fix-ups
  auto row_amax = [&](bool nan_max) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vi = i * kTokenThreads + tid;
      if (vi < nvec) {
        const uint4 v = ld_shared_v4(row + vi * 16);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (nan_max) {
            m = max_abs_nan(max_abs_nan(m, bf16_lo(w4[u])), bf16_hi(w4[u]));
          } else {
            m = fmaxf(m, fmaxf(fabsf(bf16_lo(w4[u])), fabsf(bf16_hi(w4[u]))));
          }
        }
      }
    }
    return m;
  };
  float amax = row_amax(true);
  const bool special = !(amax <= 3.402823466e38f);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, o));
  if (lane == 0) warp_max[warp] = amax;
  const bool any_special = __syncthreads_or(special);
  if (any_special) {  // CTA-uniform: the amax ignores NaN, as the definition does
    amax = row_amax(false);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, o));
    if (lane == 0) warp_max[warp] = amax;  // nobody has read the first values yet
    __syncthreads();
  }
  amax = fmaxf(fmaxf(warp_max[0], warp_max[1]), fmaxf(warp_max[2], warp_max[3]));
  const float inv = __fdiv_rn(448.0f, amax);
  const float scale = __fdiv_rn(amax, 448.0f);
  const bool finite = inv <= 3.402823466e38f;  // then the product keeps a zero's sign
  uint2 q[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = i * kTokenThreads + tid;
    q[i] = make_uint2(0, 0);
    if (vi < nvec) {
      const uint4 v = ld_shared_v4(row + vi * 16);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float p[8];
      if (finite) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          p[2 * u] = __fmul_rn(bf16_lo(w4[u]), inv);
          p[2 * u + 1] = __fmul_rn(bf16_hi(w4[u]), inv);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float lo = bf16_lo(w4[u]), hi = bf16_hi(w4[u]);
          p[2 * u] = lo != 0.0f ? __fmul_rn(lo, inv) : lo;
          p[2 * u + 1] = hi != 0.0f ? __fmul_rn(hi, inv) : hi;
        }
      }
      if (any_special) {
        q[i].x = e4m3x2(p[0], p[1]) | (e4m3x2(p[2], p[3]) << 16);
        q[i].y = e4m3x2(p[4], p[5]) | (e4m3x2(p[6], p[7]) << 16);
      } else {
        q[i].x = e4m3x2_nonan(p[0], p[1]) | (e4m3x2_nonan(p[2], p[3]) << 16);
        q[i].y = e4m3x2_nonan(p[4], p[5]) | (e4m3x2_nonan(p[6], p[7]) << 16);
      }
    }
  }
  for (int j = 0; j < k; ++j) {
    const int slot = slots[j];
    if (slot < 0 || slot >= S) continue;
    uint8_t* dst = recv_x + static_cast<size_t>(slot) * H;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vi = i * kTokenThreads + tid;
      if (vi < nvec) *reinterpret_cast<uint2*>(dst + static_cast<size_t>(vi) * 8) = q[i];
    }
    if (tid == 0) recv_scale[slot] = scale;
  }
}

// NVFP4: one CTA of THREADS threads per token (128, or 64 for rows of up to
// 4096 channels).  One thread copies the token's row into shared memory with
// a 1-D bulk copy (no tensor map, no multicast) that completes on an
// mbarrier; the CTA then works from shared memory, so the row does not
// occupy registers and many tokens are in flight per SM.  Each thread owns
// the 16-channel blocks tid, tid + THREADS, ... (BPT of them): block maxima, the
// CTA-wide row amax (row scale g = amax / 2688, inv = 2688 / amax), then per
// block sb = e4m3((amax_b / 6) * inv), r = inv / value(sb), codes e2m1(x * r).
// Four neighbouring threads hold four consecutive blocks, so their scale
// bytes leave as one 32-bit word (H % 64 == 0).  The copy's wait is bounded
// (MOE_ERR_TIMEOUT).
constexpr int kNvThreads = 128;
constexpr int kNvThreadsShort = 64;  // rows of up to 4096 channels

template <int BPT, int SL, int THREADS>
__global__ void __launch_bounds__(THREADS)
    dispatch_nvfp4_kernel(const uint16_t* __restrict__ x, int N, int H, int k,
                          const int32_t* __restrict__ token_slot, long long S,
                          uint8_t* __restrict__ recv_x, uint8_t* __restrict__ block_scale,
                          float* __restrict__ row_scale, long long ld, int32_t* d_status) {
  extern __shared__ __align__(128) unsigned char smem[];  // mbarrier at 0, the row from 128
  __shared__ float warp_max[THREADS / 32];
  __shared__ int slots[MOE_MAX_TOPK];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = blockIdx.x;
  const int nb = H / 16;
  const uint32_t bar = smem_addr(smem);
  const uint32_t row = smem_addr(smem + 128);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(H) * 2u);
    bulk_g2s(row, x + static_cast<size_t>(t) * H, static_cast<uint32_t>(H) * 2u, bar);
  }
  if (tid < k) {
    const int sl = token_slot[static_cast<size_t>(t) * k + tid];
    slots[tid] = sl;
    if (sl < -1 || sl >= S) report_bad_index(d_status);
  }
  // one thread takes the bounded wait, so the give-up decision is the same
  // for the whole CTA (no thread may leave while others reach a barrier);
  // after it every thread observes the completed phase, which makes the
  // copied bytes visible to it
  __shared__ int copy_ok;
  if (tid == 0) {
    copy_ok = mbar_wait(bar, 0) ? 1 : 0;
    if (!copy_ok) {
      report_timeout(d_status);
      mbar_wait(bar, 0);  // bounded again: the copy must land before the CTA may exit
    }
  }
  __syncthreads();
  if (!copy_ok) return;
  mbar_wait(bar, 0);  // the phase has completed: returns at once (and is bounded regardless)

  float bmax[BPT];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    const int b = tid + i * THREADS;
    bmax[i] = 0.0f;
    if (b < nb) {
      const uint4 va = ld_shared_v4(row + b * 32), vb = ld_shared_v4(row + b * 32 + 16);
      const uint32_t w[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int u = 0; u < 8; ++u) bmax[i] = fmaxf(bmax[i], fmaxf(fabsf(bf16_lo(w[u])), fabsf(bf16_hi(w[u]))));
    }
    amax = fmaxf(amax, bmax[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, o));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < THREADS / 32; ++w) amax = fmaxf(amax, warp_max[w]);
  const float g = __fdiv_rn(amax, 2688.0f);
  const float inv = __fdiv_rn(2688.0f, amax);
  uint2 q[BPT];
  uint32_t sword[BPT];
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    const int b = tid + i * THREADS;
    const float sbf = __fmul_rn(__fdiv_rn(bmax[i], 6.0f), inv);
    const uint32_t sb = bmax[i] > 0.0f ? (e4m3x2(sbf, 0.0f) & 0xffu) : 0u;
    q[i] = make_uint2(0, 0);
    if (b < nb) {
      const float r = __fdiv_rn(inv, e4m3_value(sb));
      const uint4 va = ld_shared_v4(row + b * 32), vb = ld_shared_v4(row + b * 32 + 16);
      const uint32_t w[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
      float p[16];
      if (r <= 3.402823466e38f) {  // finite: the product keeps a zero's sign
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          p[2 * u] = __fmul_rn(bf16_lo(w[u]), r);
          p[2 * u + 1] = __fmul_rn(bf16_hi(w[u]), r);
        }
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float lo = bf16_lo(w[u]), hi = bf16_hi(w[u]);
          p[2 * u] = (lo == 0.0f) ? lo : __fmul_rn(lo, r);
          p[2 * u + 1] = (hi == 0.0f) ? hi : __fmul_rn(hi, r);
        }
      }
      q[i] = make_uint2(e2m1x8(p), e2m1x8(p + 8));
    }
    // bytes of blocks b..b+3 (threads tid..tid+3) into tid % 4 == 0
    uint32_t word = sb;
    word |= (__shfl_down_sync(kFullMask, sb, 1) & 0xffu) << 8;
    word |= (__shfl_down_sync(kFullMask, sb, 2) & 0xffu) << 16;
    word |= (__shfl_down_sync(kFullMask, sb, 3) & 0xffu) << 24;
    sword[i] = SL == MOE_SCALE_MN_MAJOR ? sb : word;
  }
  const size_t row_bytes = static_cast<size_t>(H) / 2;
  for (int j = 0; j < k; ++j) {
    const int slot = slots[j];
    if (slot < 0 || slot >= S) continue;
    uint8_t* dst = recv_x + static_cast<size_t>(slot) * row_bytes;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int b = tid + i * THREADS;
      if (b < nb) {
        *reinterpret_cast<uint2*>(dst + static_cast<size_t>(b) * 8) = q[i];
        if constexpr (SL == MOE_SCALE_MN_MAJOR) {
          block_scale[scale_at<SL>(slot, b, nb, ld)] = static_cast<uint8_t>(sword[i]);
        } else if ((tid & 3) == 0) {
          *reinterpret_cast<uint32_t*>(block_scale + scale_at<SL>(slot, b, nb, ld)) = sword[i];
        }
      }
    }
    if (tid == 0) row_scale[slot] = g;
  }
}

// E5M6 (12-bit float: FP16 without its 4 lowest fraction bits), rounded to
// nearest even, saturating to +-65024.  Normal range: rebias the fp32
// exponent (127 -> 15) and round the fraction to 6 bits in the integer
// domain; subnormals (|f| < 2^-14) in units of 2^-20, rounded by adding
// 1.5 * 2^23 (the product |f| * 2^20 is exact and below 64).
__device__ __forceinline__ uint32_t e5m6_code(float f) {
  const uint32_t u = __float_as_uint(f);
  const uint32_t sign = (u >> 20) & 0x800u;
  const uint32_t a = u & 0x7fffffffu;
  if (a > 0x7f800000u) return sign | 0x7ffu;  // NaN
  if (a >= 0x38800000u) {
    const uint32_t r = a - (112u << 23);
    const uint32_t c = (r + 0xffffu + ((r >> 17) & 1u)) >> 17;
    return sign | (c >= 0x7c0u ? 0x7bfu : c);
  }
  const float t = __fadd_rn(__fmul_rn(__uint_as_float(a), 0x1p20f), 12582912.0f);
  return sign | (__float_as_uint(t) - 0x4B400000u);
}

// The same codes for two bf16 values at once (w: low half first) when both
// magnitudes lie in [2^-14, 65024], the range where the code is the bf16
// exponent rebiased (127 -> 15) with the 7-bit fraction rounded to 6 bits
// (ties to even) and no saturation: on the 16-bit halves, r = |h| - (112 << 7)
// and the code is (r + bit 1 of r) >> 1.  No half carries into the other.
// Returns the 24-bit pair (low value's code in bits 0..11).
__device__ __forceinline__ uint32_t e5m6_pair_normal(uint32_t w) {
  const uint32_t r = (w & 0x7fff7fffu) - 0x38003800u;
  const uint32_t c = (r + ((r >> 1) & 0x00010001u)) >> 1;
  const uint32_t lo = (c & 0x7ffu) | ((w >> 4) & 0x800u);
  const uint32_t hi = ((c >> 16) & 0x7ffu) | ((w >> 20) & 0x800u);
  return lo | (hi << 12);
}
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// E5M6 dispatch: lane owns 16 channels (two 16-byte loads) -> 16 codes ->
// 24 bytes (two codes per 3 bytes, little endian).  The warp's 768 bytes are
// staged in shared memory and leave as 16-byte streaming stores covering 512
// and 256 contiguous bytes (lanes 0..31, then 0..15), so no sector is
// written in pieces.  SPW: segments per warp, as in the FP8 kernel.
template <int SPW = 1>
__global__ void __launch_bounds__(kWarps * 32)
    dispatch_e5m6_kernel(const uint16_t* __restrict__ x, int N, int H, int k,
                         const int32_t* __restrict__ token_slot, long long S,
                         uint8_t* __restrict__ recv_x, int32_t* d_status) {
  __shared__ __align__(16) uint2 stage[kWarps][96];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int segs = (H + 511) / 512;
  const int groups = (segs + SPW - 1) / SPW;  // work items per token
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(N) * groups) return;
  const int t = static_cast<int>(item / groups);
  const int s0 = static_cast<int>(item - static_cast<long long>(t) * groups) * SPW;
  pdl_wait();
  pdl_trigger();
  const int my_slot = lane < k ? token_slot[static_cast<size_t>(t) * k + lane] : -1;
  uint4 av[SPW], bv[SPW];
#pragma unroll
  for (int u = 0; u < SPW; ++u) {
    const int cu = (s0 + u) * 512 + lane * 16;
    av[u] = make_uint4(0, 0, 0, 0);
    bv[u] = av[u];
    if (cu < H) {  // H % 32 == 0: 16 whole channels or none
      const uint16_t* src = x + static_cast<size_t>(t) * H + cu;
      av[u] = ld_stream(src);
      bv[u] = ld_stream(src + 8);
    }
  }
#pragma unroll
  for (int u = 0; u < SPW; ++u) {
  const int s = s0 + u;
  if (s >= segs) break;  // warp-uniform
  const uint4 a = av[u], b = bv[u];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t p[8];  // 24-bit pairs
  // the lane's 16 magnitudes all in [2^-14, 65024] (no zero, subnormal,
  // saturating value, infinity or NaN): the two-at-a-time codes
  uint32_t hmax = 0u, hmin = 0xffffffffu;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    hmax = max_u16x2(hmax, w[i] & 0x7fff7fffu);
    hmin = min_u16x2(hmin, w[i] & 0x7fff7fffu);
  }
  const uint32_t top = max(hmax & 0xffffu, hmax >> 16), bottom = min(hmin & 0xffffu, hmin >> 16);
  if (top <= 0x477Eu && bottom >= 0x3880u) {
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = e5m6_pair_normal(w[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = e5m6_code(bf16_lo(w[i])) | (e5m6_code(bf16_hi(w[i])) << 12);
  }
  if (u > 0) __syncwarp();  // every lane has read the previous segment's stage
  stage[warp][3 * lane] = make_uint2(p[0] | (p[1] << 24), (p[1] >> 8) | (p[2] << 16));
  stage[warp][3 * lane + 1] = make_uint2((p[2] >> 16) | (p[3] << 8), p[4] | (p[5] << 24));
  stage[warp][3 * lane + 2] = make_uint2((p[5] >> 8) | (p[6] << 16), (p[6] >> 16) | (p[7] << 8));
  __syncwarp();
  // 16-byte chunk c of the warp's 768 bytes: lanes take c = lane and c = 32 + lane
  const uint4* st4 = reinterpret_cast<const uint4*>(stage[warp]);
  const uint4 v0 = st4[lane];
  const uint4 v1 = lane < 16 ? st4[32 + lane] : make_uint4(0, 0, 0, 0);
  // the segment's live bytes: 24 per active lane (the last segment of a row may be short)
  const int live = (H - s * 512 < 512 ? H - s * 512 : 512) / 16 * 24;
  const size_t row_bytes = static_cast<size_t>(H) / 2 * 3;
  for (int j = 0; j < k; ++j) {
    const int slot = __shfl_sync(kFullMask, my_slot, j);
    if (slot == -1) continue;
    if (slot < -1 || slot >= S) {
      if (lane == 0 && u == 0) report_bad_index(d_status);
      continue;
    }
    uint8_t* dst = recv_x + static_cast<size_t>(slot) * row_bytes + static_cast<size_t>(s) * 768;
    if (16 * lane < live) st_stream_v4(dst + 16 * lane, v0);
    if (lane < 16 && 512 + 16 * lane < live) st_stream_v4(dst + 512 + 16 * lane, v1);
  }
  }  // segments of the warp
}

// BF16: lane owns 8 channels (one 16-byte vector), a warp covers 256 channels.
__global__ void __launch_bounds__(kWarps * 32)
    dispatch_bf16_kernel(const uint16_t* __restrict__ x, int N, int H, int k,
                         const int32_t* __restrict__ token_slot, long long S,
                         uint16_t* __restrict__ recv_x, int32_t* d_status) {
  const int lane = threadIdx.x & 31;
  const int segs = (H + 255) / 256;
  const long long item = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(N) * segs) return;
  const int t = static_cast<int>(item / segs);
  const int s = static_cast<int>(item - static_cast<long long>(t) * segs);
  const int c0 = s * 256 + lane * 8;
  const bool active = c0 < H;  // H % 8 == 0
  pdl_wait();
  pdl_trigger();
  const int my_slot = lane < k ? token_slot[static_cast<size_t>(t) * k + lane] : -1;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (active) v = ld_stream(x + static_cast<size_t>(t) * H + c0);
  for (int j = 0; j < k; ++j) {
    const int slot = __shfl_sync(kFullMask, my_slot, j);
    if (slot == -1) continue;
    if (slot < -1 || slot >= S) {
      if (lane == 0) report_bad_index(d_status);
      continue;
    }
    if (active) st_stream_v4(recv_x + static_cast<size_t>(slot) * H + c0, v);
  }
}

__global__ void e4m3_encode_kernel(const float* __restrict__ in, size_t n,
                                   uint8_t* __restrict__ out) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; 2 * i < n;
       i += stride) {
    const float lo = in[2 * i];
    const float hi = 2 * i + 1 < n ? in[2 * i + 1] : 0.0f;
    const uint32_t v = e4m3x2(lo, hi);
    out[2 * i] = static_cast<uint8_t>(v & 0xff);
    if (2 * i + 1 < n) out[2 * i + 1] = static_cast<uint8_t>(v >> 8);
  }
}

// The CTA-per-token kernels keep the token's row in shared memory; many CTAs
// per SM need the shared-memory side of the L1/shared split at its largest.
template <typename K>
cudaError_t prefer_shared(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared);
}

// Segments per warp: reading x is most of the traffic when k is small, and
// load latency then sets the pace, so each warp issues the loads of several
// neighbouring 512-channel segments before working on the first.
int segments_per_warp(int k) { return k <= 2 ? 4 : k <= 4 ? 2 : 1; }

template <int SL, bool UE8M0>
cudaError_t launch_fp8(int spw, const uint16_t* x, int N, int H, int k, const int32_t* token_slot,
                       long long num_rows, uint8_t* recv_x, float* recv_scale, long long ld,
                       int32_t* d_status, cudaStream_t stream) {
  const int segs = (H + 511) / 512;
  const long long items = static_cast<long long>(N) * ((segs + spw - 1) / spw);
  const unsigned blocks = static_cast<unsigned>((items + kWarps - 1) / kWarps);
  if (spw == 4)
    return launch_pdl(dispatch_fp8_kernel<SL, UE8M0, 4>, blocks, kWarps * 32, 0, stream, x, N, H, k,
                      token_slot, num_rows, recv_x, recv_scale, ld, d_status);
  if (spw == 2)
    return launch_pdl(dispatch_fp8_kernel<SL, UE8M0, 2>, blocks, kWarps * 32, 0, stream, x, N, H, k,
                      token_slot, num_rows, recv_x, recv_scale, ld, d_status);
  return launch_pdl(dispatch_fp8_kernel<SL, UE8M0, 1>, blocks, kWarps * 32, 0, stream, x, N, H, k,
                    token_slot, num_rows, recv_x, recv_scale, ld, d_status);
}

template <int SL>
cudaError_t launch_mx(int spw, const uint16_t* x, int N, int H, int k, const int32_t* token_slot,
                      long long num_rows, uint8_t* recv_x, uint8_t* recv_e8m0, long long ld,
                      int32_t* d_status, cudaStream_t stream) {
  const int segs = (H + 511) / 512;
  const long long items = static_cast<long long>(N) * ((segs + spw - 1) / spw);
  const unsigned blocks = static_cast<unsigned>((items + kWarps - 1) / kWarps);
  if (spw == 4)
    return launch_pdl(dispatch_mxfp8_kernel<SL, 4>, blocks, kWarps * 32, 0, stream, x, N, H, k, token_slot,
                      num_rows, recv_x, recv_e8m0, ld, d_status);
  if (spw == 2)
    return launch_pdl(dispatch_mxfp8_kernel<SL, 2>, blocks, kWarps * 32, 0, stream, x, N, H, k, token_slot,
                      num_rows, recv_x, recv_e8m0, ld, d_status);
  return launch_pdl(dispatch_mxfp8_kernel<SL, 1>, blocks, kWarps * 32, 0, stream, x, N, H, k, token_slot,
                    num_rows, recv_x, recv_e8m0, ld, d_status);
}

}  // namespace

long long scale_ld(long long num_rows, int dtype) {
  const long long per16 = (dtype == MOE_DTYPE_MXFP8_E4M3 || dtype == MOE_DTYPE_NVFP4 ||
                           dtype == MOE_DTYPE_FP8_E4M3_UE8M0)
                              ? 16
                              : 4;  // scales per 16 bytes
  return (num_rows + per16 - 1) / per16 * per16;
}

cudaError_t launch_dispatch(const void* x, int N, int H, int k, const int32_t* token_slot,
                            long long num_rows, int dtype, int scale_layout, void* recv_x,
                            void* recv_scale, int32_t* d_status, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* r8 = static_cast<uint8_t*>(recv_x);
  const long long ld = scale_ld(num_rows, dtype);
  if (dtype == MOE_DTYPE_FP8_E4M3 || dtype == MOE_DTYPE_MXFP8_E4M3 || dtype == MOE_DTYPE_FP8_E4M3_UE8M0) {
    float* f32 = static_cast<float*>(recv_scale);
    uint8_t* e8 = static_cast<uint8_t*>(recv_scale);
    const int two = segments_per_warp(k);
    if (dtype == MOE_DTYPE_FP8_E4M3_UE8M0) {
      if (scale_layout == MOE_SCALE_MN_MAJOR)
        return launch_fp8<MOE_SCALE_MN_MAJOR, true>(two, xs, N, H, k, token_slot, num_rows, r8, f32, ld,
                                                    d_status, stream);
      if (scale_layout == MOE_SCALE_MN_MAJOR_PACK4)
        return launch_fp8<MOE_SCALE_MN_MAJOR_PACK4, true>(two, xs, N, H, k, token_slot, num_rows, r8, f32,
                                                          (num_rows + 3) / 4 * 4, d_status, stream);
      return launch_fp8<MOE_SCALE_ROW_MAJOR, true>(two, xs, N, H, k, token_slot, num_rows, r8, f32, ld,
                                                   d_status, stream);
    }
    if (dtype == MOE_DTYPE_FP8_E4M3) {
      if (scale_layout == MOE_SCALE_MN_MAJOR)
        return launch_fp8<MOE_SCALE_MN_MAJOR, false>(two, xs, N, H, k, token_slot, num_rows, r8, f32, ld,
                                                     d_status, stream);
      return launch_fp8<MOE_SCALE_ROW_MAJOR, false>(two, xs, N, H, k, token_slot, num_rows, r8, f32, ld,
                                                    d_status, stream);
    }
    if (scale_layout == MOE_SCALE_MN_MAJOR)
      return launch_mx<MOE_SCALE_MN_MAJOR>(two, xs, N, H, k, token_slot, num_rows, r8, e8, ld, d_status,
                                           stream);
    if (scale_layout == MOE_SCALE_MMA_TILED)
      return launch_mx<MOE_SCALE_MMA_TILED>(two, xs, N, H, k, token_slot, num_rows, r8, e8, ld, d_status,
                                            stream);
    return launch_mx<MOE_SCALE_ROW_MAJOR>(two, xs, N, H, k, token_slot, num_rows, r8, e8, ld, d_status,
                                          stream);
  } else if (dtype == MOE_DTYPE_FP8_E4M3_TOKEN) {
    // vectors of 8 channels per thread; H <= 16384 -> at most 16
    const int vpt = (H / 8 + kTokenThreads - 1) / kTokenThreads;
    float* sc = static_cast<float*>(recv_scale);
    const size_t smem = 128 + static_cast<size_t>(H) * 2;
    cudaError_t err = vpt <= 2 ? prefer_shared(dispatch_fp8_token_kernel<2>)
                    : vpt <= 4 ? prefer_shared(dispatch_fp8_token_kernel<4>)
                    : vpt <= 8 ? prefer_shared(dispatch_fp8_token_kernel<8>)
                               : prefer_shared(dispatch_fp8_token_kernel<16>);
    if (err != cudaSuccess) return err;
    if (vpt <= 2)
      return launch_pdl(dispatch_fp8_token_kernel<2>, N, kTokenThreads, smem, stream, xs, N, H, k,
                        token_slot, num_rows, r8, sc, d_status);
    if (vpt <= 4)
      return launch_pdl(dispatch_fp8_token_kernel<4>, N, kTokenThreads, smem, stream, xs, N, H, k,
                        token_slot, num_rows, r8, sc, d_status);
    if (vpt <= 8)
      return launch_pdl(dispatch_fp8_token_kernel<8>, N, kTokenThreads, smem, stream, xs, N, H, k,
                        token_slot, num_rows, r8, sc, d_status);
    return launch_pdl(dispatch_fp8_token_kernel<16>, N, kTokenThreads, smem, stream, xs, N, H, k,
                      token_slot, num_rows, r8, sc, d_status);
  } else if (dtype == MOE_DTYPE_E5M6) {
    const int segs = (H + 511) / 512;
    const int spw = segments_per_warp(k);  // as the FP8 kernels
    const long long items = static_cast<long long>(N) * ((segs + spw - 1) / spw);
    const unsigned blocks = static_cast<unsigned>((items + kWarps - 1) / kWarps);
    if (spw == 4)
      return launch_pdl(dispatch_e5m6_kernel<4>, blocks, kWarps * 32, 0, stream, xs, N, H, k, token_slot,
                        num_rows, r8, d_status);
    if (spw == 2)
      return launch_pdl(dispatch_e5m6_kernel<2>, blocks, kWarps * 32, 0, stream, xs, N, H, k, token_slot,
                        num_rows, r8, d_status);
    return launch_pdl(dispatch_e5m6_kernel<1>, blocks, kWarps * 32, 0, stream, xs, N, H, k, token_slot,
                      num_rows, r8, d_status);
  } else {
    const long long items = static_cast<long long>(N) * ((H + 255) / 256);
    const unsigned blocks = static_cast<unsigned>((items + kWarps - 1) / kWarps);
    return launch_pdl(dispatch_bf16_kernel, blocks, kWarps * 32, 0, stream,
                      static_cast<const uint16_t*>(x), N, H, k, token_slot, num_rows,
                      static_cast<uint16_t*>(recv_x), d_status);
  }
}

template <int BPT, int SL, int THREADS>
cudaError_t launch_nvfp4_bpt(const uint16_t* x, int N, int H, int k, const int32_t* token_slot,
                             long long num_rows, uint8_t* recv_x, uint8_t* block_scale,
                             float* row_scale, long long ld, int32_t* d_status, cudaStream_t stream) {
  const size_t smem = 128 + static_cast<size_t>(H) * 2;  // H <= 16384: at most 32 KB + 128
  cudaError_t err = prefer_shared(dispatch_nvfp4_kernel<BPT, SL, THREADS>);
  if (err != cudaSuccess) return err;
  return launch_pdl(dispatch_nvfp4_kernel<BPT, SL, THREADS>, N, THREADS, smem, stream, x, N, H, k,
                    token_slot, num_rows, recv_x, block_scale, row_scale, ld, d_status);
}

template <int SL>
cudaError_t launch_nvfp4(const uint16_t* x, int N, int H, int k, const int32_t* token_slot,
                         long long num_rows, uint8_t* recv_x, uint8_t* block_scale,
                         float* row_scale, long long ld, int32_t* d_status, cudaStream_t stream) {
  // rows of up to 4096 channels: 64-thread CTAs, so twice as many tokens'
  // rows are in flight per SM (a short row is little work for a CTA)
  if (H <= 4096) {
    const int bpt = (H / 16 + kNvThreadsShort - 1) / kNvThreadsShort;  // <= 4
    if (bpt <= 1)
      return launch_nvfp4_bpt<1, SL, kNvThreadsShort>(x, N, H, k, token_slot, num_rows, recv_x, block_scale,
                                                      row_scale, ld, d_status, stream);
    if (bpt <= 2)
      return launch_nvfp4_bpt<2, SL, kNvThreadsShort>(x, N, H, k, token_slot, num_rows, recv_x, block_scale,
                                                      row_scale, ld, d_status, stream);
    return launch_nvfp4_bpt<4, SL, kNvThreadsShort>(x, N, H, k, token_slot, num_rows, recv_x, block_scale,
                                                    row_scale, ld, d_status, stream);
  }
  const int bpt = (H / 16 + kNvThreads - 1) / kNvThreads;  // blocks per thread, <= 8
  if (bpt <= 4)
    return launch_nvfp4_bpt<4, SL, kNvThreads>(x, N, H, k, token_slot, num_rows, recv_x, block_scale,
                                               row_scale, ld, d_status, stream);
  return launch_nvfp4_bpt<8, SL, kNvThreads>(x, N, H, k, token_slot, num_rows, recv_x, block_scale,
                                             row_scale, ld, d_status, stream);
}

cudaError_t launch_dispatch_nvfp4(const void* x, int N, int H, int k, const int32_t* token_slot,
                                  long long num_rows, int scale_layout, void* recv_x,
                                  void* block_scale, float* row_scale, int32_t* d_status,
                                  cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  uint8_t* r8 = static_cast<uint8_t*>(recv_x);
  uint8_t* bs = static_cast<uint8_t*>(block_scale);
  const long long ld = scale_ld(num_rows, MOE_DTYPE_NVFP4);
  if (scale_layout == MOE_SCALE_MN_MAJOR)
    return launch_nvfp4<MOE_SCALE_MN_MAJOR>(xs, N, H, k, token_slot, num_rows, r8, bs, row_scale,
                                            ld, d_status, stream);
  if (scale_layout == MOE_SCALE_MMA_TILED)
    return launch_nvfp4<MOE_SCALE_MMA_TILED>(xs, N, H, k, token_slot, num_rows, r8, bs, row_scale,
                                             ld, d_status, stream);
  return launch_nvfp4<MOE_SCALE_ROW_MAJOR>(xs, N, H, k, token_slot, num_rows, r8, bs, row_scale,
                                           ld, d_status, stream);
}

cudaError_t launch_e4m3_encode(const float* in, size_t n, uint8_t* out, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const size_t pairs = (n + 1) / 2;
  size_t blocks = (pairs + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  e4m3_encode_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(in, n, out);
  return cudaGetLastError();
}

}  // namespace moe
