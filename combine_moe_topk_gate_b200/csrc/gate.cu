// gate.cu -- router top-k selection and weights, one warp per token.
//
// [pplx] "Efficient and portable mixture-of-experts communication",
// Introduction: the router's logits become a probability distribution, the
// top-K experts are chosen and weighted by it.  DeepSeek Tile-Kernels news,
// "Funktionen der DeepSeek-Tile-Kernel": top-k selection, scoring, weight
// normalisation.  "DeepSeek, DeepEP 오픈소스 공개", Topic Body and 일반 커널:
// DeepSeek-V3 group-limited gating, top-4 groups / top-8 experts.
//
// Layout in registers: lane l holds experts l, l+32, l+64, ... (coalesced
// 128-byte row loads).  A selection round finds, per lane, the best candidate
// ranked strictly after the previous winner (value descending, lower index on
// ties) and a 5-step butterfly leaves the warp's winner in every lane, so
// k rounds produce the slots in order without "taken" flags.
#include <float.h>

#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kGateWarps = 4;
constexpr int kNone = 0x7fffffff;

// (va, ia) is ranked before (vb, ib): larger value first, lower index on ties.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void warp_best(float& bv, int& bi) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(kFullMask, bv, off);
    const int oi = __shfl_xor_sync(kFullMask, bi, off);
    if (oi != kNone && (bi == kNone || ranks_before(ov, oi, bv, bi))) {
      bv = ov;
      bi = oi;
    }
  }
}

// Per-warp shared memory: vals[E] (scores or exp terms), gscore[G], gkeep[G].
template <int V>
__global__ void __launch_bounds__(kGateWarps * 32)
    topk_gate_kernel(const float* __restrict__ logits, int N, int E, int k, int kind, int G,
                     int TG, int topn, int32_t* __restrict__ topk_idx,
                     float* __restrict__ topk_w) {
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  float* vals = smem + warp * (E + 2 * G);
  float* gscore = vals + E;
  int* gkeep = reinterpret_cast<int*>(gscore + G);
  const int eg = E / G;

  for (int t = blockIdx.x * kGateWarps + warp; t < N; t += gridDim.x * kGateWarps) {
    const float* row = logits + static_cast<size_t>(t) * E;
    float key[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int e = v * 32 + lane;
      key[v] = e < E ? row[e] : 0.0f;
    }
    int sel_i = -1;
    float sel_v = 0.0f;
    float sum_sel = 0.0f;

    if (kind == MOE_GATE_SIGMOID_GROUP) {
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int e = v * 32 + lane;
        if (e < E) {
          key[v] = logistic(key[v]);
          vals[e] = key[v];
        }
      }
      __syncwarp();
      // group score: the topn best scores of the group, added best first
      for (int g = lane; g < G; g += 32) {
        const float* gv = vals + g * eg;
        float pv = INFINITY, sum = 0.0f;
        int pi = -1;
        for (int p = 0; p < topn; ++p) {
          float bv = 0.0f;
          int bi = kNone;
          for (int i = 0; i < eg; ++i) {
            const float v = gv[i];
            if (ranks_before(pv, pi, v, i) && (bi == kNone || ranks_before(v, i, bv, bi))) {
              bv = v;
              bi = i;
            }
          }
          sum = (p == 0) ? bv : __fadd_rn(sum, bv);
          pv = bv;
          pi = bi;
        }
        gscore[g] = sum;
      }
      __syncwarp();
      // a group is kept when fewer than TG groups rank before it
      for (int g = lane; g < G; g += 32) {
        const float s = gscore[g];
        int before = 0;
        for (int h = 0; h < G; ++h) before += ranks_before(gscore[h], h, s, g) ? 1 : 0;
        gkeep[g] = before < TG;
      }
      __syncwarp();
      bool cand[V];
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int e = v * 32 + lane;
        cand[v] = e < E && gkeep[e / eg] != 0;
      }
      float pv = INFINITY;
      int pi = -1;
      for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int bi = kNone;
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const int e = v * 32 + lane;
          if (cand[v] && ranks_before(pv, pi, key[v], e) &&
              (bi == kNone || ranks_before(key[v], e, bv, bi))) {
            bv = key[v];
            bi = e;
          }
        }
        warp_best(bv, bi);
        sum_sel = (j == 0) ? bv : __fadd_rn(sum_sel, bv);
        if (lane == j) {
          sel_i = bi;
          sel_v = bv;
        }
        pv = bv;
        pi = bi;
      }
      if (lane < k) sel_v = __fdiv_rn(sel_v, sum_sel);
    } else {
      // softmax: m = max logit, e_i = exp(l_i - m), Z summed in expert order
      float m = -INFINITY;
#pragma unroll
      for (int v = 0; v < V; ++v)
        if (v * 32 + lane < E) m = fmaxf(m, key[v]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int e = v * 32 + lane;
        if (e < E) vals[e] = fixed_exp(__fsub_rn(key[v], m));
      }
      __syncwarp();
      float z = 0.0f;
      if (lane == 0)
        for (int i = 0; i < E; ++i) z = __fadd_rn(z, vals[i]);
      z = __shfl_sync(kFullMask, z, 0);
      float pv = INFINITY;
      int pi = -1;
      for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int bi = kNone;
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const int e = v * 32 + lane;
          if (e < E && ranks_before(pv, pi, key[v], e) &&
              (bi == kNone || ranks_before(key[v], e, bv, bi))) {
            bv = key[v];
            bi = e;
          }
        }
        warp_best(bv, bi);
        // only NaN logits can leave a round without a candidate
        const float p = bi == kNone ? 0.0f : __fdiv_rn(vals[bi], z);
        sum_sel = (j == 0) ? p : __fadd_rn(sum_sel, p);
        if (lane == j) {
          sel_i = bi;
          sel_v = p;
        }
        pv = bv;
        pi = bi;
      }
      if (lane < k && kind == MOE_GATE_SOFTMAX_RENORM) sel_v = __fdiv_rn(sel_v, sum_sel);
    }
    if (lane < k) {
      if (sel_i == kNone) sel_i = -1;
      topk_idx[static_cast<size_t>(t) * k + lane] = sel_i;
      topk_w[static_cast<size_t>(t) * k + lane] = sel_v;
    }
    __syncwarp();  // the next token reuses this warp's shared memory
  }
}

template <int V>
cudaError_t launch_v(const float* logits, int N, int E, int k, int kind, int G, int TG, int topn,
                     int32_t* idx, float* w, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(kGateWarps) * (E + 2 * G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(topk_gate_kernel<V>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  int blocks = (N + kGateWarps - 1) / kGateWarps;
  if (blocks > 148 * 64) blocks = 148 * 64;
  topk_gate_kernel<V><<<blocks, kGateWarps * 32, smem, stream>>>(logits, N, E, k, kind, G, TG,
                                                                  topn, idx, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk_gate(const float* logits, int N, int E, int k, int kind, int n_groups,
                             int topk_groups, int group_topn, int32_t* topk_idx, float* topk_w,
                             cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  int G = n_groups, TG = topk_groups, topn = group_topn;
  if (kind != MOE_GATE_SIGMOID_GROUP) G = TG = topn = 1;
  const int per_lane = (E + 31) / 32;
  if (per_lane <= 1) return launch_v<1>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, stream);
  if (per_lane <= 2) return launch_v<2>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, stream);
  if (per_lane <= 4) return launch_v<4>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, stream);
  if (per_lane <= 8) return launch_v<8>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, stream);
  if (per_lane <= 16) return launch_v<16>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, stream);
  return launch_v<32>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, stream);
}

}  // namespace moe
