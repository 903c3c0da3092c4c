// gate.cu -- router top-k selection and weights, one warp per token.
//
// [pplx] "Efficient and portable mixture-of-experts communication",
// Introduction: the router's logits become a probability distribution, the
// top-K experts are chosen and weighted by it.  DeepSeek Tile-Kernels news,
// "Funktionen der DeepSeek-Tile-Kernel": top-k selection, scoring, weight
// normalisation.  "DeepSeek, DeepEP 오픈소스 공개", Topic Body and 일반 커널:
// DeepSeek-V3 group-limited gating, top-4 groups / top-8 experts.
//
// Selection keys.  A candidate (value v, expert e) is packed into 64 bits as
// (order-preserving bits of v) << 32 | (0xffffffff - e), so a larger key means
// a larger value and, on equal values, a lower index -- the tie rule.  -0.0 is
// turned into +0.0 first so that the two compare equal.  The warp's largest
// key comes from two redux.sync max operations (high word, then low word among
// the lanes that hold the high maximum); k rounds give the slots in order.
// The lanes kernel sorts each lane's keys once, so a round is O(1) per lane
// (offer the head, pop it if it won); the generic kernel scans its keys for
// the largest one below the previous winner.
//
// Two kernels:
//  * lanes kernel (E = 32*V): lane l holds experts [l*V, (l+1)*V) -- one
//    vector load per lane.  For group-limited gating whose groups cover whole
//    lanes (E/G a multiple of V), a group is LPG = E/(G*V) neighbouring lanes:
//    each lane takes the top-n of its own values and LPG-lane xor-shuffle
//    merges give every lane its group's top-n, summed largest first.
//  * generic kernel (any E <= 1024): lane l holds experts l, l+32, ...; group
//    scores come from a per-warp shared-memory scan.
#include "layout_impl.cuh"
#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

constexpr int kGateWarps = 8;
constexpr int kSmallRouteTokens = 8;  // tokens gated per CTA on the one-launch routing path
constexpr int kMaxTopn = 4;

// Order-preserving map of a float onto uint32 (larger float -> larger code).
__device__ __forceinline__ uint32_t ord32(float v) {
  const uint32_t b = __float_as_uint(__fadd_rn(v, 0.0f));  // -0 -> +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_ord32(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}
__device__ __forceinline__ uint64_t make_key(float v, int e) {
  return (static_cast<uint64_t>(ord32(v)) << 32) | (0xffffffffu - static_cast<uint32_t>(e));
}
__device__ __forceinline__ int key_index(uint64_t key) {
  return static_cast<int>(0xffffffffu - static_cast<uint32_t>(key));  // sentinel 0 -> -1
}
__device__ __forceinline__ float key_value(uint64_t key) {
  return from_ord32(static_cast<uint32_t>(key >> 32));
}

// Largest key of the warp (all lanes get it).  Key 0 means "no candidate".
__device__ __forceinline__ uint64_t warp_max_key(uint64_t key) {
  const uint32_t hi = __reduce_max_sync(kFullMask, static_cast<uint32_t>(key >> 32));
  const uint32_t lo =
      __reduce_max_sync(kFullMask, static_cast<uint32_t>(key >> 32) == hi ? static_cast<uint32_t>(key) : 0u);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_xor_key(uint64_t key, int m) {
  const uint32_t hi = __shfl_xor_sync(kFullMask, static_cast<uint32_t>(key >> 32), m);
  const uint32_t lo = __shfl_xor_sync(kFullMask, static_cast<uint32_t>(key), m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_key(uint64_t key, int src) {
  const uint32_t hi = __shfl_sync(kFullMask, static_cast<uint32_t>(key >> 32), src);
  const uint32_t lo = __shfl_sync(kFullMask, static_cast<uint32_t>(key), src);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// k selection rounds over the lane's keys (key 0 = not a candidate).  Lane j
// receives slot j; every lane gets the slot-order sum of the winners' values.
template <int V>
__device__ __forceinline__ void select_topk(const uint64_t (&key)[V], int k, int lane, int& sel_i,
                                            float& sel_v, float& sum) {
  uint64_t prev = ~0ull;
  for (int j = 0; j < k; ++j) {
    uint64_t best = 0;
#pragma unroll
    for (int v = 0; v < V; ++v)
      if (key[v] < prev && key[v] > best) best = key[v];
    const uint64_t win = warp_max_key(best);
    const float wv = key_value(win);
    sum = (j == 0) ? wv : __fadd_rn(sum, wv);
    if (lane == j) {
      sel_i = key_index(win);
      sel_v = wv;
    }
    prev = win;
  }
}

// Sorts a lane's keys, largest first, with a fixed comparator network
// (Knuth's 19-comparator network for 8 keys).
__device__ __forceinline__ void cswap_desc(uint64_t& a, uint64_t& b) {
  const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
  a = hi;
  b = lo;
}
template <int V>
__device__ __forceinline__ void sort_desc(uint64_t (&k)[V]) {
  if constexpr (V == 2) {
    cswap_desc(k[0], k[1]);
  } else if constexpr (V == 4) {
    cswap_desc(k[0], k[1]); cswap_desc(k[2], k[3]);
    cswap_desc(k[0], k[2]); cswap_desc(k[1], k[3]);
    cswap_desc(k[1], k[2]);
  } else if constexpr (V == 8) {
    cswap_desc(k[0], k[2]); cswap_desc(k[1], k[3]); cswap_desc(k[4], k[6]); cswap_desc(k[5], k[7]);
    cswap_desc(k[0], k[4]); cswap_desc(k[1], k[5]); cswap_desc(k[2], k[6]); cswap_desc(k[3], k[7]);
    cswap_desc(k[0], k[1]); cswap_desc(k[2], k[3]); cswap_desc(k[4], k[5]); cswap_desc(k[6], k[7]);
    cswap_desc(k[2], k[4]); cswap_desc(k[3], k[5]);
    cswap_desc(k[1], k[4]); cswap_desc(k[3], k[6]);
    cswap_desc(k[1], k[2]); cswap_desc(k[3], k[4]); cswap_desc(k[5], k[6]);
  }
}

// Selection over per-lane lists sorted largest first: a lane offers its head,
// the warp's largest head wins, and the winning lane pops it.  Lane j
// receives slot j; every lane gets the slot-order sum of the winners' values.
template <int V>
__device__ __forceinline__ void select_sorted(uint64_t (&key)[V], int k, int lane, int& sel_i,
                                              float& sel_v, float& sum) {
  for (int j = 0; j < k; ++j) {
    const uint64_t win = warp_max_key(key[0]);
    const float wv = key_value(win);
    sum = (j == 0) ? wv : __fadd_rn(sum, wv);
    if (lane == j) {
      sel_i = key_index(win);
      sel_v = wv;
    }
    const bool pop = win != 0 && key[0] == win;
#pragma unroll
    for (int v = 0; v + 1 < V; ++v) key[v] = pop ? key[v + 1] : key[v];
    key[V - 1] = pop ? 0 : key[V - 1];
  }
}

// Extras of the routing entry point: a buffer the caller reads next (x of
// the dispatch that follows), which the gate CTAs ask L2 to fetch while they
// run.  prefetch == NULL: none.
struct GateExtras {
  const char* prefetch;
  unsigned long long prefetch_bytes;
};

// ------------------------------------------------------------------ lanes kernel
template <int V, int TOPN>
__device__ __forceinline__ void gate_lanes_token(const float* __restrict__ logits, int t, int k,
                                                 int kind, int LPG_log2, int TG, float* sh_exp,
                                                 int lane, int32_t* __restrict__ topk_idx,
                                                 float* __restrict__ topk_w, const GateExtras& cc) {
  constexpr int E = 32 * V;
  constexpr int topn = TOPN;  // group score = sum of the TOPN best scores of a group
  const int e0 = lane * V;
  const float* row = logits + static_cast<size_t>(t) * E + e0;
  float l[V];
  if constexpr (V % 4 == 0) {
#pragma unroll
    for (int q = 0; q < V / 4; ++q) {
      const float4 f = reinterpret_cast<const float4*>(row)[q];
      l[4 * q] = f.x;
      l[4 * q + 1] = f.y;
      l[4 * q + 2] = f.z;
      l[4 * q + 3] = f.w;
    }
  } else if constexpr (V == 2) {
    const float2 f = *reinterpret_cast<const float2*>(row);
    l[0] = f.x;
    l[1] = f.y;
  } else {
    l[0] = row[0];
  }
  uint64_t key[V];
  int sel_i = -1;
  float sel_v = 0.0f, sum = 0.0f;

  if (kind == MOE_GATE_SIGMOID_GROUP) {
#pragma unroll
    for (int v = 0; v < V; ++v) key[v] = make_key(logistic(l[v]), e0 + v);
    sort_desc<V>(key);
    // this lane's top-n, best first (key 0 pads when n > V)
    uint64_t top[topn];
#pragma unroll
    for (int p = 0; p < topn; ++p) top[p] = p < V ? key[p < V ? p : 0] : 0;
    // merge with the other lanes of the group: top-n of two sorted lists is
    // max(a_i, b_{n-1-i}) (a bitonic sequence), then sorted again
#pragma unroll
    for (int step = 0; step < 5; ++step) {  // LPG <= 32 lanes: at most 5 merges
      if (step >= LPG_log2) break;            // warp-uniform
      const int m = 1 << step;
      uint64_t other[topn], mrg[topn];
#pragma unroll
      for (int p = 0; p < topn; ++p) other[p] = shfl_xor_key(top[p], m);
#pragma unroll
      for (int p = 0; p < topn; ++p) mrg[p] = top[p] > other[topn - 1 - p] ? top[p] : other[topn - 1 - p];
      // sort the merged keys, largest first
#pragma unroll
      for (int a = 0; a < topn; ++a)
#pragma unroll
        for (int b = topn - 1; b > a; --b)
          if (mrg[b] > mrg[b - 1]) {
            const uint64_t tmp = mrg[b];
            mrg[b] = mrg[b - 1];
            mrg[b - 1] = tmp;
          }
#pragma unroll
      for (int p = 0; p < topn; ++p) top[p] = mrg[p];
    }
    float gscore = key_value(top[0]);
#pragma unroll
    for (int p = 1; p < topn; ++p) gscore = __fadd_rn(gscore, key_value(top[p]));
    // rank of this lane's group among all groups (group h leads lanes h*LPG..)
    const int g = lane >> LPG_log2;
    const int G = 32 >> LPG_log2;
    const uint64_t gkey = make_key(gscore, g);
    int before = 0;
    for (int h = 0; h < G; ++h) before += shfl_key(gkey, h << LPG_log2) > gkey ? 1 : 0;
    if (before >= TG) {
#pragma unroll
      for (int v = 0; v < V; ++v) key[v] = 0;
    }
    select_sorted<V>(key, k, lane, sel_i, sel_v, sum);
    if (lane < k) sel_v = __fdiv_rn(sel_v, sum);
  } else {
    float m = l[0];
#pragma unroll
    for (int v = 1; v < V; ++v) m = fmaxf(m, l[v]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
#pragma unroll
    for (int v = 0; v < V; ++v) {
      sh_exp[e0 + v] = fixed_exp(__fsub_rn(l[v], m));
      key[v] = make_key(l[v], e0 + v);
    }
    __syncwarp();
    float z = 0.0f;
    if (lane == 0)
      for (int i = 0; i < E; ++i) z = __fadd_rn(z, sh_exp[i]);
    z = __shfl_sync(kFullMask, z, 0);
    sort_desc<V>(key);
    for (int j = 0; j < k; ++j) {
      const uint64_t win = warp_max_key(key[0]);
      const int wi = key_index(win);
      const float p = (wi >= 0 && wi < E) ? __fdiv_rn(sh_exp[wi], z) : 0.0f;
      sum = (j == 0) ? p : __fadd_rn(sum, p);
      if (lane == j) {
        sel_i = (wi >= 0 && wi < E) ? wi : -1;
        sel_v = p;
      }
      const bool pop = win != 0 && key[0] == win;
#pragma unroll
      for (int v = 0; v + 1 < V; ++v) key[v] = pop ? key[v + 1] : key[v];
      key[V - 1] = pop ? 0 : key[V - 1];
    }
    if (lane < k && kind == MOE_GATE_SOFTMAX_RENORM) sel_v = __fdiv_rn(sel_v, sum);
    __syncwarp();  // sh_exp is rewritten for the next token
  }
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = sel_i;
    topk_w[static_cast<size_t>(t) * k + lane] = sel_v;
  }
}

// Softmax needs Z summed in ascending expert order: the exp terms go to shared
// memory (one row per warp) and lane 0 adds them one by one.
template <int V, int TOPN>
__global__ void __launch_bounds__(kGateWarps * 32)
    topk_gate_lanes_kernel(const float* __restrict__ logits, int N, int k, int kind, int LPG_log2,
                           int TG, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                           GateExtras cc) {
  __shared__ float sh_exp[kGateWarps][32 * V];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  prefetch_share_l2(cc.prefetch, cc.prefetch_bytes);
  for (int t = blockIdx.x * kGateWarps + warp; t < N; t += gridDim.x * kGateWarps)
    gate_lanes_token<V, TOPN>(logits, t, k, kind, LPG_log2, TG, sh_exp[warp], lane, topk_idx, topk_w, cc);
}

// ------------------------------------------------------------------ fused routing, small batches
// Gate and layout in one launch when every entry fits one layout chunk
// (N*k <= kLayoutThreads): CTAs of kLayoutThreads threads of which the first
// kSmallRouteTokens warps gate one token each (as many tokens per SM as the
// gate kernel's CTAs take, so the gating spreads over as many SMs); all
// kLayoutWarps warps of the last CTA build the layout.
// Each CTA publishes its tokens' choices (fence, then an arrival on a counter
// in the caller's zeroed workspace); the CTA that arrives last -- every
// other CTA's outputs are visible to it by then -- builds the whole layout
// with the single-CTA layout body and puts the counter back to zero.  No CTA
// waits for another.
template <int V, int TOPN>
__global__ void __launch_bounds__(kLayoutThreads)
    route_small_kernel(const float* __restrict__ logits, int N, int k, int kind, int LPG_log2, int TG,
                       int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int R,
                       int32_t* __restrict__ expert_count, int32_t* __restrict__ expert_offset,
                       int32_t* __restrict__ rank_count, int32_t* __restrict__ rank_offset,
                       int32_t* __restrict__ rank_tokens, int32_t* __restrict__ token_slot,
                       int32_t* __restrict__ slot_token, int align, long long num_rows,
                       int32_t* d_status, unsigned* done, const char* prefetch,
                       unsigned long long prefetch_bytes) {
  extern __shared__ int32_t sm[];  // gate: one row of E floats per warp; then the layout's words
  __shared__ int last_cta;
  constexpr int E = 32 * V;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  prefetch_share_l2(prefetch, prefetch_bytes);
  const int t = blockIdx.x * kSmallRouteTokens + warp;
  const GateExtras none{nullptr, 0};
  if (warp < kSmallRouteTokens && t < N)
    gate_lanes_token<V, TOPN>(logits, t, k, kind, LPG_log2, TG, reinterpret_cast<float*>(sm) + warp * E,
                              lane, topk_idx, topk_w, none);
  __threadfence();  // this thread's outputs reach device scope before the CTA's arrival
  __syncthreads();
  if (threadIdx.x == 0) last_cta = atomicAdd(done, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  layout_single_body<false>(sm, topk_idx, N, k, E, R, expert_count, expert_offset, rank_count,
                            rank_offset, rank_tokens, token_slot, slot_token, align, num_rows, d_status);
  if (threadIdx.x == 0) *done = 0u;
}

// ------------------------------------------------------------------ generic kernel
// One token by one warp for any E <= 1024: lane l holds experts l, l + 32,
// ...; per-warp shared memory vals[E] (scores or exp terms), gscore[G],
// gkeep[G] (group kind) -- wsm points at this warp's E + 2G words.
template <int V>
__device__ __forceinline__ void gate_generic_token(const float* __restrict__ logits, int t, int E, int k,
                                                   int kind, int G, int TG, int topn, float* wsm, int lane,
                                                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  float* vals = wsm;
  float* gscore = vals + E;
  int* gkeep = reinterpret_cast<int*>(gscore + G);
  const int eg = E / G;
  const float* row = logits + static_cast<size_t>(t) * E;
  float l[V];
  uint64_t key[V];
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const int e = v * 32 + lane;
    l[v] = e < E ? row[e] : 0.0f;
  }
  int sel_i = -1;
  float sel_v = 0.0f, sum = 0.0f;

  if (kind == MOE_GATE_SIGMOID_GROUP) {
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int e = v * 32 + lane;
      if (e < E) {
        const float s = logistic(l[v]);
        vals[e] = s;
        key[v] = make_key(s, e);
      } else {
        key[v] = 0;
      }
    }
    __syncwarp();
    // group score: the topn best scores of the group, added best first
    for (int g = lane; g < G; g += 32) {
      const float* gv = vals + g * eg;
      uint64_t prev = ~0ull;
      float gs = 0.0f;
      for (int p = 0; p < topn; ++p) {
        uint64_t best = 0;
        for (int i = 0; i < eg; ++i) {
          const uint64_t kv = make_key(gv[i], i);
          if (kv < prev && kv > best) best = kv;
        }
        gs = (p == 0) ? key_value(best) : __fadd_rn(gs, key_value(best));
        prev = best;
      }
      gscore[g] = gs;
    }
    __syncwarp();
    // a group is kept when fewer than TG groups rank before it
    for (int g = lane; g < G; g += 32) {
      const uint64_t mine = make_key(gscore[g], g);
      int before = 0;
      for (int h = 0; h < G; ++h) before += make_key(gscore[h], h) > mine ? 1 : 0;
      gkeep[g] = before < TG;
    }
    __syncwarp();
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int e = v * 32 + lane;
      if (e < E && !gkeep[e / eg]) key[v] = 0;
    }
    select_topk<V>(key, k, lane, sel_i, sel_v, sum);
    if (lane < k) sel_v = __fdiv_rn(sel_v, sum);
  } else {
    float m = -INFINITY;
#pragma unroll
    for (int v = 0; v < V; ++v)
      if (v * 32 + lane < E) m = fmaxf(m, l[v]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int e = v * 32 + lane;
      if (e < E) {
        vals[e] = fixed_exp(__fsub_rn(l[v], m));
        key[v] = make_key(l[v], e);
      } else {
        key[v] = 0;
      }
    }
    __syncwarp();
    float z = 0.0f;
    if (lane == 0)
      for (int i = 0; i < E; ++i) z = __fadd_rn(z, vals[i]);
    z = __shfl_sync(kFullMask, z, 0);
    uint64_t prev = ~0ull;
    for (int j = 0; j < k; ++j) {
      uint64_t best = 0;
#pragma unroll
      for (int v = 0; v < V; ++v)
        if (key[v] < prev && key[v] > best) best = key[v];
      const uint64_t win = warp_max_key(best);
      const int wi = key_index(win);
      // only NaN logits can leave a round without a candidate
      const float p = (wi >= 0 && wi < E) ? __fdiv_rn(vals[wi], z) : 0.0f;
      sum = (j == 0) ? p : __fadd_rn(sum, p);
      if (lane == j) {
        sel_i = (wi >= 0 && wi < E) ? wi : -1;
        sel_v = p;
      }
      prev = win;
    }
    if (lane < k && kind == MOE_GATE_SOFTMAX_RENORM) sel_v = __fdiv_rn(sel_v, sum);
  }
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = sel_i;
    topk_w[static_cast<size_t>(t) * k + lane] = sel_v;
  }
  __syncwarp();  // the next token reuses this warp's shared memory
}

template <int V>
__global__ void __launch_bounds__(kGateWarps * 32)
    topk_gate_generic_kernel(const float* __restrict__ logits, int N, int E, int k, int kind,
                             int G, int TG, int topn, int32_t* __restrict__ topk_idx,
                             float* __restrict__ topk_w, GateExtras cc) {
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  prefetch_share_l2(cc.prefetch, cc.prefetch_bytes);
  for (int t = blockIdx.x * kGateWarps + warp; t < N; t += gridDim.x * kGateWarps)
    gate_generic_token<V>(logits, t, E, k, kind, G, TG, topn, smem + warp * (E + 2 * G), lane, topk_idx,
                          topk_w);
}

// One-launch routing for the expert counts the lanes kernel does not take:
// as route_small_kernel, with the generic gate (shared memory per warp).
template <int V>
__global__ void __launch_bounds__(kLayoutThreads)
    route_small_generic_kernel(const float* __restrict__ logits, int N, int E, int k, int kind, int G,
                               int TG, int topn, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                               int R, int32_t* __restrict__ expert_count, int32_t* __restrict__ expert_offset,
                               int32_t* __restrict__ rank_count, int32_t* __restrict__ rank_offset,
                               int32_t* __restrict__ rank_tokens, int32_t* __restrict__ token_slot,
                               int32_t* __restrict__ slot_token, int align, long long num_rows,
                               int32_t* d_status, unsigned* done, const char* prefetch,
                               unsigned long long prefetch_bytes) {
  extern __shared__ int32_t sm[];
  __shared__ int last_cta;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  prefetch_share_l2(prefetch, prefetch_bytes);
  const int t = blockIdx.x * kSmallRouteTokens + warp;
  if (warp < kSmallRouteTokens && t < N)
    gate_generic_token<V>(logits, t, E, k, kind, G, TG, topn, reinterpret_cast<float*>(sm) + warp * (E + 2 * G),
                          lane, topk_idx, topk_w);
  __threadfence();  // this thread's outputs reach device scope before the CTA's arrival
  __syncthreads();
  if (threadIdx.x == 0) last_cta = atomicAdd(done, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  layout_single_body<false>(sm, topk_idx, N, k, E, R, expert_count, expert_offset, rank_count,
                            rank_offset, rank_tokens, token_slot, slot_token, align, num_rows, d_status);
  if (threadIdx.x == 0) *done = 0u;
}

unsigned grid_for(int N) {
  int blocks = (N + kGateWarps - 1) / kGateWarps;
  if (blocks > 148 * 32) blocks = 148 * 32;
  return static_cast<unsigned>(blocks);
}

template <int V>
cudaError_t launch_generic(const float* logits, int N, int E, int k, int kind, int G, int TG,
                           int topn, int32_t* idx, float* w, const GateExtras& cc, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(kGateWarps) * (E + 2 * G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(topk_gate_generic_kernel<V>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  return launch_pdl(topk_gate_generic_kernel<V>, grid_for(N), kGateWarps * 32, smem, stream, logits,
                    N, E, k, kind, G, TG, topn, idx, w, cc);
}

template <int V, int TOPN>
cudaError_t launch_lanes_n(const float* logits, int N, int k, int kind, int lpg_log2, int TG,
                           int32_t* idx, float* w, const GateExtras& cc, cudaStream_t stream) {
  return launch_pdl(topk_gate_lanes_kernel<V, TOPN>, grid_for(N), kGateWarps * 32, 0, stream,
                    logits, N, k, kind, lpg_log2, TG, idx, w, cc);
}

template <int V>
cudaError_t launch_lanes(const float* logits, int N, int k, int kind, int lpg_log2, int TG,
                         int topn, int32_t* idx, float* w, const GateExtras& cc, cudaStream_t stream) {
  switch (topn) {
    case 1: return launch_lanes_n<V, 1>(logits, N, k, kind, lpg_log2, TG, idx, w, cc, stream);
    case 2: return launch_lanes_n<V, 2>(logits, N, k, kind, lpg_log2, TG, idx, w, cc, stream);
    case 3: return launch_lanes_n<V, 3>(logits, N, k, kind, lpg_log2, TG, idx, w, cc, stream);
    default: return launch_lanes_n<V, 4>(logits, N, k, kind, lpg_log2, TG, idx, w, cc, stream);
  }
}

int log2_exact(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return (1 << r) == x ? r : -1;
}

// The gate's exp and sigmoid on consecutive fp32 bit patterns: thread i
// takes patterns first + 4i .. first + 4i + 3 (mod 2^32) and stores them as
// one 16-byte vector per output (a shorter run at the end of the range).
__global__ void gate_math_kernel(uint32_t first, size_t n, float* __restrict__ exp_out,
                                 float* __restrict__ sig_out, float* __restrict__ silu_out) {
  const size_t quads = (n + 3) / 4;
  for (size_t q = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; q < quads;
       q += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t i0 = 4 * q;
    float e[4], s[4], g[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float x = __uint_as_float(first + static_cast<uint32_t>(i0 + u));
      e[u] = fixed_exp(x);
      s[u] = logistic(x);
      // the SwiGLU kernels' choice for a lone value
      g[u] = fabsf(x) <= 87.0f ? silu_in_range(x) : silu_exact(x);
    }
    if (i0 + 4 <= n) {
      if (exp_out) *reinterpret_cast<float4*>(exp_out + i0) = make_float4(e[0], e[1], e[2], e[3]);
      if (sig_out) *reinterpret_cast<float4*>(sig_out + i0) = make_float4(s[0], s[1], s[2], s[3]);
      if (silu_out) *reinterpret_cast<float4*>(silu_out + i0) = make_float4(g[0], g[1], g[2], g[3]);
    } else {
      for (int u = 0; u < 4 && i0 + u < n; ++u) {
        if (exp_out) exp_out[i0 + u] = e[u];
        if (sig_out) sig_out[i0 + u] = s[u];
        if (silu_out) silu_out[i0 + u] = g[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_gate_math(uint32_t first, size_t n, float* exp_out, float* sigmoid_out,
                             float* silu_out, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  size_t blocks = (n + 4 * 256 - 1) / (4 * 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  gate_math_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(first, n, exp_out, sigmoid_out,
                                                                      silu_out);
  return cudaGetLastError();
}

namespace {

// Which gate kernel a shape takes: the lanes kernel when E = 32*V with V a
// power of two up to 8, rows 16-byte aligned and (group kind) groups made of
// whole lanes with topn <= 4; lpg_log2 = log2(lanes per group).
struct GatePlan {
  bool lanes;
  int V, lpg_log2, G, TG, topn;
};

GatePlan plan_gate(const float* logits, int E, int kind, int n_groups, int topk_groups,
                   int group_topn) {
  GatePlan p{false, E / 32, 0, n_groups, topk_groups, group_topn};
  if (kind != MOE_GATE_SIGMOID_GROUP) p.G = p.TG = p.topn = 1;
  p.lanes = E % 32 == 0 && log2_exact(p.V) >= 0 && p.V <= 8 &&
            (reinterpret_cast<uintptr_t>(logits) & 15) == 0;
  if (p.lanes && kind == MOE_GATE_SIGMOID_GROUP) {
    const int eg = E / p.G;
    p.lpg_log2 = (eg % p.V == 0) ? log2_exact(eg / p.V) : -1;
    p.lanes = p.lpg_log2 >= 0 && p.topn <= kMaxTopn;
  }
  return p;
}

cudaError_t launch_gate(const float* logits, int N, int E, int k, int kind, const GatePlan& p,
                        int32_t* topk_idx, float* topk_w, const GateExtras& cc, cudaStream_t stream) {
  if (p.lanes) {
    switch (p.V) {
      case 1: return launch_lanes<1>(logits, N, k, kind, p.lpg_log2, p.TG, p.topn, topk_idx, topk_w, cc, stream);
      case 2: return launch_lanes<2>(logits, N, k, kind, p.lpg_log2, p.TG, p.topn, topk_idx, topk_w, cc, stream);
      case 4: return launch_lanes<4>(logits, N, k, kind, p.lpg_log2, p.TG, p.topn, topk_idx, topk_w, cc, stream);
      default: return launch_lanes<8>(logits, N, k, kind, p.lpg_log2, p.TG, p.topn, topk_idx, topk_w, cc, stream);
    }
  }
  const int per_lane = (E + 31) / 32;
  const int G = p.G, TG = p.TG, topn = p.topn;
  if (per_lane <= 1) return launch_generic<1>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, cc, stream);
  if (per_lane <= 2) return launch_generic<2>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, cc, stream);
  if (per_lane <= 4) return launch_generic<4>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, cc, stream);
  if (per_lane <= 8) return launch_generic<8>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, cc, stream);
  if (per_lane <= 16) return launch_generic<16>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, cc, stream);
  return launch_generic<32>(logits, N, E, k, kind, G, TG, topn, topk_idx, topk_w, cc, stream);
}

template <int V, int TOPN>
cudaError_t launch_route_small_n(const float* logits, int N, int k, int kind, int lpg_log2, int TG,
                                 int32_t* idx, float* w, int R, const RouteOut& o, unsigned* done,
                                 cudaStream_t stream) {
  const char* pf = static_cast<const char*>(o.prefetch);
  constexpr int E = 32 * V;
  size_t words = layout_single_smem_words(E, R);
  const size_t smem = (words > static_cast<size_t>(kLayoutWarps) * E ? words : static_cast<size_t>(kLayoutWarps) * E) *
                      sizeof(int32_t);
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(route_small_kernel<V, TOPN>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  const unsigned grid = static_cast<unsigned>((N + kSmallRouteTokens - 1) / kSmallRouteTokens);
  return launch_pdl(route_small_kernel<V, TOPN>, grid, kLayoutThreads, smem, stream, logits, N, k, kind,
                    lpg_log2, TG, idx, w, R, o.expert_count, o.expert_offset, o.rank_count, o.rank_offset,
                    o.rank_tokens, o.token_slot, o.slot_token, o.align, o.num_rows, o.d_status, done, pf,
                    static_cast<unsigned long long>(o.prefetch_bytes));
}

template <int V>
cudaError_t launch_route_small(const float* logits, int N, int k, int kind, const GatePlan& p, int32_t* idx,
                               float* w, int R, const RouteOut& o, unsigned* done, cudaStream_t stream) {
  switch (p.topn) {
    case 1: return launch_route_small_n<V, 1>(logits, N, k, kind, p.lpg_log2, p.TG, idx, w, R, o, done, stream);
    case 2: return launch_route_small_n<V, 2>(logits, N, k, kind, p.lpg_log2, p.TG, idx, w, R, o, done, stream);
    case 3: return launch_route_small_n<V, 3>(logits, N, k, kind, p.lpg_log2, p.TG, idx, w, R, o, done, stream);
    default: return launch_route_small_n<V, 4>(logits, N, k, kind, p.lpg_log2, p.TG, idx, w, R, o, done, stream);
  }
}

template <int V>
cudaError_t launch_route_small_generic_v(const float* logits, int N, int E, int k, int kind, const GatePlan& p,
                                         int32_t* idx, float* w, int R, const RouteOut& o, unsigned* done,
                                         cudaStream_t stream) {
  size_t words = layout_single_smem_words(E, R);
  const size_t gate_words = static_cast<size_t>(kSmallRouteTokens) * (E + 2 * p.G);
  if (gate_words > words) words = gate_words;
  const size_t smem = words * sizeof(int32_t);
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(route_small_generic_kernel<V>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  const unsigned grid = static_cast<unsigned>((N + kSmallRouteTokens - 1) / kSmallRouteTokens);
  return launch_pdl(route_small_generic_kernel<V>, grid, kLayoutThreads, smem, stream, logits, N, E, k, kind,
                    p.G, p.TG, p.topn, idx, w, R, o.expert_count, o.expert_offset, o.rank_count, o.rank_offset,
                    o.rank_tokens, o.token_slot, o.slot_token, o.align, o.num_rows, o.d_status, done,
                    static_cast<const char*>(o.prefetch), static_cast<unsigned long long>(o.prefetch_bytes));
}

cudaError_t launch_route_small_generic(const float* logits, int N, int E, int k, int kind, const GatePlan& p,
                                       int32_t* idx, float* w, int R, const RouteOut& o, unsigned* done,
                                       cudaStream_t stream) {
  const int per_lane = (E + 31) / 32;
  if (per_lane <= 1) return launch_route_small_generic_v<1>(logits, N, E, k, kind, p, idx, w, R, o, done, stream);
  if (per_lane <= 2) return launch_route_small_generic_v<2>(logits, N, E, k, kind, p, idx, w, R, o, done, stream);
  if (per_lane <= 4) return launch_route_small_generic_v<4>(logits, N, E, k, kind, p, idx, w, R, o, done, stream);
  if (per_lane <= 8) return launch_route_small_generic_v<8>(logits, N, E, k, kind, p, idx, w, R, o, done, stream);
  return launch_route_small_generic_v<16>(logits, N, E, k, kind, p, idx, w, R, o, done, stream);
}

}  // namespace

size_t route_workspace_bytes(int N, int k, int E, int R) {
  return kRouteCounterBytes + layout_workspace_bytes(N, k, E, R);
}

cudaError_t launch_route(const float* logits, int N, int E, int k, int kind, int n_groups,
                         int topk_groups, int group_topn, int R, int32_t* topk_idx, float* topk_w,
                         const RouteOut& o, void* workspace, cudaStream_t stream) {
  const GatePlan p = plan_gate(logits, E, kind, n_groups, topk_groups, group_topn);
  unsigned* done = static_cast<unsigned*>(workspace);
  int32_t* chunks = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kRouteCounterBytes);
  if (N == 0 || static_cast<long long>(N) * k <= kLayoutThreads) {
    if (N > 0 && p.lanes) {
      switch (p.V) {
        case 1: return launch_route_small<1>(logits, N, k, kind, p, topk_idx, topk_w, R, o, done, stream);
        case 2: return launch_route_small<2>(logits, N, k, kind, p, topk_idx, topk_w, R, o, done, stream);
        case 4: return launch_route_small<4>(logits, N, k, kind, p, topk_idx, topk_w, R, o, done, stream);
        default: return launch_route_small<8>(logits, N, k, kind, p, topk_idx, topk_w, R, o, done, stream);
      }
    }
    // other expert counts up to 512: the generic gate in the same one-launch
    // scheme (beyond 512 its 32 keys per lane do not fit the registers a
    // 1024-thread CTA leaves, so the gate and the one-CTA layout launch apart)
    if (N > 0 && E <= 512)
      return launch_route_small_generic(logits, N, E, k, kind, p, topk_idx, topk_w, R, o, done, stream);
    if (N > 0) {
      const GateExtras pf{static_cast<const char*>(o.prefetch), static_cast<unsigned long long>(o.prefetch_bytes)};
      cudaError_t err = launch_gate(logits, N, E, k, kind, p, topk_idx, topk_w, pf, stream);
      if (err != cudaSuccess) return err;
    }
    return launch_layout(topk_idx, N, k, E, R, o.align, o.num_rows, o.expert_count, o.expert_offset,
                         o.rank_count, o.rank_offset, o.rank_tokens, o.token_slot, o.slot_token, chunks,
                         o.d_status, stream);
  }
  // gate (asking L2 for the prefetch region meanwhile), then the count and
  // assignment launches of the layout: with programmatic dependent launch the
  // three overlap better than a gate that also counts (measured on the
  // 4096-token batch)
  const GateExtras pf{static_cast<const char*>(o.prefetch), static_cast<unsigned long long>(o.prefetch_bytes)};
  cudaError_t err = launch_gate(logits, N, E, k, kind, p, topk_idx, topk_w, pf, stream);
  if (err != cudaSuccess) return err;
  return launch_layout(topk_idx, N, k, E, R, o.align, o.num_rows, o.expert_count, o.expert_offset,
                       o.rank_count, o.rank_offset, o.rank_tokens, o.token_slot, o.slot_token, chunks,
                       o.d_status, stream);
}

cudaError_t launch_topk_gate(const float* logits, int N, int E, int k, int kind, int n_groups,
                             int topk_groups, int group_topn, int32_t* topk_idx, float* topk_w,
                             cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const GatePlan p = plan_gate(logits, E, kind, n_groups, topk_groups, group_topn);
  const GateExtras none{nullptr, 0};
  return launch_gate(logits, N, E, k, kind, p, topk_idx, topk_w, none, stream);
}

}  // namespace moe
