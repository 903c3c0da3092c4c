// layout_impl.cuh -- device pieces of the layout step shared by the layout
// kernels (layout.cu) and the fused routing kernels (route.cu).
//
// DeepEP V2 summary, "training / prefill / decoding usage patterns": the
// handle carries per-expert received-token counts for the grouped GEMM and
// the routing metadata combine needs.  [pplx] "Efficient and portable
// mixture-of-experts communication", Dispatch: one contiguous buffer per
// expert and the source token of every row; Sharding: experts split over EP
// ranks (here partitions of one buffer).
#pragma once

#include "moe_device.cuh"

namespace moe {
namespace {

constexpr int kLayoutThreads = 1024;
constexpr int kLayoutWarps = kLayoutThreads / 32;

__host__ __device__ __forceinline__ int tokens_per_chunk(int k) { return kLayoutThreads / k; }

__host__ __device__ __forceinline__ int num_chunks(int N, int k) {
  const int tc = tokens_per_chunk(k);
  const int c = (N + tc - 1) / tc;
  return c > 0 ? c : 1;
}

// bucket of an entry: its expert, E for masked (-1) and invalid ids
__device__ __forceinline__ int bucket_of(int e, int E) {
  return (static_cast<unsigned>(e) < static_cast<unsigned>(E)) ? e : E;
}

// True when none of the token's slots before slot j (ids at tok[0..j)) has an
// expert of the rank whose experts are [lo, lo + epr); ids outside [0, E)
// never match because that range lies inside it.  The loads are independent.
__device__ __forceinline__ bool first_on_rank(const int32_t* tok, int j, int lo, int epr) {
  bool first = true;
#pragma unroll 4
  for (int jj = 0; jj < j; ++jj)
    first = first && static_cast<unsigned>(tok[jj]) - static_cast<unsigned>(lo) >= static_cast<unsigned>(epr);
  return first;
}

// Exclusive scan of a[0..n) in shared memory, n <= 2 * kLayoutThreads.
__device__ void block_exclusive_scan(int32_t* a, int n, int32_t* warp_sums) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = 2 * tid, i1 = 2 * tid + 1;
  const int x0 = i0 < n ? a[i0] : 0;
  const int x1 = i1 < n ? a[i1] : 0;
  const int s = x0 + x1;
  int incl = s;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(kFullMask, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = warp_sums[lane];
    int wi = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFullMask, wi, off);
      if (lane >= off) wi += y;
    }
    warp_sums[lane] = wi - v;
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - s;
  if (i0 < n) a[i0] = excl;
  if (i1 < n) a[i1] = excl + x0;
  __syncthreads();
}

// Exclusive prefix over the warps of every bucket of the [kLayoutWarps][nb]
// count matrix, in place: one thread per bucket, its loads issued eight at a
// time (independent addresses) and summed in registers.  Returns the
// bucket's total.
__device__ __forceinline__ int warp_prefix_of_bucket(int32_t* wcnt, int nb, int bb) {
  int acc = 0;
#pragma unroll
  for (int w0 = 0; w0 < kLayoutWarps; w0 += 8) {
    int v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = wcnt[(w0 + i) * nb + bb];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      wcnt[(w0 + i) * nb + bb] = acc;
      acc += v[i];
    }
  }
  return acc;
}

// Turns the per-bucket totals in off[] into exclusive row offsets, each
// expert bucket rounded up to a multiple of `align` (1 = packed); cnt[] keeps
// the totals.
__device__ void aligned_offsets(int32_t* off, int32_t* cnt, int nb, int align,
                                int32_t* warp_sums) {
  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    const int v = off[i];
    cnt[i] = v;
    if (i < nb - 1 && align > 1) off[i] = (v + align - 1) / align * align;
  }
  __syncthreads();
  block_exclusive_scan(off, nb, warp_sums);
}

// Rows no entry lands in get slot_token = -1: the padding after each expert
// (align > 1 only) and every row after the masked tail.  CTA `cta` of `ncta`
// takes its share; inside it one warp per expert, lanes over the rows.
__device__ void fill_unused_rows(const int32_t* off, const int32_t* cnt, int E, int align,
                                 long long num_rows, int32_t* slot_token, int cta, int ncta,
                                 int32_t* d_status) {
  if (align > 1) {
    const int nw = blockDim.x >> 5, lane = threadIdx.x & 31;
    for (int e = cta * nw + (threadIdx.x >> 5); e < E; e += ncta * nw)
      for (int i = off[e] + cnt[e] + lane; i < off[e + 1]; i += 32)
        if (derived_row_ok(i, num_rows, d_status)) slot_token[i] = -1;
  }
  const long long tail0 = static_cast<long long>(off[E]) + cnt[E];
  for (long long i = tail0 + static_cast<long long>(cta) * blockDim.x + threadIdx.x; i < num_rows;
       i += static_cast<long long>(ncta) * blockDim.x)
    slot_token[i] = -1;
}


// Shared-memory words layout_single_body needs for E experts and R ranks.
__host__ __device__ __forceinline__ size_t layout_single_smem_words(int E, int R) {
  return 2 * (static_cast<size_t>(E) + 1) + static_cast<size_t>(kLayoutWarps) * (E + 1) + 32 + R +
         kLayoutThreads + E;
}

// The whole layout by one CTA of kLayoutThreads threads when every entry fits
// one chunk (N*k <= kLayoutThreads): histogram, scan and ranks stay in shared
// memory.  WAIT: the entries come from the previous kernel (PDL wait after the
// data-independent setup); otherwise they were written by other CTAs of this
// grid, made visible by the caller's fence, and are read from L2 (ld.global.cg).
template <bool WAIT>
__device__ __forceinline__ void layout_single_body(
    int32_t* sm, const int32_t* topk_idx, int N, int k, int E, int R, int32_t* expert_count,
    int32_t* expert_offset, int32_t* rank_count, int32_t* rank_offset, int32_t* rank_tokens,
    int32_t* token_slot, int32_t* slot_token, int align, long long num_rows, int32_t* d_status) {
  const int nb = E + 1;
  int32_t* off = sm;                              // nb: totals, then their exclusive scan
  int32_t* wcnt = off + nb;                       // kLayoutWarps * nb
  int32_t* warp_sums = wcnt + kLayoutWarps * nb;  // 32
  int32_t* rtok = warp_sums + 32;                 // R
  int32_t* sidx = rtok + R;                       // kLayoutThreads
  int32_t* cnt = sidx + kLayoutThreads;           // nb: totals
  int32_t* rank_of = cnt + nb;                    // E: rank of each expert
  const int tid = threadIdx.x, warp = tid >> 5;
  const int ne = N * k;  // <= kLayoutThreads
  const int nbits = 32 - __clz(E + 1);
  const int epr = E / R;
  // data-independent setup (overlaps the predecessor's tail under PDL)
  const int my_tok = tid / k, j = tid - my_tok * k;
  for (int i = tid; i < kLayoutWarps * nb; i += kLayoutThreads) wcnt[i] = 0;
  for (int i = tid; i < R; i += kLayoutThreads) rtok[i] = 0;
  for (int i = tid; i < E; i += kLayoutThreads) rank_of[i] = i / epr;
  if constexpr (WAIT) {
    pdl_wait();
    pdl_trigger();
  }
  int e = -1, b = -1;
  if (tid < ne) {
    e = WAIT ? topk_idx[tid] : __ldcg(topk_idx + tid);
    sidx[tid] = e;
    b = bucket_of(e, E);
    if (b == E && e != -1) report_bad_index(d_status);
  }
  __syncthreads();
  const unsigned same = warp_match(static_cast<unsigned>(b + 1), nbits);
  const int in_warp = __popc(same & lanemask_lt());
  if (b >= 0 && in_warp == 0) wcnt[warp * nb + b] = __popc(same);
  if (b >= 0 && b < E) {  // the token's first slot on this rank counts the token
    const int r = rank_of[e];
    if (first_on_rank(sidx + tid - j, j, r * epr, epr)) atomicAdd(&rtok[r], 1);
  }
  __syncthreads();
  // per bucket: exclusive prefix over the warps, total into off[]
  for (int bb = tid; bb < nb; bb += kLayoutThreads) off[bb] = warp_prefix_of_bucket(wcnt, nb, bb);
  __syncthreads();
  aligned_offsets(off, cnt, nb, align, warp_sums);
  for (int i = tid; i < E; i += kLayoutThreads) expert_count[i] = cnt[i];
  fill_unused_rows(off, cnt, E, align, num_rows, slot_token, 0, 1, d_status);
  for (int i = tid; i <= E; i += kLayoutThreads) expert_offset[i] = off[i];
  for (int r = tid; r < R; r += kLayoutThreads) {
    rank_offset[r] = off[r * epr];
    rank_count[r] = off[(r + 1) * epr] - off[r * epr];
    rank_tokens[r] = rtok[r];
  }
  if (tid == 0) rank_offset[R] = off[E];
  if (tid < ne) {
    const int slot = off[b] + wcnt[warp * nb + b] + in_warp;
    if (!derived_row_ok(slot, num_rows, d_status)) {
      token_slot[tid] = -1;
    } else if (b < E) {
      token_slot[tid] = slot;
      slot_token[slot] = my_tok;
    } else {
      token_slot[tid] = -1;
      slot_token[slot] = -1;
    }
  }
}

}  // namespace
}  // namespace moe
