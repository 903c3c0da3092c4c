// layout.cu -- per-expert / per-rank counts, offsets and token<->slot maps.
//
// DeepEP V2 summary, "training / prefill / decoding usage patterns": the
// handle carries per-expert received-token counts for the grouped GEMM and
// the routing metadata combine needs.  [pplx] "Efficient and portable
// mixture-of-experts communication", Dispatch: one contiguous buffer per
// expert and the source token of every row; Portable kernels: one warp per
// block counts the tokens bound for each destination; Sharding: experts split
// over EP ranks (here partitions of one buffer).
//
// Two launches, no atomics on the order and no spin waits.  Entries with the
// same bucket inside a warp are found with one ballot per bucket bit
// (warp_match), which on B200 costs far less than __match_any_sync:
//   count:  one CTA per chunk of whole tokens (<= 1024 entries); per-chunk
//           histogram over E+1 buckets (bucket E = masked/invalid entries,
//           which fill the tail rows) and per-chunk per-rank token counts.
//   assign: one CTA per chunk again; every CTA sums the histograms of the
//           chunks before it and of all chunks (column sums, from L2), scans
//           the totals into expert offsets, ranks its entries inside the
//           chunk (warp_match + popc, then a prefix over the 32
//           warps) and writes token_slot / slot_token.  CTA 0 writes the
//           counts and offsets.  The row of entry (t, j) in expert e is the
//           number of entries routed to e before it in (t, j) order, so the
//           result is deterministic.
#include "moe_device.cuh"
#include "moe_launch.h"

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

__global__ void __launch_bounds__(kLayoutThreads)
    layout_count_kernel(const int32_t* __restrict__ topk_idx, int N, int k, int E, int R,
                        int32_t* __restrict__ chunk_counts, int32_t* __restrict__ chunk_rtok,
                        int32_t* d_status) {
  extern __shared__ int32_t sm[];
  int32_t* hist = sm;           // E + 1
  int32_t* rtok = hist + E + 1;  // R
  int32_t* sidx = rtok + R;      // kLayoutThreads
  int32_t* rank_of = sidx + kLayoutThreads;  // E: rank of each expert
  const int tid = threadIdx.x, lane = tid & 31;
  const int c = blockIdx.x;
  const int tc = tokens_per_chunk(k);
  const long long t0 = static_cast<long long>(c) * tc;
  const int nt = static_cast<int>(min(static_cast<long long>(tc), N - t0));
  const int ne = nt > 0 ? nt * k : 0;
  const int nbits = 32 - __clz(E + 1);  // bucket + 1 lies in [0, E + 1]
  // data-independent setup (overlaps the predecessor's tail under PDL)
  const int epr = E / R;
  const int j = tid % k;  // slot of this entry inside its token
  for (int i = tid; i <= E; i += kLayoutThreads) hist[i] = 0;
  for (int i = tid; i < R; i += kLayoutThreads) rtok[i] = 0;
  for (int i = tid; i < E; i += kLayoutThreads) rank_of[i] = i / epr;
  pdl_wait();
  pdl_trigger();
  int e = -1;
  if (tid < ne) {
    e = topk_idx[t0 * k + tid];
    sidx[tid] = e;
  }
  __syncthreads();
  const int b = tid < ne ? bucket_of(e, E) : -1;
  if (tid < ne && b == E && e != -1) report_bad_index(d_status);
  // one shared-memory add per distinct bucket in the warp
  const unsigned same = warp_match(static_cast<unsigned>(b + 1), nbits);
  if (b >= 0 && (same & lanemask_lt()) == 0) atomicAdd(&hist[b], __popc(same));
  if (b >= 0 && b < E) {
    // the token's first slot landing on this rank counts the token once
    const int r = rank_of[e];
    if (first_on_rank(sidx + tid - j, j, r * epr, epr)) atomicAdd(&rtok[r], 1);
  }
  (void)lane;
  __syncthreads();
  for (int i = tid; i <= E; i += kLayoutThreads)
    chunk_counts[static_cast<size_t>(c) * (E + 1) + i] = hist[i];
  for (int i = tid; i < R; i += kLayoutThreads) chunk_rtok[static_cast<size_t>(c) * R + i] = rtok[i];
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

__global__ void __launch_bounds__(kLayoutThreads)
    layout_assign_kernel(const int32_t* __restrict__ topk_idx, int N, int k, int E, int R, int C,
                         const int32_t* __restrict__ chunk_counts,
                         const int32_t* __restrict__ chunk_rtok, int32_t* __restrict__ expert_count,
                         int32_t* __restrict__ expert_offset, int32_t* __restrict__ rank_count,
                         int32_t* __restrict__ rank_offset, int32_t* __restrict__ rank_tokens,
                         int32_t* __restrict__ token_slot, int32_t* __restrict__ slot_token,
                         int align, long long num_rows, int32_t* d_status) {
  extern __shared__ int32_t sm[];
  const int nb = E + 1;
  int32_t* off = sm;                 // nb: totals, then their exclusive (aligned) scan
  int32_t* base = off + nb;          // nb: first row of this chunk per bucket
  int32_t* wcnt = base + nb;         // kLayoutWarps * nb
  int32_t* warp_sums = wcnt + kLayoutWarps * nb;  // 32
  int32_t* rtok = warp_sums + 32;                 // R (CTA 0: tokens per rank)
  int32_t* cnt = rtok + R;                        // nb: totals
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x;
  const int nbits = 32 - __clz(E + 1);
  const int my_tok = tid / k;  // token of this entry inside the chunk
  pdl_wait();
  pdl_trigger();

  // this CTA's entries are loaded first so their latency overlaps the sums
  const int tc = tokens_per_chunk(k);
  const long long t0 = static_cast<long long>(c) * tc;
  const int nt = static_cast<int>(min(static_cast<long long>(tc), N - t0));
  const int ne = nt > 0 ? nt * k : 0;
  int e = -1, b = -1;
  if (tid < ne) {
    e = topk_idx[t0 * k + tid];
    b = bucket_of(e, E);
  }
  // 1. column sums over chunks: all chunks (totals) and chunks before c,
  //    without atomics.  P threads per bucket each add a contiguous range of
  //    chunks (independent L2 loads); their partials go to shared memory (the
  //    warp-count array, zeroed only after) and one thread per bucket folds
  //    them.
  for (int i = tid; i < R; i += kLayoutThreads) rtok[i] = 0;
  if (c == 0) {  // block-uniform: CTA 0 also sums the per-chunk tokens per rank
    __syncthreads();
    const int total_vals = C * R;
    for (int i = tid; i < total_vals; i += kLayoutThreads) {
      const int v = chunk_rtok[i];
      if (v != 0) atomicAdd(&rtok[i % R], v);
    }
  }
  {
    const int P = min(16, max(1, kLayoutThreads / nb));  // 2 * nb * P <= kLayoutWarps * nb
    const int Lc = (C + P - 1) / P;
    int32_t* ptot = wcnt;           // [nb][P] partial totals
    int32_t* ppre = wcnt + nb * P;  // [nb][P] partial sums of the chunks before c
    for (int item = tid; item < nb * P; item += kLayoutThreads) {
      const int bb = item / P, p = item - bb * P;
      const int ca = p * Lc, cb = min(C, ca + Lc);
      int tot = 0, pre = 0;
#pragma unroll 4
      for (int cc = ca; cc < cb; ++cc) {
        const int v = chunk_counts[static_cast<size_t>(cc) * nb + bb];
        tot += v;
        pre += cc < c ? v : 0;
      }
      ptot[item] = tot;
      ppre[item] = pre;
    }
    __syncthreads();
    for (int bb = tid; bb < nb; bb += kLayoutThreads) {
      int tot = 0, pre = 0;
      for (int p = 0; p < P; ++p) {
        tot += ptot[bb * P + p];
        pre += ppre[bb * P + p];
      }
      off[bb] = tot;
      base[bb] = pre;
    }
    __syncthreads();
    for (int i = tid; i < kLayoutWarps * nb; i += kLayoutThreads) wcnt[i] = 0;
  }
  __syncthreads();
  // 2. bucket offsets (experts aligned), unused rows marked
  aligned_offsets(off, cnt, nb, align, warp_sums);
  if (c == 0)
    for (int i = tid; i < E; i += kLayoutThreads) expert_count[i] = cnt[i];
  for (int i = tid; i < nb; i += kLayoutThreads) base[i] += off[i];
  fill_unused_rows(off, cnt, E, align, num_rows, slot_token, c, C, d_status);
  if (c == 0) {
    const int epr = E / R;
    for (int i = tid; i <= E; i += kLayoutThreads) expert_offset[i] = off[i];
    for (int r = tid; r < R; r += kLayoutThreads) {
      rank_offset[r] = off[r * epr];
      rank_count[r] = off[(r + 1) * epr] - off[r * epr];
      rank_tokens[r] = rtok[r];
    }
    if (tid == 0) rank_offset[R] = off[E];
  }
  // 3. ranks inside the chunk
  const unsigned same = warp_match(static_cast<unsigned>(b + 1), nbits);
  const int in_warp = __popc(same & lanemask_lt());
  if (b >= 0 && in_warp == 0) wcnt[warp * nb + b] = __popc(same);
  __syncthreads();
  // exclusive prefix over the 32 warps of every bucket
  for (int bb = tid; bb < nb; bb += kLayoutThreads) warp_prefix_of_bucket(wcnt, nb, bb);
  __syncthreads();
  if (tid < ne) {
    const int slot = base[b] + wcnt[warp * nb + b] + in_warp;
    const long long flat = t0 * k + tid;
    // counts and ranks come from the same entries, so slot < num_rows; the
    // check only guards against topk_idx changing between the two launches
    if (slot < 0 || static_cast<long long>(slot) >= num_rows) {
      token_slot[flat] = -1;
      report_bad_index(d_status);
    } else if (b < E) {
      token_slot[flat] = slot;
      slot_token[slot] = static_cast<int32_t>(t0 + my_tok);
    } else {
      token_slot[flat] = -1;
      slot_token[slot] = -1;
    }
  }
  (void)lane;
}

// Whole layout in one CTA when every entry fits one chunk (N*k <= 1024, the
// decode-sized batches): histogram, scan and ranks stay in shared memory, so
// there is one launch and no workspace round trip.
__global__ void __launch_bounds__(kLayoutThreads)
    layout_single_kernel(const int32_t* __restrict__ topk_idx, int N, int k, int E, int R,
                         int32_t* __restrict__ expert_count, int32_t* __restrict__ expert_offset,
                         int32_t* __restrict__ rank_count, int32_t* __restrict__ rank_offset,
                         int32_t* __restrict__ rank_tokens, int32_t* __restrict__ token_slot,
                         int32_t* __restrict__ slot_token, int align, long long num_rows,
                         int32_t* d_status) {
  extern __shared__ int32_t sm[];
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
  pdl_wait();
  pdl_trigger();
  int e = -1, b = -1;
  if (tid < ne) {
    e = topk_idx[tid];
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

size_t layout_workspace_bytes(int N, int k, int E, int R) {
  const size_t C = static_cast<size_t>(num_chunks(N, k));
  size_t bytes = C * static_cast<size_t>(E + 1 + R) * sizeof(int32_t);
  bytes = (bytes + 255) / 256 * 256;
  return bytes < 256 ? 256 : bytes;
}

cudaError_t launch_layout(const int32_t* topk_idx, int N, int k, int E, int R, int align,
                          long long num_rows, int32_t* expert_count, int32_t* expert_offset,
                          int32_t* rank_count, int32_t* rank_offset, int32_t* rank_tokens,
                          int32_t* token_slot, int32_t* slot_token, void* workspace,
                          int32_t* d_status, cudaStream_t stream) {
  const int C = num_chunks(N, k);
  cudaError_t err;
  if (static_cast<long long>(N) * k <= kLayoutThreads) {
    const size_t smem = (2 * (static_cast<size_t>(E) + 1) +
                         static_cast<size_t>(kLayoutWarps) * (E + 1) + 32 + R + kLayoutThreads + E) *
                        sizeof(int32_t);
    if (smem > 48 * 1024) {
      err = cudaFuncSetAttribute(layout_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
      if (err != cudaSuccess) return err;
    }
    return launch_pdl(layout_single_kernel, 1, kLayoutThreads, smem, stream, topk_idx, N, k, E, R,
                      expert_count, expert_offset, rank_count, rank_offset, rank_tokens, token_slot,
                      slot_token, align, num_rows, d_status);
  }
  int32_t* chunk_counts = static_cast<int32_t*>(workspace);
  int32_t* chunk_rtok = chunk_counts + static_cast<size_t>(C) * (E + 1);
  const size_t smem_count = (2 * static_cast<size_t>(E) + 1 + R + kLayoutThreads) * sizeof(int32_t);
  const size_t smem_assign =
      (3 * (static_cast<size_t>(E) + 1) + static_cast<size_t>(kLayoutWarps) * (E + 1) + 32 + R) *
      sizeof(int32_t);
  if (smem_count > 48 * 1024) {
    err = cudaFuncSetAttribute(layout_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_count));
    if (err != cudaSuccess) return err;
  }
  if (smem_assign > 48 * 1024) {
    err = cudaFuncSetAttribute(layout_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_assign));
    if (err != cudaSuccess) return err;
  }
  err = launch_pdl(layout_count_kernel, C, kLayoutThreads, smem_count, stream, topk_idx, N, k, E, R,
                   chunk_counts, chunk_rtok, d_status);
  if (err != cudaSuccess) return err;
  return launch_pdl(layout_assign_kernel, C, kLayoutThreads, smem_assign, stream, topk_idx, N, k, E,
                    R, C, chunk_counts, chunk_rtok, expert_count, expert_offset, rank_count,
                    rank_offset, rank_tokens, token_slot, slot_token, align, num_rows, d_status);
}

}  // namespace moe
