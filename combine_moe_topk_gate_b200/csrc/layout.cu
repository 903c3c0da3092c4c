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
#include "layout_impl.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

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
  layout_single_body<true>(sm, topk_idx, N, k, E, R, expert_count, expert_offset, rank_count,
                           rank_offset, rank_tokens, token_slot, slot_token, align, num_rows, d_status);
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
    const size_t smem = layout_single_smem_words(E, R) * sizeof(int32_t);
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
