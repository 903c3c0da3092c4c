// api.cu -- the extern "C" entry points of libmoe.so (declared in moe.h).
//
// Each call checks its arguments on the host before anything is enqueued,
// then hands over to the launcher of its kernels on the caller's stream.  No
// call allocates, frees, synchronises or keeps state.
#include <stdint.h>

#include "moe.h"
#include "moe_launch.h"

namespace {

constexpr long long kMaxRows = 0x7fffffffLL;  // int32 slot ids
constexpr size_t kMaxPrefetchBytes = size_t(64) << 20;  // moe_route's L2 prefetch: half the L2 at most

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

cudaStream_t as_stream(moe_stream_t s) { return static_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

int moe_abi_version(void) { return 8; }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported size or option";
    case MOE_ERR_CUDA: return "CUDA launch error";
    case MOE_ERR_BAD_INDEX: return "index out of range (skipped)";
    case MOE_ERR_TIMEOUT: return "device wait timed out (output incomplete)";
  }
  return "unknown status";
}

moe_status_t moe_topk_gate(const float* logits, int num_tokens, int num_experts, int k,
                           moe_gate_kind_t kind, int n_groups, int topk_groups, int group_topn,
                           int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  const int N = num_tokens, E = num_experts;
  if (N < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (kind == MOE_GATE_SIGMOID_GROUP) {
    if (n_groups < 1 || E % n_groups != 0) return MOE_ERR_INVALID_ARG;
    const int eg = E / n_groups;
    if (topk_groups < 1 || topk_groups > n_groups) return MOE_ERR_INVALID_ARG;
    if (group_topn < 1 || group_topn > eg) return MOE_ERR_INVALID_ARG;
    if (static_cast<long long>(topk_groups) * eg < k) return MOE_ERR_INVALID_ARG;
  } else if (kind != MOE_GATE_SOFTMAX && kind != MOE_GATE_SOFTMAX_RENORM) {
    return MOE_ERR_INVALID_ARG;
  }
  if (N == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_topk_gate(logits, N, E, k, kind, n_groups, topk_groups,
                                         group_topn, topk_idx, topk_w, as_stream(stream)));
}

size_t moe_layout_workspace_bytes(int num_tokens, int k, int num_experts, int num_ranks) {
  if (num_tokens < 0 || k < 1 || num_experts < 1 || num_ranks < 1) return 0;
  return moe::layout_workspace_bytes(num_tokens, k, num_experts, num_ranks);
}

size_t moe_aligned_recv_rows(int num_tokens, int k, int num_experts, int align) {
  if (num_tokens < 0 || k < 1 || num_experts < 1 || align < 1) return 0;
  return static_cast<size_t>(num_tokens) * k + static_cast<size_t>(num_experts) * (align - 1);
}

moe_status_t moe_get_layout_aligned(const int32_t* topk_idx, int num_tokens, int k,
                                    int num_experts, int num_ranks, int align,
                                    int num_recv_rows, int32_t* expert_count,
                                    int32_t* expert_offset, int32_t* rank_count,
                                    int32_t* rank_offset, int32_t* rank_tokens,
                                    int32_t* token_slot, int32_t* slot_token, void* workspace,
                                    size_t workspace_bytes, int32_t* d_status,
                                    moe_stream_t stream) {
  const int N = num_tokens, E = num_experts, R = num_ranks;
  if (N < 0 || k < 1 || E < 1 || R < 1 || E % R != 0) return MOE_ERR_INVALID_ARG;
  if (align < 1 || align > MOE_MAX_ALIGN) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  const long long need = static_cast<long long>(N) * k + static_cast<long long>(E) * (align - 1);
  if (need > kMaxRows) return MOE_ERR_UNSUPPORTED;
  if (num_recv_rows < need) return MOE_ERR_INVALID_ARG;
  if (!expert_count || !expert_offset || !rank_count || !rank_offset || !rank_tokens ||
      !workspace)
    return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!topk_idx || !token_slot)) return MOE_ERR_INVALID_ARG;
  if (num_recv_rows > 0 && !slot_token) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe::layout_workspace_bytes(N, k, E, R)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {topk_idx, expert_count, expert_offset, rank_count, rank_offset,
                        rank_tokens, token_slot, slot_token, d_status};
  for (const void* p : ptrs)
    if (!aligned(p, 4)) return MOE_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_layout(topk_idx, N, k, E, R, align, num_recv_rows, expert_count,
                                      expert_offset, rank_count, rank_offset, rank_tokens,
                                      token_slot, slot_token, workspace, d_status,
                                      as_stream(stream)));
}

moe_status_t moe_get_layout(const int32_t* topk_idx, int num_tokens, int k, int num_experts,
                            int num_ranks, int32_t* expert_count, int32_t* expert_offset,
                            int32_t* rank_count, int32_t* rank_offset, int32_t* rank_tokens,
                            int32_t* token_slot, int32_t* slot_token, void* workspace,
                            size_t workspace_bytes, int32_t* d_status, moe_stream_t stream) {
  if (num_tokens < 0 || k < 1) return MOE_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(num_tokens) * k;
  if (rows > kMaxRows) return MOE_ERR_UNSUPPORTED;
  return moe_get_layout_aligned(topk_idx, num_tokens, k, num_experts, num_ranks, 1,
                                static_cast<int>(rows), expert_count, expert_offset, rank_count,
                                rank_offset, rank_tokens, token_slot, slot_token, workspace,
                                workspace_bytes, d_status, stream);
}

size_t moe_route_workspace_bytes(int num_tokens, int k, int num_experts, int num_ranks) {
  if (num_tokens < 0 || k < 1 || num_experts < 1 || num_ranks < 1) return 0;
  return moe::route_workspace_bytes(num_tokens, k, num_experts, num_ranks);
}

moe_status_t moe_route(const float* logits, int num_tokens, int num_experts, int k,
                       moe_gate_kind_t kind, int n_groups, int topk_groups, int group_topn,
                       int num_ranks, int align, int num_recv_rows, int32_t* topk_idx,
                       float* topk_w, int32_t* expert_count, int32_t* expert_offset,
                       int32_t* rank_count, int32_t* rank_offset, int32_t* rank_tokens,
                       int32_t* token_slot, int32_t* slot_token, void* workspace,
                       size_t workspace_bytes, const void* prefetch, size_t prefetch_bytes,
                       int32_t* d_status, moe_stream_t stream) {
  const int N = num_tokens, E = num_experts, R = num_ranks;
  // the gate's checks
  if (N < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (kind == MOE_GATE_SIGMOID_GROUP) {
    if (n_groups < 1 || E % n_groups != 0) return MOE_ERR_INVALID_ARG;
    const int eg = E / n_groups;
    if (topk_groups < 1 || topk_groups > n_groups) return MOE_ERR_INVALID_ARG;
    if (group_topn < 1 || group_topn > eg) return MOE_ERR_INVALID_ARG;
    if (static_cast<long long>(topk_groups) * eg < k) return MOE_ERR_INVALID_ARG;
  } else if (kind != MOE_GATE_SOFTMAX && kind != MOE_GATE_SOFTMAX_RENORM) {
    return MOE_ERR_INVALID_ARG;
  }
  // the layout's checks
  if (R < 1 || E % R != 0) return MOE_ERR_INVALID_ARG;
  if (align < 1 || align > MOE_MAX_ALIGN) return MOE_ERR_INVALID_ARG;
  const long long need = static_cast<long long>(N) * k + static_cast<long long>(E) * (align - 1);
  if (need > kMaxRows) return MOE_ERR_UNSUPPORTED;
  if (num_recv_rows < need) return MOE_ERR_INVALID_ARG;
  if (!expert_count || !expert_offset || !rank_count || !rank_offset || !rank_tokens || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!logits || !topk_idx || !topk_w || !token_slot)) return MOE_ERR_INVALID_ARG;
  if (num_recv_rows > 0 && !slot_token) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe::route_workspace_bytes(N, k, E, R)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, topk_idx, topk_w, expert_count, expert_offset, rank_count,
                        rank_offset, rank_tokens, token_slot, slot_token, d_status};
  for (const void* p : ptrs)
    if (!aligned(p, 4)) return MOE_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return MOE_ERR_INVALID_ARG;
  if (prefetch_bytes > 0 && (!prefetch || !aligned(prefetch, 16))) return MOE_ERR_INVALID_ARG;
  const size_t pf_bytes = prefetch_bytes < kMaxPrefetchBytes ? prefetch_bytes : kMaxPrefetchBytes;
  const moe::RouteOut out{expert_count, expert_offset, rank_count, rank_offset,
                          rank_tokens,  token_slot,    slot_token, align,
                          num_recv_rows, d_status,     pf_bytes ? prefetch : nullptr, pf_bytes};
  return from_cuda(moe::launch_route(logits, N, E, k, kind, n_groups, topk_groups, group_topn, R,
                                     topk_idx, topk_w, out, workspace, as_stream(stream)));
}

size_t moe_recv_bytes(int num_tokens, int hidden, int k, moe_dtype_t dtype) {
  if (num_tokens < 0 || hidden < 1 || k < 1) return 0;
  const size_t esz = dtype == MOE_DTYPE_BF16 ? 2 : 1;
  if (dtype == MOE_DTYPE_NVFP4) return static_cast<size_t>(num_tokens) * k * (hidden / 2);
  if (dtype == MOE_DTYPE_E5M6) return static_cast<size_t>(num_tokens) * k * (hidden / 2 * 3);
  return static_cast<size_t>(num_tokens) * k * hidden * esz;
}

size_t moe_scale_bytes(int num_tokens, int hidden, int k, moe_dtype_t dtype) {
  if (num_tokens < 0 || hidden < 1 || k < 1) return 0;
  const size_t rows = static_cast<size_t>(num_tokens) * k;
  switch (dtype) {
    case MOE_DTYPE_FP8_E4M3: return rows * (hidden / MOE_FP8_BLOCK) * sizeof(float);
    case MOE_DTYPE_FP8_E4M3_TOKEN: return rows * sizeof(float);
    case MOE_DTYPE_MXFP8_E4M3: return rows * (hidden / 32);
    case MOE_DTYPE_NVFP4: return rows * (hidden / 16);  /* block scales; + 4 bytes per row */
    case MOE_DTYPE_FP8_E4M3_UE8M0: return rows * (hidden / MOE_FP8_BLOCK);
    default: return 0;
  }
}

static int scale_blocks(int H, moe_dtype_t dtype) {
  switch (dtype) {
    case MOE_DTYPE_FP8_E4M3: return H / MOE_FP8_BLOCK;
    case MOE_DTYPE_FP8_E4M3_TOKEN: return 1;
    case MOE_DTYPE_MXFP8_E4M3: return H / 32;
    case MOE_DTYPE_NVFP4: return H / 16;
    case MOE_DTYPE_FP8_E4M3_UE8M0: return H / MOE_FP8_BLOCK;
    default: return 0;
  }
}

static bool byte_scales(moe_dtype_t dtype) {
  return dtype == MOE_DTYPE_MXFP8_E4M3 || dtype == MOE_DTYPE_NVFP4 || dtype == MOE_DTYPE_FP8_E4M3_UE8M0;
}

// whether `layout` is defined for the payload type (and its block count)
static bool scale_layout_defined(int H, moe_dtype_t dtype, moe_scale_layout_t layout) {
  if (layout == MOE_SCALE_ROW_MAJOR) return true;
  if (dtype == MOE_DTYPE_BF16 || scale_blocks(H, dtype) < 1) return false;
  if (layout == MOE_SCALE_MN_MAJOR) return true;
  if (layout == MOE_SCALE_MN_MAJOR_PACK4) return dtype == MOE_DTYPE_FP8_E4M3_UE8M0;
  return layout == MOE_SCALE_MMA_TILED &&
         (dtype == MOE_DTYPE_MXFP8_E4M3 || dtype == MOE_DTYPE_NVFP4) && scale_blocks(H, dtype) % 4 == 0;
}

size_t moe_recv_scale_bytes(int num_recv_rows, int hidden, moe_dtype_t dtype,
                            moe_scale_layout_t layout) {
  if (num_recv_rows < 0 || hidden < 1 || !scale_layout_defined(hidden, dtype, layout)) return 0;
  const size_t B = static_cast<size_t>(scale_blocks(hidden, dtype));
  const size_t es = byte_scales(dtype) ? 1 : sizeof(float);
  const size_t rows = static_cast<size_t>(num_recv_rows);
  switch (layout) {
    case MOE_SCALE_MN_MAJOR: return B * static_cast<size_t>(moe::scale_ld(num_recv_rows, dtype)) * es;
    case MOE_SCALE_MMA_TILED: return (rows + 127) / 128 * 128 * B;
    case MOE_SCALE_MN_MAJOR_PACK4: return (B + 3) / 4 * 4 * ((rows + 3) / 4 * 4);
    default: return rows * B * es;
  }
}

moe_status_t moe_selftest_bounded_wait(int32_t* d_status, moe_stream_t stream) {
  if (!d_status || !aligned(d_status, 4)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_bounded_wait_selftest(d_status, as_stream(stream)));
}

size_t moe_quant_fp8_channel_workspace_bytes(int num_experts, int hidden) {
  if (num_experts < 1 || num_experts > MOE_MAX_EXPERTS || hidden < 128 || hidden % 128 != 0) return 0;
  return moe::quant_fp8_channel_workspace_bytes(num_experts, hidden);
}

int moe_quant_fp8_channel_takes_workspace(int num_rows, int num_experts) {
  if (num_rows < 0 || num_experts < 1 || num_experts > MOE_MAX_EXPERTS) return 0;
  return moe::quant_fp8_channel_takes_workspace(num_rows, num_experts) ? 1 : 0;
}

moe_status_t moe_quant_fp8_channel(const void* recv, int num_rows, int hidden, int num_experts,
                                   const int32_t* expert_offset, const int32_t* expert_count,
                                   int transpose, void* out, float* scale, void* workspace,
                                   size_t workspace_bytes, int32_t* d_status, moe_stream_t stream) {
  if (num_rows < 0 || hidden < 1 || num_experts < 1) return MOE_ERR_INVALID_ARG;
  if (hidden % 128 != 0 || (transpose != 0 && transpose != 1)) return MOE_ERR_INVALID_ARG;
  if (num_experts > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!expert_offset || !expert_count || !scale || (num_rows > 0 && (!recv || !out)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(recv, 16) || !aligned(out, 16) || !aligned(scale, 4) || !aligned(expert_offset, 4) ||
      !aligned(expert_count, 4) || !aligned(d_status, 4) || !aligned(workspace, 16))
    return MOE_ERR_INVALID_ARG;
  if (workspace &&
      workspace_bytes < moe::quant_fp8_channel_workspace_bytes(num_experts, hidden))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_quant_fp8_channel(recv, num_rows, hidden, num_experts, expert_offset,
                                                 expert_count, transpose != 0, out, scale, d_status,
                                                 workspace, as_stream(stream)));
}

moe_status_t moe_swiglu_quant(const void* h, int num_rows, int inter, const int32_t* slot_token,
                              moe_dtype_t dtype, moe_scale_layout_t scale_layout, void* out,
                              void* out_scale, moe_stream_t stream) {
  if (num_rows < 0 || inter < 1) return MOE_ERR_INVALID_ARG;
  if (scale_layout != MOE_SCALE_ROW_MAJOR && scale_layout != MOE_SCALE_MN_MAJOR &&
      scale_layout != MOE_SCALE_MMA_TILED)
    return MOE_ERR_INVALID_ARG;
  switch (dtype) {
    case MOE_DTYPE_BF16:
      if (inter % 16 != 0) return MOE_ERR_INVALID_ARG;
      break;
    case MOE_DTYPE_FP8_E4M3:
      if (inter % MOE_FP8_BLOCK != 0) return MOE_ERR_INVALID_ARG;
      break;
    case MOE_DTYPE_FP8_E4M3_TOKEN:
      if (inter % 8 != 0) return MOE_ERR_INVALID_ARG;
      if (inter > 16384) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_DTYPE_MXFP8_E4M3:
      if (inter % 32 != 0) return MOE_ERR_INVALID_ARG;
      break;
    default:
      return MOE_ERR_INVALID_ARG;
  }
  if (!scale_layout_defined(inter, dtype, scale_layout)) return MOE_ERR_INVALID_ARG;
  // grid: y = 512-channel segments of a row (at most 65535)
  if ((inter + 511) / 512 > 65535) return MOE_ERR_UNSUPPORTED;
  if (num_rows == 0) return MOE_OK;
  if (!h || !out) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_BF16 && !out_scale) return MOE_ERR_INVALID_ARG;
  const int scale_align =
      (dtype == MOE_DTYPE_MXFP8_E4M3 || scale_layout != MOE_SCALE_ROW_MAJOR) ? 16 : 4;
  if (!aligned(h, 16) || !aligned(out, 16) || !aligned(slot_token, 4)) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_BF16 && !aligned(out_scale, scale_align)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_swiglu_quant(h, num_rows, inter, slot_token, dtype, scale_layout,
                                            out, out_scale, as_stream(stream)));
}

moe_status_t moe_dispatch_nvfp4(const void* x, int num_tokens, int hidden, int k,
                                const int32_t* token_slot, int num_recv_rows,
                                moe_scale_layout_t scale_layout, void* recv_x,
                                void* recv_block_scale, float* recv_row_scale, int32_t* d_status,
                                moe_stream_t stream) {
  const int N = num_tokens, H = hidden;
  if (N < 0 || H < 1 || k < 1 || num_recv_rows < 0) return MOE_ERR_INVALID_ARG;
  if (H % 64 != 0) return MOE_ERR_INVALID_ARG;
  if (scale_layout != MOE_SCALE_ROW_MAJOR && scale_layout != MOE_SCALE_MN_MAJOR &&
      scale_layout != MOE_SCALE_MMA_TILED)
    return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK || H > 16384) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * k > kMaxRows) return MOE_ERR_UNSUPPORTED;
  if (N == 0) return MOE_OK;
  if (!x || !token_slot || !recv_x || !recv_block_scale || !recv_row_scale) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(recv_x, 16) || !aligned(recv_block_scale, 16) ||
      !aligned(recv_row_scale, 4) || !aligned(token_slot, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_dispatch_nvfp4(x, N, H, k, token_slot, num_recv_rows, scale_layout,
                                              recv_x, recv_block_scale, recv_row_scale, d_status,
                                              as_stream(stream)));
}

moe_status_t moe_dispatch(const void* x, int num_tokens, int hidden, int k,
                          const int32_t* token_slot, int num_recv_rows, moe_dtype_t dtype,
                          void* recv_x, void* recv_scale, int32_t* d_status,
                          moe_stream_t stream) {
  return moe_dispatch_ex(x, num_tokens, hidden, k, token_slot, num_recv_rows, dtype,
                         MOE_SCALE_ROW_MAJOR, recv_x, recv_scale, d_status, stream);
}

moe_status_t moe_dispatch_ex(const void* x, int num_tokens, int hidden, int k,
                             const int32_t* token_slot, int num_recv_rows, moe_dtype_t dtype,
                             moe_scale_layout_t scale_layout, void* recv_x, void* recv_scale,
                             int32_t* d_status, moe_stream_t stream) {
  const int N = num_tokens, H = hidden;
  if (N < 0 || H < 1 || k < 1 || num_recv_rows < 0) return MOE_ERR_INVALID_ARG;
  if (scale_layout < MOE_SCALE_ROW_MAJOR || scale_layout > MOE_SCALE_MN_MAJOR_PACK4)
    return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * k > kMaxRows) return MOE_ERR_UNSUPPORTED;
  if (dtype == MOE_DTYPE_BF16) {
    if (H % 8 != 0) return MOE_ERR_INVALID_ARG;
  } else if (dtype == MOE_DTYPE_FP8_E4M3) {
    if (H % MOE_FP8_BLOCK != 0) return MOE_ERR_INVALID_ARG;
  } else if (dtype == MOE_DTYPE_FP8_E4M3_TOKEN) {
    if (H % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (H > 16384) return MOE_ERR_UNSUPPORTED;
  } else if (dtype == MOE_DTYPE_MXFP8_E4M3) {
    if (H % 32 != 0) return MOE_ERR_INVALID_ARG;
  } else if (dtype == MOE_DTYPE_E5M6) {
    if (H % 32 != 0) return MOE_ERR_INVALID_ARG;
  } else if (dtype == MOE_DTYPE_FP8_E4M3_UE8M0) {
    if (H % MOE_FP8_BLOCK != 0) return MOE_ERR_INVALID_ARG;
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  if (!scale_layout_defined(H, dtype, scale_layout)) return MOE_ERR_INVALID_ARG;
  if (N == 0) return MOE_OK;
  if (!x || !token_slot || !recv_x) return MOE_ERR_INVALID_ARG;
  const bool scaled = dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_E5M6;
  if (scaled && !recv_scale) return MOE_ERR_INVALID_ARG;
  const int scale_align = (byte_scales(dtype) || scale_layout != MOE_SCALE_ROW_MAJOR) ? 16 : 4;
  if (scaled && !aligned(recv_scale, scale_align)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(recv_x, 16) || !aligned(token_slot, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_dispatch(x, N, H, k, token_slot, num_recv_rows, dtype,
                                        scale_layout, recv_x, recv_scale, d_status,
                                        as_stream(stream)));
}

moe_status_t moe_combine(const void* y, int num_tokens, int hidden, int k,
                         const int32_t* token_slot, int num_recv_rows, const float* topk_w,
                         void* out, int32_t* d_status, moe_stream_t stream) {
  const int N = num_tokens, H = hidden;
  if (N < 0 || H < 1 || k < 1 || H % 8 != 0 || num_recv_rows < 0) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * k > kMaxRows) return MOE_ERR_UNSUPPORTED;
  if (N == 0) return MOE_OK;
  if (!y || !token_slot || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(out, 16) || !aligned(token_slot, 4) || !aligned(topk_w, 4) ||
      !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine(y, N, H, k, token_slot, num_recv_rows, topk_w, out,
                                       d_status, as_stream(stream)));
}

moe_status_t moe_dispatch_backward(const void* grad_recv, int num_tokens, int hidden, int k,
                                   const int32_t* token_slot, int num_recv_rows, void* grad_x,
                                   int32_t* d_status, moe_stream_t stream) {
  const int N = num_tokens, H = hidden;
  if (N < 0 || H < 1 || k < 1 || H % 8 != 0 || num_recv_rows < 0) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * k > kMaxRows) return MOE_ERR_UNSUPPORTED;
  if (N == 0) return MOE_OK;
  if (!grad_recv || !token_slot || !grad_x) return MOE_ERR_INVALID_ARG;
  if (!aligned(grad_recv, 16) || !aligned(grad_x, 16) || !aligned(token_slot, 4) ||
      !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARG;
  // the combine kernel with unit weights
  return from_cuda(moe::launch_combine(grad_recv, N, H, k, token_slot, num_recv_rows, nullptr,
                                       grad_x, d_status, as_stream(stream)));
}

moe_status_t moe_combine_backward(const void* grad_out, const void* y, int num_tokens, int hidden,
                                  int k, const int32_t* token_slot, int num_recv_rows,
                                  const float* topk_w, void* grad_y, float* grad_w,
                                  int32_t* d_status, moe_stream_t stream) {
  const int N = num_tokens, H = hidden;
  if (N < 0 || H < 1 || k < 1 || H % 8 != 0 || num_recv_rows < 0) return MOE_ERR_INVALID_ARG;
  if (k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * k > kMaxRows) return MOE_ERR_UNSUPPORTED;
  if (N == 0) return MOE_OK;
  if (!grad_out || !y || !token_slot || !topk_w || !grad_y || !grad_w) return MOE_ERR_INVALID_ARG;
  if (!aligned(grad_out, 16) || !aligned(y, 16) || !aligned(grad_y, 16) ||
      !aligned(token_slot, 4) || !aligned(topk_w, 4) || !aligned(grad_w, 4) ||
      !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_combine_backward(grad_out, y, N, H, k, token_slot, num_recv_rows,
                                                topk_w, grad_y, grad_w, d_status,
                                                as_stream(stream)));
}

moe_status_t moe_gate_math(uint32_t first, size_t n, float* exp_out, float* sigmoid_out,
                           float* silu_out, moe_stream_t stream) {
  if (n == 0) return MOE_OK;
  if ((!exp_out && !sigmoid_out && !silu_out) || !aligned(exp_out, 16) ||
      !aligned(sigmoid_out, 16) || !aligned(silu_out, 16))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(
      moe::launch_gate_math(first, n, exp_out, sigmoid_out, silu_out, as_stream(stream)));
}

moe_status_t moe_e4m3_encode(const float* in, size_t n, uint8_t* out, moe_stream_t stream) {
  if (n == 0) return MOE_OK;
  if (!in || !out || !aligned(in, 4)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_e4m3_encode(in, n, out, as_stream(stream)));
}

}  // extern "C"
