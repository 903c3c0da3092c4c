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

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

cudaStream_t as_stream(moe_stream_t s) { return static_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

int moe_abi_version(void) { return 2; }

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

size_t moe_recv_bytes(int num_tokens, int hidden, int k, moe_dtype_t dtype) {
  if (num_tokens < 0 || hidden < 1 || k < 1) return 0;
  const size_t esz = dtype == MOE_DTYPE_FP8_E4M3 ? 1 : 2;
  return static_cast<size_t>(num_tokens) * k * hidden * esz;
}

size_t moe_scale_bytes(int num_tokens, int hidden, int k, moe_dtype_t dtype) {
  if (num_tokens < 0 || hidden < 1 || k < 1) return 0;
  const size_t rows = static_cast<size_t>(num_tokens) * k;
  switch (dtype) {
    case MOE_DTYPE_FP8_E4M3: return rows * (hidden / MOE_FP8_BLOCK) * sizeof(float);
    case MOE_DTYPE_FP8_E4M3_TOKEN: return rows * sizeof(float);
    case MOE_DTYPE_MXFP8_E4M3: return rows * (hidden / 32);
    default: return 0;
  }
}

moe_status_t moe_dispatch(const void* x, int num_tokens, int hidden, int k,
                          const int32_t* token_slot, int num_recv_rows, moe_dtype_t dtype,
                          void* recv_x, void* recv_scale, int32_t* d_status,
                          moe_stream_t stream) {
  const int N = num_tokens, H = hidden;
  if (N < 0 || H < 1 || k < 1 || num_recv_rows < 0) return MOE_ERR_INVALID_ARG;
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
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  if (N == 0) return MOE_OK;
  if (!x || !token_slot || !recv_x) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_BF16 && !recv_scale) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_BF16 && !aligned(recv_scale, dtype == MOE_DTYPE_MXFP8_E4M3 ? 16 : 4))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(recv_x, 16) || !aligned(token_slot, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_dispatch(x, N, H, k, token_slot, num_recv_rows, dtype, recv_x,
                                        recv_scale, d_status, as_stream(stream)));
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

moe_status_t moe_e4m3_encode(const float* in, size_t n, uint8_t* out, moe_stream_t stream) {
  if (n == 0) return MOE_OK;
  if (!in || !out || !aligned(in, 4)) return MOE_ERR_INVALID_ARG;
  return from_cuda(moe::launch_e4m3_encode(in, n, out, as_stream(stream)));
}

}  // extern "C"
