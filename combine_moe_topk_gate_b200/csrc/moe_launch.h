// moe_launch.h -- internal launchers behind the C ABI (api.cu validates the
// arguments, these only pick a launch shape and enqueue the kernels).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

cudaError_t launch_topk_gate(const float* logits, int N, int E, int k, int kind, int n_groups,
                             int topk_groups, int group_topn, int32_t* topk_idx, float* topk_w,
                             cudaStream_t stream);

size_t layout_workspace_bytes(int N, int k, int E, int R);

// Outputs of the layout step (the routing handle) and the receive buffer's
// shape, as the fused routing launcher takes them.
struct RouteOut {
  int32_t* expert_count;
  int32_t* expert_offset;
  int32_t* rank_count;
  int32_t* rank_offset;
  int32_t* rank_tokens;
  int32_t* token_slot;
  int32_t* slot_token;
  int align;
  long long num_rows;
  int32_t* d_status;
  const void* prefetch;   // optional: a buffer the caller reads next, fetched into L2
  size_t prefetch_bytes;
};

// Routing workspace: an arrival counter in the first kRouteCounterBytes (zero
// before the first call, left zero by every call), then the layout's
// per-chunk counts (scratch).
constexpr size_t kRouteCounterBytes = 256;
size_t route_workspace_bytes(int N, int k, int E, int R);
cudaError_t launch_route(const float* logits, int N, int E, int k, int kind, int n_groups,
                         int topk_groups, int group_topn, int R, int32_t* topk_idx, float* topk_w,
                         const RouteOut& out, void* workspace, cudaStream_t stream);


cudaError_t launch_layout(const int32_t* topk_idx, int N, int k, int E, int R, int align,
                          long long num_rows, int32_t* expert_count, int32_t* expert_offset,
                          int32_t* rank_count, int32_t* rank_offset, int32_t* rank_tokens,
                          int32_t* token_slot, int32_t* slot_token, void* workspace,
                          int32_t* d_status, cudaStream_t stream);

// num_rows: rows of the receive buffer (N*k packed, more for aligned layouts);
// slots outside [-1, num_rows) are skipped and reported.
cudaError_t launch_dispatch(const void* x, int N, int H, int k, const int32_t* token_slot,
                            long long num_rows, int dtype, int scale_layout, void* recv_x,
                            void* recv_scale, int32_t* d_status, cudaStream_t stream);
// leading dimension of MN-major scales: num_rows padded to 16 bytes of scales
long long scale_ld(long long num_rows, int dtype);
cudaError_t launch_dispatch_nvfp4(const void* x, int N, int H, int k, const int32_t* token_slot,
                                  long long num_rows, int scale_layout, void* recv_x,
                                  void* block_scale, float* row_scale, int32_t* d_status,
                                  cudaStream_t stream);
size_t quant_fp8_channel_workspace_bytes(int E, int H);
bool quant_fp8_channel_takes_workspace(long long num_rows, int E);
cudaError_t launch_quant_fp8_channel(const void* x, long long num_rows, int H, int E,
                                     const int32_t* expert_offset, const int32_t* expert_count,
                                     bool transpose, void* out, float* scale, int32_t* d_status,
                                     void* workspace, cudaStream_t stream);
cudaError_t launch_bounded_wait_selftest(int32_t* d_status, cudaStream_t stream);
cudaError_t launch_swiglu_quant(const void* h, long long num_rows, int I, const int32_t* slot_token,
                                int dtype, int scale_layout, void* out, void* out_scale,
                                cudaStream_t stream);

cudaError_t launch_combine(const void* y, int N, int H, int k, const int32_t* token_slot,
                           long long num_rows, const float* topk_w, void* out, int32_t* d_status,
                           cudaStream_t stream);

cudaError_t launch_combine_backward(const void* grad_out, const void* y, int N, int H, int k,
                                    const int32_t* token_slot, long long num_rows,
                                    const float* topk_w, void* grad_y, float* grad_w,
                                    int32_t* d_status, cudaStream_t stream);

cudaError_t launch_gate_math(uint32_t first, size_t n, float* exp_out, float* sigmoid_out,
                             float* silu_out, cudaStream_t stream);

cudaError_t launch_e4m3_encode(const float* in, size_t n, uint8_t* out, cudaStream_t stream);

}  // namespace moe
