// layout_noalloc.cu -- moe_get_layout for callers that cannot allocate.
//
// moe_get_layout needs a few kilobytes of device scratch (per-chunk
// histograms) that the caller normally passes in.  Some callers have no way
// to produce it: a serving runtime that reserves all of the GPU's memory for
// its own pool at start-up, or a deployment whose memory plan is frozen
// before the first request, cannot call cudaMalloc (it would fail, or break
// the budget) and may have no pool this library can borrow from.  For them
// this file keeps the scratch in a file-scope __device__ array of fixed size,
// loaded with the library, and runs the same layout kernels on it.
//
// Costs and rules:
//  - every GPU that loads the library holds kScratchBytes of this array
//    until the process exits;
//  - all calls share the one array: calls whose GPU work overlaps (different
//    streams, or several host threads) race on it and corrupt each other's
//    result; serialise them;
//  - the array keeps whatever the last call left; nothing in it has to start
//    at zero, because the first layout kernel writes every word the second
//    one reads;
//  - the first call on a device looks up the array's device address (a
//    runtime call, done once per device with that device current); make that
//    first call before any stream capture.
#include <mutex>

#include "moe.h"

namespace {

constexpr size_t kScratchBytes = MOE_LAYOUT_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_layout_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the name g_layout_scratch is only a host-side stand-in, never a device
// address, so it must not be handed to a kernel.
moe_status_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_get_layout_noalloc(const int32_t* topk_idx, int num_tokens, int k,
                                               int num_experts, int num_ranks,
                                               int32_t* expert_count, int32_t* expert_offset,
                                               int32_t* rank_count, int32_t* rank_offset,
                                               int32_t* rank_tokens, int32_t* token_slot,
                                               int32_t* slot_token, int32_t* d_status,
                                               moe_stream_t stream) {
  const size_t need = moe_layout_workspace_bytes(num_tokens, k, num_experts, num_ranks);
  if (need == 0) return MOE_ERR_INVALID_ARG;
  if (need > kScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const moe_status_t st = scratch_address(&scratch);
  if (st != MOE_OK) return st;
  return moe_get_layout(topk_idx, num_tokens, k, num_experts, num_ranks, expert_count,
                        expert_offset, rank_count, rank_offset, rank_tokens, token_slot,
                        slot_token, scratch, kScratchBytes, d_status, stream);
}
