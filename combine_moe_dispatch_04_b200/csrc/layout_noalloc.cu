// moe_dispatch_layout_noalloc: the dispatch layout for callers that cannot
// allocate device memory. Instead of a caller-provided workspace it uses one
// fixed scratch array compiled into this library (declared below), so the
// call needs no cudaMalloc, no cudaFree and no allocator of any framework.
//
// The scratch is a file-scope __device__ array: every GPU that loads the
// library holds it (kNoAllocScratchBytes) until the process exits. In host
// code its name only stands in for the symbol; the device address is looked
// up once per device with cudaGetSymbolAddress (with that device current) the
// first time the entry point runs on that device, and cached.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "launch.cuh"
#include "moe_dc.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{1} << 20;  // 1 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_layout_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_layout_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t moe_layout_noalloc_max_workspace_bytes(void) { return kNoAllocScratchBytes; }

moe_status moe_dispatch_layout_noalloc(const moe_shape* s, const int32_t* topk_idx,
                                       const uint8_t* x_active_mask, int32_t* expert_token_nums,
                                       int32_t* ep_send_counts, int32_t* assist_info,
                                       uint32_t* dev_status, void* stream) {
  const size_t need = moe_layout_workspace_bytes(s);
  if (s != nullptr && need > kNoAllocScratchBytes) return MOE_ERR_CAPACITY;
  void* scratch = nullptr;
  if (need > 0) {
    // need > 0 only for shapes the size query accepted.
    const cudaError_t err = scratch_address(&scratch);
    if (err != cudaSuccess) return moe::report_cuda_error(err);
  }
  // Every entry of the scratch that the layout reads is written earlier in the
  // same call, so nothing has to be cleared between calls.
  return moe_dispatch_layout(s, topk_idx, x_active_mask, expert_token_nums, ep_send_counts,
                             assist_info, dev_status, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
