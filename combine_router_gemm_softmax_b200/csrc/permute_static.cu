// moe_permute_static_scratch: moe_permute for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand this library a workspace: code running
// under a custom or pool-only allocator that forbids cudaMalloc outside its
// own arena, plug-ins whose host framework owns all device memory, or code
// that must not allocate at all on a latency-critical path. This entry point
// takes the same inputs and outputs as moe_permute but keeps the permute
// scratch (the per-chunk expert counts and their scanned bases) in a
// fixed-size array that is part of the library's device image.
//
// Costs and rules:
//  - Every GPU that loads the library holds kStaticScratchBytes (1 MiB) for
//    this array until the process exits, whether or not this entry point is
//    ever called.
//  - All calls share the one array and it keeps whatever the last call left
//    there. Nothing in it has to start at zero (the counting kernel writes
//    every entry before the scan reads it), so nothing is cleared. Two calls
//    that can run at the same time on the GPU (different streams without an
//    ordering between them) race on the array and give wrong results.
//  - Every call that is not being captured into a CUDA graph looks up the
//    array's device address with cudaGetSymbolAddress while the stream's
//    device is current, and remembers it for that device. A call made during
//    stream capture uses the remembered address (it makes no runtime call that
//    capture could forbid), so make one call on each device before capturing.
//    Looking the address up again outside capture means a context torn down
//    and created again (cudaDeviceReset) cannot leave a stale address behind,
//    as long as it is not done between a capture and the graph's replay.
//  - The scratch needs 2 * roundup256(4 * E * ceil(T / 128)) bytes; when that
//    exceeds 1 MiB (E * ceil(T/128) > 131072, e.g. E = 256 with T > 65536)
//    the call returns MOE_ERR_WORKSPACE and enqueues nothing.
//  - No cudaMalloc, cudaFree or other allocating call is made.
#include <mutex>

#include "moe_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_permute_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_permute_scratch on the current device: looked up
// afresh outside stream capture, taken from the per-device record during
// capture. Host code must not use the symbol itself as a device pointer.
int scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_NO_DEVICE;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  } else if (g_scratch_addr[dev] == nullptr) {
    return MOE_ERR_CUDA;  // first call on this device made during capture
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int32_t moe_permute_static_scratch(const moe_config* cfg, const void* h, const int32_t* topk_idx,
                                              int32_t* routed_counts, int32_t* counts, int32_t* offsets,
                                              int32_t* dest_row, int32_t* perm_src, void* x_perm,
                                              int32_t* status_dev, moe_stream_t stream) {
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  if (moe_workspace_size(cfg, MOE_OP_PERMUTE) > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (rc != MOE_OK) return rc;
  return moe_permute(cfg, h, topk_idx, routed_counts, counts, offsets, dest_row, perm_src, x_perm, scratch,
                     kStaticScratchBytes, status_dev, stream);
}
