// Split-K decode whose partition scratch lives in a fixed device array.
//
// pa_decode needs a caller-provided workspace when it splits sequences into
// partitions.  Some callers cannot allocate one: a serving process that hands
// all device memory to its KV pool and weights at start-up and treats any later
// cudaMalloc as a failure (a late cudaMalloc can stall until the device is idle
// and fails once the pool owns the memory), or a plugin whose host framework
// owns the device allocator and forbids raw allocations.  This entry point
// gives them the same decode with the scratch taken from a file-scope
// __device__ array of PA_STATIC_SCRATCH_BYTES that every GPU loading the
// library keeps until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pa.h"
#include "launch.hpp"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];  // device address of the array, per device
std::mutex g_scratch_mu;

// The array's name in host code is only a host-side handle; the kernel needs
// its device address, looked up once per device with that device current.
pa_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_static_scratch(pa_pool* pool, const void* q, int32_t B,
                                              int32_t H, const int32_t* d_block_tables,
                                              int32_t max_blocks, const int32_t* d_kv_lens,
                                              float scale, int32_t partition_tokens,
                                              float* out, void* stream) {
  if (!pool) return PA_ERR_INVALID_ARG;
  // a host-only pool answers like every other device call, before any CUDA
  // call could create a context on whatever device is current
  if (pa::pool_device(pool) < 0) return PA_ERR_NO_DEVICE;
  pa::DeviceScope on_pool_device(pa::pool_device(pool));   // the scratch of the pool's device
  void* scratch = nullptr;
  pa_status st = scratch_for_current_device(&scratch);
  if (st != PA_OK) return st;
  const size_t need =
      pa_decode_workspace_bytes(pool, B, H, max_blocks, partition_tokens);
  if (need > size_t(PA_STATIC_SCRATCH_BYTES)) return PA_ERR_SCRATCH_LIMIT;
  // every partition writes all of its (m, l, o) entries before the combine
  // reads them, so nothing left over from an earlier call is ever read
  return pa_decode(pool, q, B, H, d_block_tables, max_blocks, d_kv_lens, scale,
                   partition_tokens, scratch, size_t(PA_STATIC_SCRATCH_BYTES), out,
                   stream);
}
