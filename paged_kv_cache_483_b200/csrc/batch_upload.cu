// The step-input upload of a prepared decode batch (pa_batch_step).
#include "launch.hpp"

namespace pa {

// Upload of a prepared batch step's inputs in one launch: the threads read
// the caller's pinned host buffers through their mapped device addresses and
// write the device copies, 16 bytes per load, two loads in flight per thread.
// One launch stands in for one copy per buffer, whose fixed set-up cost was as
// large as the transfer for buffers of a few hundred KB.  128 threads of at
// most 32 registers: a CTA fits beside three CTAs of the bf16 decode on an SM,
// so the upload runs while the previous step's decode does.
__device__ __forceinline__ void upload_segment(const UploadSeg& g, int64_t first,
                                               int64_t stride) {
  const uint4* __restrict__ src = g.src;
  uint4* __restrict__ dst = g.dst;
  int64_t i = first;
#pragma unroll 1
  for (; i + stride < g.n16; i += 2 * stride) {
    const uint4 a = src[i], b = src[i + stride];
    dst[i] = a;
    dst[i + stride] = b;
  }
  if (i < g.n16) dst[i] = src[i];
}

__global__ void __launch_bounds__(128, 16) upload_kernel(const __grid_constant__ UploadArgs a) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t first = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  upload_segment(a.seg[0], first, stride);
  upload_segment(a.seg[1], first, stride);
  upload_segment(a.seg[2], first, stride);
  upload_segment(a.seg[3], first, stride);
}

cudaError_t launch_upload(const UploadArgs& a, int sms, cudaStream_t stream) {
  static_assert(kUploadSegs == 4, "upload_kernel walks four segments");
  int64_t total = 0;
  for (const auto& g : a.seg) total += g.n16;
  if (total <= 0) return cudaSuccess;
  int64_t grid = (total + 511) / 512;
  if (grid > sms) grid = sms;
  upload_kernel<<<int(grid), 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace pa
