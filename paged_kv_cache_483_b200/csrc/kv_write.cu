// K1 reshape_and_cache and K2 copy-on-write block copy.
//
// Both are byte copies bounded by HBM bandwidth: 16-byte vector loads and
// stores, consecutive threads on consecutive 16-byte chunks of a row so every
// warp moves 512 contiguous bytes, grid sized as a multiple of the SM count.
//
// K1 writes token t's K/V rows (all KV heads) into slot slot_mapping[t]
// ("abhik.ai examples/pagedattention.py", KVPool.append: keys[physical,
// offset] = key).  K2 copies a whole block, every slot and head, of both
// caches ("abhik.ai examples/pagedattention.py", KVPool._private_tail).
#include <algorithm>

#include "common.cuh"
#include "launch.hpp"

namespace pa {

// One warp per token row: the slot is read once and the lanes copy the row's
// K and V vectors (no index division; up to four vectors of each in flight
// per lane).  The row's first vectors are loaded before the slot is known, so
// the slot's round trip overlaps the row's.
template <typename V>
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const V* __restrict__ key, const V* __restrict__ value,
    V* __restrict__ k_cache, V* __restrict__ v_cache,
    const int64_t* __restrict__ slot_mapping, int32_t T, int64_t row_vecs,
    int64_t num_slots, int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const int64_t slot = __ldg(slot_mapping + t);
    const V* ks = key + t * row_vecs;
    const V* vs = value + t * row_vecs;
    V k4[4], v4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (lane + 32 * u < row_vecs) {
        k4[u] = ks[lane + 32 * u];
        v4[u] = vs[lane + 32 * u];
      }
    }
    if (slot < 0) continue;                    // padding token
    if (slot >= num_slots) {
      if (lane == 0) raise_err(err, PA_DEVERR_SLOT);
      continue;
    }
    V* kd = k_cache + slot * row_vecs;
    V* vd = v_cache + slot * row_vecs;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (lane + 32 * u < row_vecs) {
        kd[lane + 32 * u] = k4[u];
        vd[lane + 32 * u] = v4[u];
      }
    }
    int64_t c = lane + 128;
    for (; c + 96 < row_vecs; c += 128) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        k4[u] = ks[c + 32 * u];
        v4[u] = vs[c + 32 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        kd[c + 32 * u] = k4[u];
        vd[c + 32 * u] = v4[u];
      }
    }
    for (; c < row_vecs; c += 32) {
      kd[c] = ks[c];
      vd[c] = vs[c];
    }
  }
}

template <typename V>
__global__ void __launch_bounds__(256) cow_copy_kernel(
    V* __restrict__ k_cache, V* __restrict__ v_cache,
    const int32_t* __restrict__ src, const int32_t* __restrict__ dst,
    int32_t n, int64_t block_vecs, int32_t num_blocks, int32_t* err) {
  const int64_t total = int64_t(n) * block_vecs;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t p = i / block_vecs, c = i - p * block_vecs;
    const int32_t s = __ldg(src + p), d = __ldg(dst + p);
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
      if (c == 0) raise_err(err, PA_DEVERR_BLOCK_ID);
      continue;
    }
    k_cache[int64_t(d) * block_vecs + c] = k_cache[int64_t(s) * block_vecs + c];
    if (v_cache) v_cache[int64_t(d) * block_vecs + c] = v_cache[int64_t(s) * block_vecs + c];
  }
}

// E4M3 code of y, |y| <= 448 (float64): the nearest value of the E4M3 grid
// of the OCP 8-bit floating point specification (exponent bias 7, 3 mantissa
// bits, subnormals, largest finite 448), ties to the even code; a zero
// magnitude gives +0.  Inside binade e (floored at -6, the subnormal range)
// the grid step is 2^(e - 3), so m = rint(|y| / 2^(e - 3)) lies in [8, 16]
// ([0, 8] for subnormals) and the code is (e + 7) * 8 + m - 8 -- which is
// also right when m rounds up to 16, the next binade's first value.
__device__ __forceinline__ uint32_t e4m3_code(double y) {
  const double a = fmin(fabs(y), 448.0);
  const int e = max(int((__double_as_longlong(a) >> 52) & 0x7FF) - 1023, -6);
  const double m = rint(a * __longlong_as_double(int64_t(1023 + 3 - e) << 52));
  const uint32_t mag = uint32_t((e + 7) * 8 + int(m) - 8);
  return (mag != 0u && y < 0.0) ? (mag | 0x80u) : mag;
}

// Quantised pools: one warp per (token, head) row of K and of V.  The row's
// absmax is exact in float32 (bf16 inputs); the codes are decided in float64
// as the quantisation experiment of "vladkulikov.com modern-llms module 9
// notebook" states:
//  * int8: scale = absmax / 127, code = rint(x / scale) clipped to +-127;
//  * fp8 (E4M3): scale = absmax / 448, code = the nearest E4M3 value to
//    x / scale (the same per-row recipe on the 8-bit float grid).
// A zero row takes scale 1.  The scale is stored as float32.  Returns this
// lane's 4 codes (d = 4 lane .. 4 lane + 3) packed in a word; lane 0 also
// stores the scale.
template <bool kFp8>
__device__ __forceinline__ uint32_t quantize_row(const __nv_bfloat16* __restrict__ src,
                                                 float* scale_dst, int lane) {
  const uint2 w = *reinterpret_cast<const uint2*>(src + 4 * lane);
  float x[4];
  x[0] = __uint_as_float(w.x << 16);
  x[1] = __uint_as_float(w.x & 0xFFFF0000u);
  x[2] = __uint_as_float(w.y << 16);
  x[3] = __uint_as_float(w.y & 0xFFFF0000u);
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const double limit = kFp8 ? 448.0 : 127.0;
  double scale = double(amax) / limit;
  if (scale == 0.0) scale = 1.0;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double t = fmin(fmax(double(x[i]) / scale, -limit), limit);
    const uint32_t code = kFp8 ? e4m3_code(t) : (uint32_t(int32_t(rint(t))) & 0xFFu);
    packed |= code << (8 * i);
  }
  if (lane == 0) *scale_dst = __double2float_rn(scale);
  return packed;
}

// Writes each row into its packed (block, head) record: K codes at
// token * 128 + ((chunk ^ (token & 7)) << 4) + byte, V codes at 2048 + d * 16
// + token, scales at 4096 + 4 token (K) and 4160 + 4 token (V).
template <bool kFp8>
__global__ void __launch_bounds__(256) reshape_and_cache_q8_kernel(
    const __nv_bfloat16* __restrict__ key, const __nv_bfloat16* __restrict__ value,
    uint8_t* __restrict__ records, const int64_t* __restrict__ slot_mapping, int32_t T,
    int32_t Hkv, int64_t num_slots, int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = int64_t(T) * Hkv;
  const int64_t stride = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += stride) {
    const int64_t t = r / Hkv;
    const int h = int(r - t * Hkv);
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;                    // padding token
    if (slot >= num_slots) {
      if (lane == 0 && h == 0) raise_err(err, PA_DEVERR_SLOT);
      continue;
    }
    const int tok = int(slot & 15);
    uint8_t* rec = records + ((slot >> 4) * Hkv + h) * kQ8RecordBytes;
    const uint32_t kw =
        quantize_row<kFp8>(key + r * 128, reinterpret_cast<float*>(rec + 4096) + tok, lane);
    const uint32_t vw =
        quantize_row<kFp8>(value + r * 128, reinterpret_cast<float*>(rec + 4160) + tok, lane);
    // lane covers d = 4 lane .. + 3: chunk lane / 4, byte 4 (lane % 4)
    *reinterpret_cast<uint32_t*>(rec + tok * 128 + (((lane >> 2) ^ (tok & 7)) << 4) +
                                 4 * (lane & 3)) = kw;
#pragma unroll
    for (int i = 0; i < 4; ++i) rec[2048 + (4 * lane + i) * 16 + tok] = uint8_t(vw >> (8 * i));
  }
}

cudaError_t launch_reshape_and_cache_q8(const void* key, const void* value, void* records,
                                        const int64_t* slots, int32_t T, int32_t Hkv,
                                        int64_t num_slots, bool fp8, int32_t* err, int sms,
                                        cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int64_t rows = int64_t(T) * Hkv;
  int64_t g = (rows + 7) / 8;
  g = g > int64_t(sms) * 8 ? int64_t(sms) * 8 : g;
  const int grid = int(g < 1 ? 1 : g);
  auto* kern = fp8 ? reshape_and_cache_q8_kernel<true> : reshape_and_cache_q8_kernel<false>;
  kern<<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(key), static_cast<const __nv_bfloat16*>(value),
      static_cast<uint8_t*>(records), slots, T, Hkv, num_slots, err);
  return cudaGetLastError();
}

// Block-table patches of a prepared decode batch: entry (row, index) of the
// device tables [rows, width] takes value, for each (row, index, value) triple
// the host found changed since the previous step.
__global__ void __launch_bounds__(256) table_patch_kernel(int32_t* __restrict__ tables,
                                                          int32_t width,
                                                          const int32_t* __restrict__ patches,
                                                          int32_t n) {
  for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    tables[int64_t(patches[3 * i]) * width + patches[3 * i + 1]] = patches[3 * i + 2];
}

cudaError_t launch_table_patch(int32_t* tables, int32_t width, const int32_t* patches,
                               int32_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int grid = int(std::min<int64_t>((int64_t(n) + 255) / 256, 1024));
  table_patch_kernel<<<grid, 256, 0, stream>>>(tables, width, patches, n);
  return cudaGetLastError();
}

static int grid_for(int64_t work, int sms) {
  int64_t g = (work + 255) / 256;
  int64_t cap = int64_t(sms) * 8;
  if (g > cap) g = cap;
  return int(g < 1 ? 1 : g);
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value,
                                     void* k_cache, void* v_cache,
                                     const int64_t* slots, int32_t T,
                                     int64_t row_bytes, int64_t num_slots,
                                     int32_t* err, int sms,
                                     cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  auto aligned = [](const void* p, int a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
  };
  if (row_bytes % 16 == 0 && aligned(key, 16) && aligned(value, 16) &&
      aligned(k_cache, 16) && aligned(v_cache, 16)) {
    int64_t rv = row_bytes / 16;
    reshape_and_cache_kernel<uint4><<<grid_for(int64_t(T) * 32, sms), 256, 0, stream>>>(
        (const uint4*)key, (const uint4*)value, (uint4*)k_cache,
        (uint4*)v_cache, slots, T, rv, num_slots, err);
  } else if (row_bytes % 4 == 0) {
    int64_t rv = row_bytes / 4;
    reshape_and_cache_kernel<uint32_t><<<grid_for(int64_t(T) * 32, sms), 256, 0, stream>>>(
        (const uint32_t*)key, (const uint32_t*)value, (uint32_t*)k_cache,
        (uint32_t*)v_cache, slots, T, rv, num_slots, err);
  } else {
    int64_t rv = row_bytes / 2;
    reshape_and_cache_kernel<uint16_t><<<grid_for(int64_t(T) * 32, sms), 256, 0, stream>>>(
        (const uint16_t*)key, (const uint16_t*)value, (uint16_t*)k_cache,
        (uint16_t*)v_cache, slots, T, rv, num_slots, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_cow_copy(void* k_cache, void* v_cache, const int32_t* src,
                            const int32_t* dst, int32_t n, int64_t block_bytes,
                            int32_t num_blocks, int32_t* err, int sms,
                            cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  if (block_bytes % 16 == 0) {
    int64_t bv = block_bytes / 16;
    cow_copy_kernel<uint4><<<grid_for(n * bv, sms), 256, 0, stream>>>(
        (uint4*)k_cache, (uint4*)v_cache, src, dst, n, bv, num_blocks, err);
  } else if (block_bytes % 4 == 0) {
    int64_t bv = block_bytes / 4;
    cow_copy_kernel<uint32_t><<<grid_for(n * bv, sms), 256, 0, stream>>>(
        (uint32_t*)k_cache, (uint32_t*)v_cache, src, dst, n, bv, num_blocks,
        err);
  } else {
    int64_t bv = block_bytes / 2;
    cow_copy_kernel<uint16_t><<<grid_for(n * bv, sms), 256, 0, stream>>>(
        (uint16_t*)k_cache, (uint16_t*)v_cache, src, dst, n, bv, num_blocks,
        err);
  }
  return cudaGetLastError();
}

}  // namespace pa
