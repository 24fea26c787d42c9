// Generic CUDA-core paged attention (any dtype, head_dim <= 512, any block
// size, any group size, q_tokens >= 1).  One CTA per output row (b, qt, h);
// keys are visited in chunks of 128 with the one-pass (m, l, acc) update of
// "semidirectx cmu11-667 lecture19 infer_world.py", section 3
// (tiled_attention).  The scores follow "docs.rs ferrum-kv 0.4.0
// src/attention.rs" (paged_attention): kv_h = h / (H / Hkv), query qt sees
// positions j <= kv_len - q_tokens + qt.  This is the path for fp32 pools and
// for shapes the tensor-core kernels do not take (also chunked prefill and
// large groups over int8 / FP8 pools, whose elements it dequantises one by
// one); it is correct, not fast.
#include <math.h>

#include "common.cuh"
#include "launch.hpp"

namespace pa {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// Value of an E4M3 code (OCP 8-bit floating point: sign, 4 exponent bits of
// bias 7, 3 mantissa bits; exponent field 0 holds the subnormals m * 2^-9;
// 0x7F / 0xFF are NaN).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  float v;
  if (e == 0u)
    v = float(m) * 0.001953125f;                       // 2^-9
  else if (e == 15u && m == 7u)
    v = __int_as_float(0x7FC00000);
  else
    v = ldexpf(float(8u + m), int(e) - 10);            // (1 + m/8) 2^(e-7)
  return (c & 0x80u) ? -v : v;
}

// Element (token slot off of physical block pb, KV head kvh, dimension i) of
// a pool's K and V.
template <typename T>
struct PlainKV {                       // [num_blocks, bs, Hkv, d] K and V arrays
  const T* kc;
  const T* vc;
  int Hkv, d, bs;
  __device__ float k(int pb, int off, int kvh, int i) const {
    return to_f(kc[((int64_t(pb) * bs + off) * Hkv + kvh) * d + i]);
  }
  __device__ float v(int pb, int off, int kvh, int i) const {
    return to_f(vc[((int64_t(pb) * bs + off) * Hkv + kvh) * d + i]);
  }
};

template <bool kFp8>
struct Q8KV {                          // packed (block, head) records, bs 16, d 128
  const uint8_t* rec;
  int Hkv;
  __device__ const uint8_t* at(int pb, int kvh) const {
    return rec + (int64_t(pb) * Hkv + kvh) * kQ8RecordBytes;
  }
  __device__ float code(uint32_t c) const {
    return kFp8 ? e4m3_value(c) : float(int(int8_t(uint8_t(c))));
  }
  __device__ float k(int pb, int off, int kvh, int i) const {
    const uint8_t* r = at(pb, kvh);
    const uint32_t c = r[off * 128 + ((((i >> 4) ^ (off & 7)) << 4) | (i & 15))];
    return code(c) * reinterpret_cast<const float*>(r + 4096)[off];
  }
  __device__ float v(int pb, int off, int kvh, int i) const {
    const uint8_t* r = at(pb, kvh);
    return code(r[2048 + i * 16 + off]) * reinterpret_cast<const float*>(r + 4160)[off];
  }
};

constexpr int kGenThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kGenThreads / 32; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < kGenThreads / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

template <typename T, typename KV>
__global__ void __launch_bounds__(kGenThreads) attention_generic_kernel(
    const T* __restrict__ q, const KV kv,
    const int32_t* __restrict__ tables, int MB, const int32_t* __restrict__ kv_lens,
    int q_tokens, int H, int Hkv, int d, int bs, int NB, float scale_log2,
    float* __restrict__ out, int32_t* err, int window, int sinks) {
  extern __shared__ float gen_smem[];
  float* qf = gen_smem;              // [d]
  float* pr = qf + d;                // [128] scores, then weights
  int* blk = (int*)(pr + kGenThreads);   // [128] physical block per key
  float* red = (float*)(blk + kGenThreads);  // [32]
  __shared__ int bad;

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (H / Hkv);
  const int tid = threadIdx.x;
  const int kv_len = kv_lens[b];
  float* orow = out + ((int64_t(b) * q_tokens + qt) * H + h) * d;

  const bool len_bad = kv_len < 0 || kv_len > MB * bs ||
                       (q_tokens > 1 && kv_len < q_tokens) ||
                       (q_tokens == 1 && kv_len < 0);
  if (tid == 0) bad = 0;
  if (len_bad) {
    if (tid == 0 && qt == 0 && h == 0) raise_err(err, PA_DEVERR_KV_LEN);
    for (int i = tid; i < d; i += kGenThreads) orow[i] = 0.f;
    return;
  }
  int visible = kv_len - q_tokens + qt + 1;  // keys 0 .. visible-1
  // Sink + recent window (decode, window > 0): the keys walked are the first
  // `sinks` and the last `window` ("vladkulikov.com modern-llms module 9
  // notebook", streaming_keep_indices); walk index v maps to key key_at(v).
  int lo = 0, ns = visible;
  if (window > 0 && visible > sinks + window) {
    ns = sinks;
    lo = visible - window;
    visible = sinks + window;
  }
  auto key_at = [&](int v) { return v < ns ? v : lo + (v - ns); };
  const T* qrow = q + ((int64_t(b) * q_tokens + qt) * H + h) * d;
  for (int i = tid; i < d; i += kGenThreads) qf[i] = to_f(qrow[i]) * scale_log2;
  __syncthreads();

  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // d <= 512 = 4 x 128
  float m = -INFINITY, l = 0.f;
  for (int c0 = 0; c0 < visible; c0 += kGenThreads) {
    const int j = c0 + tid < visible ? key_at(c0 + tid) : 0;
    float s = -INFINITY;
    int pb = -1;
    if (c0 + tid < visible) {
      pb = tables[int64_t(b) * MB + j / bs];
      if (pb < 0 || pb >= NB) {
        bad = 1;
        pb = -1;
      } else {
        const int off = j % bs;
        float dot = 0.f;
        for (int i = 0; i < d; ++i) dot = fmaf(qf[i], kv.k(pb, off, kvh, i), dot);
        s = dot;
      }
    }
    blk[tid] = pb;
    const float cmax = block_max(s, red);
    const float m_new = fmaxf(m, cmax);
    const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
    const float p = (s == -INFINITY) ? 0.f : exp2f(s - m_new);
    pr[tid] = p;
    const float csum = block_sum(p, red);  // also publishes pr/blk
    l = l * alpha + csum;
    m = (cmax == -INFINITY) ? m : m_new;
    const int n = min(kGenThreads, visible - c0);
    for (int r = 0; r < 4; ++r) {
      const int i = tid + r * kGenThreads;
      if (i >= d) break;
      float a = acc[r] * alpha;
      for (int jj = 0; jj < n; ++jj) {
        const int pbj = blk[jj];
        if (pbj < 0) continue;
        const int jt = key_at(c0 + jj);
        a = fmaf(pr[jj], kv.v(pbj, jt % bs, kvh, i), a);
      }
      acc[r] = a;
    }
    __syncthreads();
  }
  const bool zero = bad || !(l > 0.f);
  if (bad && tid == 0) raise_err(err, PA_DEVERR_BLOCK_ID);
  for (int r = 0; r < 4; ++r) {
    const int i = tid + r * kGenThreads;
    if (i < d) orow[i] = zero ? 0.f : acc[r] / l;
  }
}

cudaError_t launch_attention_generic(const GenericArgs& a, cudaStream_t s) {
  dim3 grid(a.q_tokens, a.H, a.B);
  size_t smem = sizeof(float) * (a.d + kGenThreads + 32) + sizeof(int) * kGenThreads;
  const float sl2 = a.scale * kLog2e;
  const int32_t* t = a.tables;
  if (a.q8) {                          // bf16 queries over packed int8 / FP8 records
    const auto* q = static_cast<const __nv_bfloat16*>(a.q);
    const auto* rec = static_cast<const uint8_t*>(a.k_cache);
    if (a.q8 == 2)
      attention_generic_kernel<<<grid, kGenThreads, smem, s>>>(
          q, Q8KV<true>{rec, a.Hkv}, t, a.MB, a.kv_lens, a.q_tokens, a.H, a.Hkv, a.d, a.bs,
          a.NB, sl2, a.out, a.err, a.window, a.sinks);
    else
      attention_generic_kernel<<<grid, kGenThreads, smem, s>>>(
          q, Q8KV<false>{rec, a.Hkv}, t, a.MB, a.kv_lens, a.q_tokens, a.H, a.Hkv, a.d, a.bs,
          a.NB, sl2, a.out, a.err, a.window, a.sinks);
  } else if (a.bf16) {
    using B = __nv_bfloat16;
    attention_generic_kernel<<<grid, kGenThreads, smem, s>>>(
        static_cast<const B*>(a.q),
        PlainKV<B>{static_cast<const B*>(a.k_cache), static_cast<const B*>(a.v_cache), a.Hkv,
                   a.d, a.bs},
        t, a.MB, a.kv_lens, a.q_tokens, a.H, a.Hkv, a.d, a.bs, a.NB, sl2, a.out, a.err,
        a.window, a.sinks);
  } else {
    attention_generic_kernel<<<grid, kGenThreads, smem, s>>>(
        static_cast<const float*>(a.q),
        PlainKV<float>{static_cast<const float*>(a.k_cache),
                       static_cast<const float*>(a.v_cache), a.Hkv, a.d, a.bs},
        t, a.MB, a.kv_lens, a.q_tokens, a.H, a.Hkv, a.d, a.bs, a.NB, sl2, a.out, a.err,
        a.window, a.sinks);
  }
  return cudaGetLastError();
}

}  // namespace pa
