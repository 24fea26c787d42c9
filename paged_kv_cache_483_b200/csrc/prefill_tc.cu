// Chunked prefill attention on tcgen05 tensor cores: bf16 K/V/Q, head_dim
// 128, block_size 16, GQA group G in {1, 2, 4, 8}.
//
// What it computes ("docs.rs ferrum-kv 0.4.0 src/attention.rs",
// paged_attention with q_tokens > 1): the chunk's q_tokens queries are the
// last q_tokens positions of the sequence; query qt of head h sees keys
// j <= kv_len - q_tokens + qt of KV head h / G, read through the block table;
// softmax(q.k * scale) weighted sum of V, with the one-pass (m, l, acc)
// update of "semidirectx cmu11-667 lecture19 infer_world.py", section 3.
//
// One CTA = one 128-row query tile of one (sequence, KV head): rows are
// (token, head) pairs, 128/G tokens x G heads, so the G query heads that share
// a KV head share every K/V tile.  Keys are visited in tiles of 128 (eight
// paged blocks, each fetched by TMA as two 64-column boxes with the 128-byte
// swizzle, landing exactly in the UMMA K-major layout).
//   warp 0      TMA producer (Q once; K and V tiles into a 2-stage ring)
//   warp 1      one thread issues tcgen05.mma: S = Q K^T into TMEM (double
//               buffered, 2 x 128 columns), then O += P V (O: 128 columns)
//   warps 2-5   softmax, one thread per row = TMEM lane: load the S row,
//               causal mask, running max, exp2, row sum, P as bf16 into shared
//               memory (K-major, swizzled) for the PV MMA; O is rescaled in
//               TMEM only when a row's max grows by more than 2^8 (a stale max
//               below that keeps every exponent <= 2^8, exact in fp32)
//   epilogue    O / l from TMEM to global fp32.
// The QK^T of tile j+1 runs on the tensor core while the softmax of tile j
// runs on the CUDA cores.  P is rounded to bf16 for the PV product.
#include <math.h>

#include "common.cuh"
#include "launch.hpp"
#include "tcgen05.cuh"

namespace pa {

namespace {

constexpr int kPfThreads = 192;
constexpr int kPfStages = 2;
constexpr uint32_t kTile = 32768;  // 128 x 128 bf16
constexpr uint32_t kHalf = 16384;  // 128 x 64 bf16 (one 128-byte-swizzled half)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTile;
constexpr uint32_t kOffV = kTile * (1 + kPfStages);
constexpr uint32_t kOffP = kTile * (1 + 2 * kPfStages);
constexpr uint32_t kDataBytes = kTile * (2 + 2 * kPfStages);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr float kRescaleTau = 8.0f;
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);

struct PfBars {
  uint64_t q_full;
  uint64_t k_full[kPfStages], k_empty[kPfStages];
  uint64_t v_full[kPfStages], v_empty[kPfStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, o_done;
  uint32_t tmem_base;
  int abort;
  int bad;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              PfBars* bars, int32_t* err) {
  if (mbar_wait(bar, parity)) return true;
  raise_err(err, PA_DEVERR_TIMEOUT);
  atomicExch(&bars->abort, 1);
  return false;
}

}  // namespace

__global__ void __launch_bounds__(kPfThreads, 1) prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const PrefillArgs p, float scale_log2) {
  extern __shared__ uint8_t pf_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(pf_raw) + 1023) & ~uintptr_t(1023));
  PfBars* bars = reinterpret_cast<PfBars*>(smem + kDataBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.H / p.Hkv, TQ = 128 / G;
  const int mt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int t0 = mt * TQ;
  const int q_tokens = p.q_tokens;
  const int kv_len = p.kv_lens[b];
  const int valid_tokens = min(TQ, q_tokens - t0);
  const bool len_bad = kv_len < q_tokens || kv_len > p.MB * 16;
  const int qpos0 = kv_len - q_tokens + t0;        // key limit of the first token
  const int key_end = len_bad ? 0 : qpos0 + valid_tokens;
  const int n_tiles = (key_end + 127) >> 7;
  const int n_blk = (key_end + 15) >> 4;
  const int32_t* trow = p.tables + int64_t(b) * p.MB;

  if (threadIdx.x == 0) {
    bars->abort = 0;
    bars->bad = len_bad ? 1 : 0;
  }
  __syncthreads();
  // every block id the tile will touch must be inside the pool
  for (int i = threadIdx.x; i < n_blk; i += blockDim.x) {
    const int blk = trow[i];
    if (blk < 0 || blk >= p.NB) bars->bad = 2;
  }
  __syncthreads();
  if (bars->bad) {
    if (threadIdx.x == 0)
      raise_err(p.err, bars->bad == 1 ? PA_DEVERR_KV_LEN : PA_DEVERR_BLOCK_ID);
    for (int idx = threadIdx.x; idx < valid_tokens * G * 32; idx += blockDim.x) {
      const int row = idx >> 5, c4 = idx & 31;
      const int64_t o = ((int64_t(b) * q_tokens + t0 + row / G) * p.H + kvh * G + row % G) * 128;
      reinterpret_cast<float4*>(p.out + o)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], 128);
    }
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();
      mbar_arrive_expect_tx(&bars->q_full, kTile);
      tma_load_3d(smem + kOffQ, &tmQ, &bars->q_full, 0, kvh * G, b * q_tokens + t0, pol_q);
      tma_load_3d(smem + kOffQ + kHalf, &tmQ, &bars->q_full, 64, kvh * G, b * q_tokens + t0,
                  pol_q);
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kPfStages, round = j / kPfStages;
        if (round > 0) {
          if (!wait_or_abort(&bars->k_empty[s], (round - 1) & 1, bars, p.err)) break;
          if (!wait_or_abort(&bars->v_empty[s], (round - 1) & 1, bars, p.err)) break;
        }
        if (bars->abort) break;
        const int nb = min(8, n_blk - j * 8);
        uint8_t* kst = smem + kOffK + s * kTile;
        uint8_t* vst = smem + kOffV + s * kTile;
        mbar_arrive_expect_tx(&bars->k_full[s], nb * 4096);
        for (int i = 0; i < nb; ++i) {
          const int z = trow[j * 8 + i] * 16;
          tma_load_3d(kst + i * 2048, &tmK, &bars->k_full[s], 0, kvh, z, pol_kv);
          tma_load_3d(kst + kHalf + i * 2048, &tmK, &bars->k_full[s], 64, kvh, z, pol_kv);
        }
        mbar_arrive_expect_tx(&bars->v_full[s], nb * 4096);
        for (int i = 0; i < nb; ++i) {
          const int z = trow[j * 8 + i] * 16;
          tma_load_3d(vst + i * 2048, &tmV, &bars->v_full[s], 0, kvh, z, pol_kv);
          tma_load_3d(vst + kHalf + i * 2048, &tmV, &bars->v_full[s], 64, kvh, z, pol_kv);
        }
        issued = j + 1;
      }
      // drain: every issued copy has landed before the CTA may exit
      mbar_wait(&bars->q_full, 0);
      for (int s = 0; s < kPfStages && s < issued; ++s) {
        const int count = (issued - 1 - s) / kPfStages + 1;
        mbar_wait(&bars->k_full[s], (count - 1) & 1);
        mbar_wait(&bars->v_full[s], (count - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = wait_or_abort(&bars->q_full, 0, bars, p.err);
      tc_fence_after();
      const uint32_t qa = smem_u32(smem + kOffQ);
      const uint32_t pa_ = smem_u32(smem + kOffP);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % kPfStages;
          ok = wait_or_abort(&bars->k_full[s], (j / kPfStages) & 1, bars, p.err);
          if (ok && j >= 2)
            ok = wait_or_abort(&bars->s_free[j & 1], ((j - 2) >> 1) & 1, bars, p.err);
          if (!ok || bars->abort) break;
          tc_fence_after();
          const uint32_t kb = smem_u32(smem + kOffK + s * kTile);
          const uint32_t d = tbase + kColS + (j & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            umma_bf16(d, desc_kmajor_sw128(qa + off), desc_kmajor_sw128(kb + off), kIdescQK,
                      kk > 0);
          }
          umma_commit(&bars->s_full[j & 1]);
          umma_commit(&bars->k_empty[s]);
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj % kPfStages;
          ok = wait_or_abort(&bars->p_full, jj & 1, bars, p.err);
          if (ok) ok = wait_or_abort(&bars->v_full[s], (jj / kPfStages) & 1, bars, p.err);
          if (!ok || bars->abort) break;
          tc_fence_after();
          const uint32_t vb = smem_u32(smem + kOffV + s * kTile);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            umma_bf16(tbase + kColO, desc_kmajor_sw128(pa_ + off),
                      desc_mnmajor_sw128(vb + kk * 2048, kHalf, 1024), kIdescPV,
                      (jj > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->o_done);
          umma_commit(&bars->v_empty[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // row = TMEM lane
    const int t_local = r / G, g = r % G;
    const bool row_valid = t_local < valid_tokens;
    const int qpos = qpos0 + t_local;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    uint8_t* prow = smem + kOffP + r * 128;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1));
      if (!ok) {
        if (lane == 0) {
          raise_err(p.err, PA_DEVERR_TIMEOUT);
          atomicExch(&bars->abort, 1);
        }
        break;
      }
      tc_fence_after();
      float s[128];
      {
        const uint32_t sb = tbase + lane_off + kColS + (j & 1) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(sb + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(v[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->s_free[j & 1]);
      const int lim = qpos - j * 128;                  // columns c <= lim are visible
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = (c <= lim) ? s[c] : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      const float mt = mx * scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mt != -INFINITY && (m_ref == -INFINITY || mt > m_ref + kRescaleTau)) {
        alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mt);
        rescale = (j > 0);
        m_ref = mt;
      }
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (j - 1) & 1));
        if (!ok) {
          if (lane == 0) {
            raise_err(p.err, PA_DEVERR_TIMEOUT);
            atomicExch(&bars->abort, 1);
          }
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
          const uint32_t ob = tbase + lane_off + kColO;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(ob + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st32(ob + c * 32, v);
          }
        }
      }
      l *= alpha;
      if (j == n_tiles - 1) {
        // V rows at or past key_end hold stale bytes: zero them (p = 0 there,
        // and 0 x NaN would poison the product)
        const int s = j % kPfStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->v_full[s], (j / kPfStages) & 1));
        if (ok && j * 128 + r >= key_end) {
          uint4* v0 = reinterpret_cast<uint4*>(smem + kOffV + s * kTile + r * 128);
          uint4* v1 = reinterpret_cast<uint4*>(smem + kOffV + s * kTile + kHalf + r * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            v0[c] = make_uint4(0u, 0u, 0u, 0u);
            v1[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      float sum = 0.f;
      const float nm = -m_ref;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2(fmaf(s[ch * 8 + 2 * e], scale_log2, nm));
          const float p1 = ex2(fmaf(s[ch * 8 + 2 * e + 1], scale_log2, nm));
          sum += p0 + p1;
          w[e] = pack_bf16x2(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + (ch >> 3) * kHalf + (((ch & 7) ^ (r & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += sum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
    // epilogue: O / l
    bool done = ok && __all_sync(0xffffffffu,
                                 mbar_wait(&bars->o_done, (n_tiles - 1) & 1));
    if (!done && lane == 0) {
      raise_err(p.err, PA_DEVERR_TIMEOUT);
      atomicExch(&bars->abort, 1);
    }
    tc_fence_after();
    const float inv = (done && l > 0.f) ? 1.f / l : 0.f;
    float* orow = p.out + ((int64_t(b) * q_tokens + t0 + t_local) * p.H + kvh * G + g) * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld32(tbase + lane_off + kColO + c * 32, v);
      if (row_valid) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(orow + c * 32 + i) =
              make_float4(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv,
                          __uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

bool prefill_fast_supported(int dtype_bf16, int d, int bs, int G) {
  return dtype_bf16 && d == 128 && bs == 16 && (G == 1 || G == 2 || G == 4 || G == 8);
}

static PFN_cuTensorMapEncodeTiled_v12000 q_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

cudaError_t launch_prefill_fast(const CUtensorMap* tmK, const CUtensorMap* tmV,
                                const PrefillArgs& a, int sms, cudaStream_t stream) {
  (void)sms;
  const int G = a.H / a.Hkv, TQ = 128 / G;
  // Q viewed as {head_dim, H, B * q_tokens}; one box = TQ tokens x G heads x 64
  CUtensorMap tmQ;
  auto fn = q_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {128, cuuint64_t(a.H), cuuint64_t(a.B) * a.q_tokens};
  const cuuint64_t strides[2] = {128 * 2, cuuint64_t(a.H) * 128 * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(G), cuuint32_t(TQ)};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (fn(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.q), dims, strides,
         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + kDataBytes + sizeof(PfBars);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((a.q_tokens + TQ - 1) / TQ, a.Hkv, a.B);
  prefill_tc_kernel<<<grid, kPfThreads, smem, stream>>>(tmQ, *tmK, *tmV, a,
                                                         a.scale * 1.4426950408889634f);
  return cudaGetLastError();
}

}  // namespace pa
