// Paged decode attention for bf16 K/V, head_dim 128, block_size 16, GQA
// group G <= 8: one CTA per (partition, KV head, sequence).
//
// What it computes ("docs.rs ferrum-kv 0.4.0 src/attention.rs",
// paged_attention with q_tokens = 1; "abhik.ai examples/pagedattention.py",
// Eq. 3): for the G query heads of KV head kvh,
//     o_h = sum_j softmax_j(q_h . k_j * scale) v_j,   j < kv_len,
// with k_j, v_j read through the block table, and the one-pass (m, l, acc)
// update of "semidirectx cmu11-667 lecture19 infer_world.py", section 3.
// With NP > 1 partitions each CTA covers part_blocks blocks and writes
// (m, l, o = acc / l) for a log-sum-exp combine.
//
// B200 design:
//  * one producer warp streams each 16-token block's K and V tiles
//    (4 KB each; two 64-column boxes per tile with the 128-byte swizzle)
//    from the pool into an NSTAGE ring with TMA (cp.async.bulk.tensor),
//    one full/empty mbarrier pair per stage; loads carry an L2 evict-first
//    hint because every byte is read exactly once;
//  * four consumer warps take blocks round-robin.  The G query heads of the
//    group share each K/V tile: S^T = K Q^T is one m16n8k16 tensor-core tile
//    per 16 d-columns (M = the block's 16 tokens, N = 8 heads), the softmax
//    statistics live in the accumulator fragment, P^T is turned into the B
//    operand of O^T += V^T P^T with movmatrix, and V^T comes from ldmatrix
//    .trans.  P is split into bf16 hi + lo parts so the product keeps ~16
//    mantissa bits (the PV error then stays at fp32-accumulation level);
//  * the four warps' partial (m, l, O) are merged through shared memory;
//  * when an unsplit grid spans several waves (many sequences of mixed
//    lengths), a one-CTA prepass orders the sequences longest-first so the
//    long ones do not form the tail.
// At G <= 8 the whole per-token arithmetic is 2 tensor-core tiles, so the
// loop stays bound by HBM rather than by the FP32 pipes (a CUDA-core dot
// product would need ~2 G FMA per byte-pair, near the B200's FP32 ridge at
// G = 8).
#include <math.h>

#include "common.cuh"
#include "device_once.hpp"
#include "launch.hpp"

namespace pa {

constexpr int kDecThreads = 160;  // 4 consumer warps + 1 producer warp
// Ring depth.  Block i of a CTA goes to consumer warp i % 4 and stage
// i % stages; with a multiple of 4 stages every stage belongs to one warp, so
// its rounds are waited on in order (a parity wait can only tell the current
// round from the previous one).  8 stages x 8 KB (64 KB) with 125 registers
// fit 3 CTAs per SM: 192 KB in flight per SM, and more resident CTAs to hide
// the per-CTA latency of short sequences (measured against 4 and 12 stages at
// 2 CTAs per SM: equal at 8K context, +5 % on the ragged batch, +2 % split-K).
constexpr int kRingStages = 8;
constexpr int kStageBytes = 8192;  // K tile 4 KB + V tile 4 KB
constexpr float kLog2eF = 1.4426950408889634f;

template <int kDecStages>
struct DecodeSmemTail {
  static_assert(kDecStages % 4 == 0, "stages must be a multiple of the 4 consumer warps");
  uint64_t full[kDecStages];
  uint64_t empty[kDecStages];
  int stage_bad[kDecStages];
  int any_bad;
};

template <int kDecStages>
__global__ void __launch_bounds__(kDecThreads, kDecStages <= 8 ? 3 : 2) decode_mma_kernel(
    const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const DecodeArgs p,
    float scale_log2) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  DecodeSmemTail<kDecStages>* tail =
      reinterpret_cast<DecodeSmemTail<kDecStages>*>(smem + kDecStages * kStageBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x, kvh = blockIdx.y;
  const int b = p.order ? p.order[blockIdx.z] : int(blockIdx.z);
  const int G = p.H / p.Hkv;
  const int kv_len = p.kv_lens[b];
  const bool len_bad = kv_len < 0 || kv_len > p.MB * 16;
  const int nblk_seq = len_bad ? 0 : (kv_len + 15) >> 4;
  // Sink + recent window (window > 0): key j is visible iff j < sinks or
  // j >= lo.  The CTAs walk the visible blocks only -- [0, sb) then [lb,
  // nblk_seq) -- numbered 0 .. nvis - 1; with no window it is every block.
  const int lo = (p.window > 0 && !len_bad) ? max(0, kv_len - p.window) : 0;
  const int sb = (min(p.sinks, kv_len) + 15) >> 4, lb = lo >> 4;
  const bool gap = lb > sb;
  const int nvis = gap ? sb + (nblk_seq - lb) : nblk_seq;
  auto vis_blk = [&](int v) { return (gap && v >= sb) ? lb + (v - sb) : v; };
  const int blk0 = part * p.part_blocks;
  const int nblk = max(0, min(blk0 + p.part_blocks, nvis) - blk0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
      tail->stage_bad[s] = 0;
    }
    tail->any_bad = len_bad ? 1 : 0;
    fence_barrier_init();
    if (len_bad && part == 0 && kvh == 0) raise_err(p.err, PA_DEVERR_KV_LEN);
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nblk > 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const uint64_t pol = policy_evict_first();
      const int32_t* trow = p.tables + int64_t(b) * p.MB;
      // Block ids in groups of 8, read one group ahead: an id read right
      // before its copies puts a table round trip on every block.
      auto load8 = [&](int base, int (&ids)[8]) {
#pragma unroll
        for (int u = 0; u < 8; ++u) ids[u] = base + u < nblk ? trow[vis_blk(blk0 + base + u)] : 0;
      };
      int cur[8], nxt[8];
      load8(0, cur);
      load8(8, nxt);
      int issued = 0;
      bool stop = false;
      for (int base = 0; base < nblk && !stop; base += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = base + u;
          if (i >= nblk) break;
          const int s = i % kDecStages, round = i / kDecStages;
          if (round > 0 && !mbar_wait(&tail->empty[s], (round - 1) & 1)) {
            raise_err(p.err, PA_DEVERR_TIMEOUT);
            stop = true;
            break;
          }
          const int blk = cur[u];
          if (blk < 0 || blk >= p.NB) {
            tail->stage_bad[s] = 1;
            tail->any_bad = 1;
            raise_err(p.err, PA_DEVERR_BLOCK_ID);
            mbar_arrive(&tail->full[s]);
          } else {
            tail->stage_bad[s] = 0;
            uint8_t* st = smem + s * kStageBytes;
            mbar_arrive_expect_tx(&tail->full[s], kStageBytes);
            tma_load_3d(st, &tmK, &tail->full[s], 0, kvh, blk * 16, pol);
            tma_load_3d(st + 2048, &tmK, &tail->full[s], 64, kvh, blk * 16, pol);
            tma_load_3d(st + 4096, &tmV, &tail->full[s], 0, kvh, blk * 16, pol);
            tma_load_3d(st + 6144, &tmV, &tail->full[s], 64, kvh, blk * 16, pol);
          }
          issued = i + 1;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) cur[u] = nxt[u];
        load8(base + 16, nxt);
      }
      // drain: no copy may still be landing in shared memory at exit
      for (int s = 0; s < kDecStages && s < issued; ++s) {
        const int count = (issued - 1 - s) / kDecStages + 1;
        mbar_wait(&tail->full[s], (count - 1) & 1);
      }
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  // Fused append: the CTA whose partition holds token kv_len-1 writes that
  // token's K/V row of its KV head into the pool (and patches it into the
  // staged tile below, so the TMA copy of the stale slot is never used).
  const bool appends = p.new_k != nullptr && nblk > 0 && blk0 + nblk == nvis;
  const int64_t new_slot = appends ? p.new_slots[b] : -1;
  if (appends && warp == 0) {
    if (new_slot >= int64_t(p.NB) * 16) {
      if (lane == 0) raise_err(p.err, PA_DEVERR_SLOT);
    } else if (new_slot >= 0) {
      const int64_t src = (int64_t(b) * p.Hkv + kvh) * 16;        // uint4 units
      const int64_t dst = (new_slot * p.Hkv + kvh) * 16;
      if (lane < 16)
        reinterpret_cast<uint4*>(p.k_cache)[dst + lane] =
            reinterpret_cast<const uint4*>(p.new_k)[src + lane];
      else
        reinterpret_cast<uint4*>(p.v_cache)[dst + lane - 16] =
            reinterpret_cast<const uint4*>(p.new_v)[src + lane - 16];
    }
  }
  const int g = lane >> 2, c = lane & 3;
  uint32_t qb[8][2];
  {
    const bool ok = g < G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        static_cast<const __nv_bfloat16*>(p.q) +
        (int64_t(b) * p.H + kvh * G + (ok ? g : 0)) * 128);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qb[kk][0] = ok ? __ldg(qrow + 8 * kk + c) : 0u;
      qb[kk][1] = ok ? __ldg(qrow + 8 * kk + 4 + c) : 0u;
    }
  }
  float o[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  // per-lane ldmatrix row/chunk pattern
  const int ld_row = (lane & 7) + ((lane >> 3) & 1) * 8;  // K: token row
  const int ld_khalf = lane >> 4;                          // K: +0/+1 chunk
  const int lv_tok = (lane & 7) + ((lane >> 4) << 3);      // V: token row
  const int lv_dc = (lane >> 3) & 1;                       // V: +0/+1 chunk
  const int tok_end = kv_len;

  for (int i = warp; i < nblk; i += 4) {
    const int s = i % kDecStages;
    const bool landed = __all_sync(0xffffffffu, mbar_wait(&tail->full[s], (i / kDecStages) & 1));
    if (!landed) {
      if (lane == 0) {
        raise_err(p.err, PA_DEVERR_TIMEOUT);
        tail->any_bad = 1;
      }
      break;
    }
    if (!tail->stage_bad[s]) {
      const uint32_t kb = smem_u32(smem + s * kStageBytes);
      const uint32_t vb = kb + 4096;
      const int tb = vis_blk(blk0 + i) * 16;
      const int valid = min(16, tok_end - tb);
      if (appends && new_slot >= 0 && new_slot < int64_t(p.NB) * 16 && tb == (nblk_seq - 1) * 16) {
        // the new token's row: 2 x 128 bytes in each of the K and V tiles
        const int row = valid - 1, ch = lane & 15;
        const uint4* src = reinterpret_cast<const uint4*>(lane < 16 ? p.new_k : p.new_v) +
                           (int64_t(b) * p.Hkv + kvh) * 16;
        uint8_t* tile = smem + s * kStageBytes + (lane < 16 ? 0 : 4096);
        *reinterpret_cast<uint4*>(tile + (ch >> 3) * 2048 + swz128(row, ch & 7)) = src[ch];
        fence_proxy_async_smem();  // a later TMA refill of this stage comes after it
        __syncwarp();
      }
      if (valid < 16) {
        // slots past the sequence end hold stale bytes (possibly NaN
        // patterns); zero their V rows so p = 0 contributes exactly 0
        uint4* vt = reinterpret_cast<uint4*>(smem + s * kStageBytes + 4096);
        for (int idx = lane; idx < (16 - valid) * 16; idx += 32) {
          const int row = valid + (idx >> 4), ch = idx & 15;
          vt[(ch >> 3) * 128 + row * 8 + (ch & 7)] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();  // order these writes before later TMA refills
        __syncwarp();
      }
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int ch = 2 * kk + ld_khalf;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(kb + (ch >> 3) * 2048 + swz128(ld_row, ch & 7), a0, a1, a2, a3);
        mma_bf16_16816(sc, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
      }
      float s0 = sc[0] * scale_log2, s1 = sc[1] * scale_log2;
      float s2 = sc[2] * scale_log2, s3 = sc[3] * scale_log2;
      // past the end, or outside the window
      auto hidden = [&](int t) { return t >= tok_end || (t < lo && t >= p.sinks); };
      if (hidden(tb + g)) s0 = s1 = -INFINITY;
      if (hidden(tb + g + 8)) s2 = s3 = -INFINITY;
      float x0 = fmaxf(s0, s2), x1 = fmaxf(s1, s3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
      }
      // every walked block holds a visible key, so x0 and x1 are finite here
      const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
      const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);
      const float p0 = exp2f(s0 - n0), p2 = exp2f(s2 - n0);
      const float p1 = exp2f(s1 - n1), p3 = exp2f(s3 - n1);
      l0 = l0 * al0 + (p0 + p2);
      l1 = l1 * al1 + (p1 + p3);
      m0 = n0;
      m1 = n1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        o[j][0] *= al0;
        o[j][1] *= al1;
        o[j][2] *= al0;
        o[j][3] *= al1;
      }
      // P^T as B fragments: hi part + lo remainder, both bf16
      const __nv_bfloat162 h01 = __floats2bfloat162_rn(p0, p1);
      const __nv_bfloat162 h23 = __floats2bfloat162_rn(p2, p3);
      const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
      const uint32_t hb0 = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h01));
      const uint32_t hb1 = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h23));
      const uint32_t lb0 = movmatrix_trans(pack_bf16x2(p0 - f01.x, p1 - f01.y));
      const uint32_t lb1 = movmatrix_trans(pack_bf16x2(p2 - f23.x, p3 - f23.y));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int ch = 2 * j + lv_dc;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(vb + (ch >> 3) * 2048 + swz128(lv_tok, ch & 7), a0, a1, a2, a3);
        mma_bf16_16816(o[j], a0, a1, a2, a3, hb0, hb1);
        mma_bf16_16816(o[j], a0, a1, a2, a3, lb0, lb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tail->empty[s]);
  }

  // ------------------------------------------- merge the four warps' states
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  named_bar_sync(1, 128);  // every consumer is done with the ring
  // [4 warps][8 heads][kORow] partial O; the row pitch of 132 floats puts the
  // four lanes c of a fragment column in four different bank octets
  constexpr int kORow = 132;
  float* so = reinterpret_cast<float*>(smem);
  float* sm = so + 4 * 8 * kORow;              // [4][8]
  float* sl = sm + 32;                         // [4][8]
  {
    float* w0 = so + (warp * 8 + 2 * c) * kORow;
    float* w1 = w0 + kORow;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      w0[16 * j + g] = o[j][0];
      w1[16 * j + g] = o[j][1];
      w0[16 * j + g + 8] = o[j][2];
      w1[16 * j + g + 8] = o[j][3];
    }
    if (g == 0) {
      sm[warp * 8 + 2 * c] = m0;
      sm[warp * 8 + 2 * c + 1] = m1;
      sl[warp * 8 + 2 * c] = l0;
      sl[warp * 8 + 2 * c + 1] = l1;
    }
  }
  named_bar_sync(1, 128);
  // per (warp, head): the weight 2^(m_w - M) / sum_w l_w 2^(m_w - M) of the
  // warp's partial O, worked out once by warp 0 (lane = warp w, head n)
  const bool zero = tail->any_bad != 0;
  float* swt = sl + 32;                        // [4][8]
  float* sM = swt + 32;                        // [8]
  float* sden = sM + 8;                        // [8]
  if (warp == 0) {
    const int n = lane & 7, w = lane >> 3;
    const float mw = sm[w * 8 + n];
    float M = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, 8));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));
    const float sc = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
    float den = sl[w * 8 + n] * sc;
    den += __shfl_xor_sync(0xffffffffu, den, 8);
    den += __shfl_xor_sync(0xffffffffu, den, 16);
    swt[w * 8 + n] = den > 0.f ? sc / den : 0.f;
    if (w == 0) {
      sM[n] = M;
      sden[n] = den;
    }
  }
  named_bar_sync(1, 128);
  const int t = threadIdx.x;  // d column
  for (int n = 0; n < G; ++n) {
    float val = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) val = fmaf(so[(w * 8 + n) * kORow + t], swt[w * 8 + n], val);
    if (zero || !(sden[n] > 0.f)) val = 0.f;
    const int64_t bh = int64_t(b) * p.H + kvh * G + n;
    if (p.NP == 1) {
      p.out[bh * 128 + t] = val;
    } else {
      const int64_t slot = bh * p.NP + part;
      float* ws_m = p.ws;
      float* ws_l = ws_m + int64_t(p.B) * p.H * p.NP;
      float* ws_o = ws_l + int64_t(p.B) * p.H * p.NP;
      ws_o[slot * 128 + t] = val;
      if (t == 0) {
        ws_m[slot] = sM[n];
        ws_l[slot] = zero ? -1.f : sden[n];  // -1 poisons the whole row
      }
    }
  }
}

// Log-sum-exp combine of the partitions: M = max_p m_p,
// w_p = l_p 2^(m_p - M), o = sum_p w_p o_p / sum_p w_p (m in log2 units).
__global__ void __launch_bounds__(128) decode_combine_kernel(
    const float* __restrict__ ws, int B, int H, int NP, float* __restrict__ out) {
  const int64_t bh = blockIdx.x;
  const float* ws_m = ws + bh * NP;
  const float* ws_l = ws + int64_t(B) * H * NP + bh * NP;
  const float* ws_o = ws + 2 * int64_t(B) * H * NP + bh * NP * 128;
  const int t = threadIdx.x;
  float M = -INFINITY;
  bool poison = false;
  for (int q = 0; q < NP; ++q) {
    M = fmaxf(M, ws_m[q]);
    poison |= ws_l[q] < 0.f;
  }
  float num = 0.f, den = 0.f;
  if (M != -INFINITY && !poison) {
    for (int q = 0; q < NP; ++q) {
      const float mq = ws_m[q];
      if (mq == -INFINITY) continue;
      const float w = ws_l[q] * exp2f(mq - M);
      num = fmaf(w, ws_o[q * 128 + t], num);
      den += w;
    }
  }
  out[bh * 128 + t] = den > 0.f ? num / den : 0.f;
}

// Longest-first order of the sequences (counting sort on the block count,
// descending; one CTA).  Launching long sequences first keeps them from
// forming the tail of a ragged batch; the result of each sequence does not
// depend on when its CTAs run.
constexpr int kOrderBuckets = 4096;
__global__ void __launch_bounds__(1024) decode_order_kernel(const int32_t* __restrict__ kv_lens,
                                                            int B, int32_t* __restrict__ order) {
  __shared__ int count[kOrderBuckets];
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int i = tid; i < kOrderBuckets; i += blockDim.x) count[i] = 0;
  __syncthreads();
  auto bucket = [&](int b) {
    const int L = kv_lens[b];
    const int nb = L > 0 ? (L + 15) >> 4 : 0;
    return kOrderBuckets - 1 - min(nb, kOrderBuckets - 1);   // descending
  };
  for (int b = tid; b < B; b += blockDim.x) atomicAdd(&count[bucket(b)], 1);
  __syncthreads();
  // exclusive prefix sum: each thread owns 4 consecutive buckets
  constexpr int kPer = kOrderBuckets / 1024;
  int local[kPer], run = 0;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    local[k] = run;
    run += count[tid * kPer + k];
  }
  int incl = run;                                  // inclusive scan across the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int t = warp_tot[lane], it = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, it, o);
      if (lane >= o) it += v;
    }
    warp_tot[lane] = it - t;                       // exclusive warp offsets
  }
  __syncthreads();
  const int base = warp_tot[wid] + incl - run;     // exclusive start of this thread
#pragma unroll
  for (int k = 0; k < kPer; ++k) count[tid * kPer + k] = base + local[k];
  __syncthreads();
  for (int b = tid; b < B; b += blockDim.x) order[atomicAdd(&count[bucket(b)], 1)] = b;
}

// Only unsplit grids of several waves are reordered: split grids already cut
// long sequences into partitions, one wave runs everything at once anyway.
bool decode_wants_order(int32_t B, int32_t Hkv, int32_t NP, int sms) {
  return NP == 1 && int64_t(B) * Hkv > 2 * int64_t(sms);
}

size_t order_workspace_bytes(int32_t B) { return sizeof(int32_t) * size_t(B); }

bool decode_fast_supported(int dtype_bf16, int d, int bs, int G) {
  return dtype_bf16 && d == 128 && bs == 16 && G >= 1 && G <= 8;
}

size_t split_workspace_bytes(int32_t B, int32_t H, int32_t NP, int32_t d) {
  if (NP <= 1) return 0;
  return sizeof(float) * size_t(B) * H * NP * (2 + size_t(d));
}

template <int NST>
static cudaError_t launch_ring(const CUtensorMap* tmK, const CUtensorMap* tmV,
                               const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = 1024 + NST * kStageBytes + sizeof(DecodeSmemTail<NST>);
  static PerDeviceOnce attr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = static_cast<cudaError_t>(attr.run(dev, [&] {
    return int(cudaFuncSetAttribute(decode_mma_kernel<NST>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
  }));
  if (e != cudaSuccess) return e;
  dim3 grid(a.NP, a.Hkv, a.B);
  decode_mma_kernel<NST><<<grid, kDecThreads, smem, stream>>>(*tmK, *tmV, a,
                                                              a.scale * kLog2eF);
  return cudaGetLastError();
}

cudaError_t launch_decode_order(const int32_t* kv_lens, int32_t B, int32_t* order,
                                cudaStream_t stream) {
  decode_order_kernel<<<1, 1024, 0, stream>>>(kv_lens, B, order);
  return cudaGetLastError();
}

cudaError_t launch_decode_combine(const float* ws, int32_t B, int32_t H, int32_t NP,
                                  float* out, cudaStream_t stream) {
  decode_combine_kernel<<<B * H, 128, 0, stream>>>(ws, B, H, NP, out);
  return cudaGetLastError();
}

cudaError_t launch_decode_fast(const CUtensorMap* tmK, const CUtensorMap* tmV,
                               const DecodeArgs& a, int sms,
                               cudaStream_t stream) {
  (void)sms;
  if (a.order) {
    cudaError_t eo = launch_decode_order(a.kv_lens, a.B, a.order, stream);
    if (eo != cudaSuccess) return eo;
  }
  cudaError_t e = launch_ring<kRingStages>(tmK, tmV, a, stream);
  if (e != cudaSuccess || a.NP == 1) return e;
  return launch_decode_combine(a.ws, a.B, a.H, a.NP, a.out, stream);
}

}  // namespace pa
