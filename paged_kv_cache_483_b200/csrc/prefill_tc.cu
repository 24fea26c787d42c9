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
// One CTA = two 128-row query tiles (A and B) of one (sequence, KV head).
// Rows are (token, head) pairs, 128/G tokens x G heads, so the G query heads
// that share a KV head share every K/V tile, and both tiles share each K/V
// tile fetched into shared memory.  Keys are visited in tiles of 128 (eight
// paged blocks, each fetched by TMA as two 64-column boxes with the 128-byte
// swizzle, landing in the UMMA K-major layout).
//   warp 0      TMA producer of Q_A, Q_B (once) and of the K ring (2 stages);
//   warp 2      TMA producer of the V ring (2 stages).  In each ring, lanes
//               0-7 issue the two boxes of one block each.
//   warp 1      one thread issues tcgen05.mma in the order
//                 ... PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1) ...
//               S_X = Q_X K^T lands in TMEM; O_X += P_X V reads P_X from TMEM
//               (the softmax writes it over S_X) and V from shared memory.
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B; one thread
//               per row = TMEM lane.  While one tile's softmax runs on the
//               CUDA cores the tensor core works on the other tile.
// TMEM (512 columns): S_A/P_A [0,128), S_B/P_B [128,256), O_A, O_B.
// The tensor core executes one CTA's MMAs in issue order, so when QK_X(j) has
// completed, PV_X(j-1) has too: the softmax may then rescale O_X in TMEM.  O
// is rescaled only when a row's max grows by more than 2^8 (a stale max below
// that keeps every exponent <= 2^8, exact in fp32).  P is rounded to bf16.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "device_once.hpp"
#include "launch.hpp"
#include "tcgen05.cuh"

namespace pa {

namespace {

constexpr int kPfThreads = 384;      // 3 warpgroups: control, softmax A, softmax B
constexpr int kCtrlRegs = 64;        // 128 x 64 + 256 x 216 <= 384 x 168 at launch
constexpr int kSoftmaxRegs = 216;
constexpr int kKStages = 2;         // K ring (tiles)
constexpr int kVStages = 2;         // V ring (tiles)
constexpr uint32_t kTile = 32768;  // 128 x 128 bf16
constexpr uint32_t kHalf = 16384;  // 128 x 64 bf16 (one 128-byte-swizzled half)
constexpr uint32_t kOffQ = 0;      // Q_A, then Q_B
constexpr uint32_t kOffK = 2 * kTile;
constexpr uint32_t kOffV = (2 + kKStages) * kTile;
constexpr uint32_t kDataBytes = (2 + kKStages + kVStages) * kTile;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr float kRescaleTau = 8.0f;
constexpr int kMaxSplit = 4;         // parts per split unit at most
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);

struct PfBars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_final;
  uint32_t tmem_base;
  int abort;
  int bad_vote[2][4];
  int ticket[2];
};

// Work decomposition.  A unit is one CTA's query tile pair of one (sequence,
// KV head); units are numbered with the query tile fastest.  Units below
// first_split run whole; each unit from first_split on is split into k parts
// over its key tiles (one CTA per part) whose partial results are merged by
// the part that finishes last.
struct PfPlan {
  int nq;           // query tile pairs per (sequence, KV head)
  int first_split;  // first unit that is split
  int k;            // parts per split unit (1 = none)
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              PfBars* bars, int32_t* err) {
  if (mbar_wait(bar, parity)) return true;
  raise_err(err, PA_DEVERR_TIMEOUT);
  atomicExch(&bars->abort, 1);
  return false;
}

// Warp-uniform wait used by the softmax warps (tcgen05.ld/st are collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, PfBars* bars,
                                          int32_t* err, int lane) {
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, parity));
  if (!ok && lane == 0) {
    raise_err(err, PA_DEVERR_TIMEOUT);
    atomicExch(&bars->abort, 1);
  }
  return ok;
}

}  // namespace

__global__ void __launch_bounds__(kPfThreads, 1) prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
    const PrefillArgs p, const PfPlan pl, float scale_log2, int use_tma_store) {
  extern __shared__ uint8_t pf_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(pf_raw) + 1023) & ~uintptr_t(1023));
  PfBars* bars = reinterpret_cast<PfBars*>(smem + kDataBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.H / p.Hkv, TQ = 128 / G;
  int u = blockIdx.x, part = 0;
  if (u >= pl.first_split) {
    const int t = u - pl.first_split;
    u = pl.first_split + t / pl.k;
    part = t % pl.k;
  }
  const int split_k = u >= pl.first_split ? pl.k : 1;
  const int xq = u % pl.nq, kvh = (u / pl.nq) % p.Hkv, b = u / (pl.nq * p.Hkv);
  const int t0 = xq * 2 * TQ;                         // first token of tile A
  const int q_tokens = p.q_tokens;
  const int kv_len = p.kv_lens[b];
  const int valid_tokens = min(2 * TQ, q_tokens - t0);  // of both tiles
  const bool len_bad = kv_len < q_tokens || kv_len > p.MB * 16;
  const int qpos0 = kv_len - q_tokens + t0;           // key limit of token t0
  const int key_end = len_bad ? 0 : qpos0 + valid_tokens;
  const int n_all = (key_end + 127) >> 7;             // key tiles of the unit
  const int j0 = part * n_all / split_k;              // this part: [j0, j0 + n_tiles)
  const int n_tiles = (part + 1) * n_all / split_k - j0;
  const int n_blk = (key_end + 15) >> 4;
  const int32_t* trow = p.tables + int64_t(b) * p.MB;

  if (threadIdx.x == 0 && len_bad && xq == 0 && kvh == 0 && part == 0)
    raise_err(p.err, PA_DEVERR_KV_LEN);
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 128);
    }
    mbar_init(&bars->o_final, 1);
    bars->abort = 0;
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

  if (warp < 4) {
  regs_dealloc<kCtrlRegs>();
  if (warp == 0 || warp == 2) {
    // ------------------------------------- TMA producers: Q and K (warp 0), V (warp 2)
    // Two warps issue the copies, eight lanes each (lane i copies block i of
    // a tile): one thread's TMA issue rate does not keep up with the K and V
    // tiles of both query tiles.
    const bool is_k = warp == 0;
    if (n_tiles > 0) {
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      if (lane == 0) prefetch_tensormap(map);
      const uint64_t pol_kv = policy_evict_last();
      if (is_k && lane == 0) {
        prefetch_tensormap(&tmQ);
        const uint64_t pol_q = policy_evict_first();
        mbar_arrive_expect_tx(&bars->q_full, 2 * kTile);
        for (int x = 0; x < 2; ++x) {
          const int z = b * q_tokens + t0 + x * TQ;
          tma_load_3d(smem + kOffQ + x * kTile, &tmQ, &bars->q_full, 0, kvh * G, z, pol_q);
          tma_load_3d(smem + kOffQ + x * kTile + kHalf, &tmQ, &bars->q_full, 64, kvh * G, z,
                      pol_q);
        }
      }
      // This lane's block id of a tile, read one tile ahead of its use: the
      // TMA issues are ordered with every memory access, so an id read next
      // to its copy would cost one global-memory round trip per block.
      auto tile_id = [&](int j) {
        const int nb = min(8, n_blk - (j0 + j) * 8);
        const int blk = lane < nb ? trow[(j0 + j) * 8 + lane] : 0;
        return (blk < 0 || blk >= p.NB) ? 0 : blk;   // reported and zeroed by the softmax
      };
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      uint8_t* ring = smem + (is_k ? kOffK : kOffV);
      const int stages = is_k ? kKStages : kVStages;
      int id = tile_id(0);
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % stages, round = j / stages;
        bool go = true;
        if (lane == 0)
          go = (round == 0 || wait_or_abort(&empty[s], (round - 1) & 1, bars, p.err)) &&
               !bars->abort;
        if (!__shfl_sync(0xffffffffu, go ? 1 : 0, 0)) break;
        uint8_t* dst = ring + s * kTile;
        const int nb = min(8, n_blk - (j0 + j) * 8);
        if (lane == 0) mbar_arrive_expect_tx(&full[s], nb * 4096);
        __syncwarp();                                  // the bytes are expected first
        if (lane < nb) {
          tma_load_3d(dst + lane * 2048, map, &full[s], 0, kvh, id * 16, pol_kv);
          tma_load_3d(dst + kHalf + lane * 2048, map, &full[s], 64, kvh, id * 16, pol_kv);
        }
        issued = j + 1;
        if (j + 1 < n_tiles) id = tile_id(j + 1);
      }
      // drain: every issued copy has landed before the CTA may exit
      if (lane == 0) {
        if (is_k) mbar_wait(&bars->q_full, 0);
        for (int s = 0; s < stages; ++s)
          if (s < issued) mbar_wait(&full[s], ((issued - 1 - s) / stages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // Descriptors of Q_A, Q_B and of each K and V stage: their high words
      // are constants and their low words differ by fixed offsets, so each
      // MMA needs one add.  This thread shares its issue slots with two
      // softmax warps, and every instruction here delays the next MMA.
      static_assert(kKStages == 2 && kVStages == 2, "two K and two V stages");
      const uint64_t dq0 = desc_kmajor_sw128(smem_u32(smem + kOffQ));
      const uint64_t dv0 = desc_mnmajor_sw128(smem_u32(smem + kOffV), kHalf, 1024);
      const uint32_t hk = uint32_t(dq0 >> 32), hv = uint32_t(dv0 >> 32);
      const uint32_t lq = uint32_t(dq0), lv = uint32_t(dv0);
      const uint32_t lk = lq + ((kOffK - kOffQ) >> 4);
      auto mk = [](uint32_t lo, uint32_t hi) { return (uint64_t(hi) << 32) | lo; };
      auto qk = [&](int x, int j) {                    // S_x = Q_x K(j)^T
        const uint32_t kl = lk + (j & 1) * (kTile >> 4), ql = lq + x * (kTile >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          umma_bf16(tbase + kColS + x * 128, mk(ql + off, hk), mk(kl + off, hk), kIdescQK,
                    kk > 0);
        }
        umma_commit(&bars->s_full[x]);
      };
      auto pv = [&](int x, int j) {                    // O_x += P_x V(j)
        const uint32_t vl = lv + (j & 1) * (kTile >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_tmem_a(tbase + kColO + x * 128, tbase + kColS + x * 128 + kk * 8,
                           mk(vl + kk * (2048 >> 4), hv), kIdescPV,
                           (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = n_tiles > 0 && wait_or_abort(&bars->q_full, 0, bars, p.err) &&
                wait_or_abort(&bars->k_full[0], 0, bars, p.err);
      if (ok) {
        tc_fence_after();
        qk(0, 0);
        qk(1, 0);
        umma_commit(&bars->k_empty[0]);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kVStages;
        const bool more = j + 1 < n_tiles;
        ok = wait_or_abort(&bars->v_full[s], (j / kVStages) & 1, bars, p.err) &&
             wait_or_abort(&bars->p_full[0], j & 1, bars, p.err);
        if (!ok || bars->abort) break;
        tc_fence_after();
        pv(0, j);
        if (more) {
          const int s1 = (j + 1) % kKStages;
          ok = wait_or_abort(&bars->k_full[s1], ((j + 1) / kKStages) & 1, bars, p.err);
          if (!ok) break;
          tc_fence_after();
          qk(0, j + 1);
        }
        ok = wait_or_abort(&bars->p_full[1], j & 1, bars, p.err);
        if (!ok || bars->abort) break;
        tc_fence_after();
        pv(1, j);
        umma_commit(&bars->v_empty[s]);
        if (more) {
          qk(1, j + 1);
          umma_commit(&bars->k_empty[(j + 1) % kKStages]);
        }
      }
      if (n_tiles > 0) umma_commit(&bars->o_final);
    }
  }
  } else {
    // ------------------------------------------------ softmax / epilogue
    regs_alloc<kSoftmaxRegs>();
    const int x = (warp - 4) >> 2;                     // query tile A (0) or B (1)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // row = TMEM lane
    const int t_local = r / G, g = r % G;
    const int tok = t0 + x * TQ + t_local;             // query token of this row
    const bool row_valid = tok < q_tokens;
    const int qpos = kv_len - q_tokens + tok;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t s_addr = tbase + lane_off + kColS + x * 128;
    const uint32_t o_addr = tbase + lane_off + kColO + x * 128;
    // every block id the CTA touches must be inside the pool (checked here,
    // while the first QK^T is still running)
    bool bad_blk = false;
    const int blk_end = min(n_blk, (j0 + n_tiles) * 8);
    for (int i = j0 * 8 + r; i < blk_end; i += 128) {
      const int blk = trow[i];
      bad_blk |= (blk < 0 || blk >= p.NB);
    }
    bad_blk = __any_sync(0xffffffffu, bad_blk);
    if (lane == 0) bars->bad_vote[x][quarter] = bad_blk ? 1 : 0;
    named_bar_sync(1 + x, 128);
    bad_blk = (bars->bad_vote[x][0] | bars->bad_vote[x][1] | bars->bad_vote[x][2] |
               bars->bad_vote[x][3]) != 0;
    if (bad_blk && r == 0 && x == 0) raise_err(p.err, PA_DEVERR_BLOCK_ID);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = warp_wait(&bars->s_full[x], j & 1, bars, p.err, lane);
      if (!ok) break;
      tc_fence_after();
      float s[128];
      {
        uint32_t v[128];
        tmem_ld128(s_addr, v);
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(v[i]);
      }
      const int lim = qpos - (j0 + j) * 128;           // columns c <= lim are visible
      if (lim < 127) {
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = (c <= lim) ? s[c] : -INFINITY;
      }
      const float2 sl2 = make_float2(scale_log2, scale_log2);
      // P = 2^(s*scale - m_ref) as bf16 pairs over the first 64 columns of S;
      // returns the row sum of this tile's P
      auto write_p = [&](float mref) -> float {
        float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 nm2 = make_float2(-mref, -mref);
#pragma unroll
        for (int hcol = 0; hcol < 2; ++hcol) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 e = __ffma2_rn(
                make_float2(s[hcol * 64 + 2 * i], s[hcol * 64 + 2 * i + 1]), sl2, nm2);
            const float2 pp = make_float2(ex2(e.x), ex2(e.y));
            sum2[i & 1] = __fadd2_rn(sum2[i & 1], pp);
            w[i] = pack_bf16x2(pp.x, pp.y);
          }
          tmem_st32(s_addr + hcol * 32, w);
        }
        return (sum2[0].x + sum2[1].x) + (sum2[0].y + sum2[1].y);
      };
      auto row_max = [&]() -> float {
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(s[i], s[i + 8]);
#pragma unroll
        for (int c = 16; c < 128; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mx8[i] = max3(mx8[i], s[c + i], s[c + 8 + i]);
        return max3(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5]),
                    fmaxf(mx8[6], mx8[7])) * scale_log2;
      };
      auto rescale_o = [&](float alpha) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(o_addr + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tmem_st32(o_addr + c * 32, v);
        }
      };
      // PV_x(j-1) has completed (it precedes QK_x(j) on the tensor core), so
      // O_x may be rescaled here.
      float tile_sum;
      if (!__any_sync(0xffffffffu, m_ref == -INFINITY)) {
        // Speculative: exponentiate against the current reference max while
        // the row max is formed in the same pass; only a row whose max grew
        // by more than 2^8 makes the warp rescale O and redo P.
        tile_sum = write_p(m_ref);
        const float mt = row_max();
        const bool grow = mt > m_ref + kRescaleTau;
        if (__any_sync(0xffffffffu, grow)) {
          const float alpha = grow ? ex2(m_ref - mt) : 1.f;
          if (grow) m_ref = mt;
          rescale_o(alpha);
          l *= alpha;
          tile_sum = write_p(m_ref);
        }
      } else {
        // a row without a visible key so far: its reference max comes first
        const float mt = row_max();
        float alpha = 1.f;
        bool grow = false;
        if (mt != -INFINITY) {
          if (m_ref == -INFINITY) {
            alpha = 0.f;
            m_ref = mt;
          } else if (mt > m_ref + kRescaleTau) {
            alpha = ex2(m_ref - mt);
            m_ref = mt;
            grow = true;
          }
        }
        if (__any_sync(0xffffffffu, grow)) rescale_o(alpha);
        l *= alpha;
        tile_sum = write_p(m_ref == -INFINITY ? 0.f : m_ref);
      }
      if (x == 0 && j0 + j == n_all - 1) {
        // V rows at or past key_end hold stale bytes: zero them (p = 0 there,
        // and 0 x NaN would poison the product); PV_B follows PV_A
        const int st = j % kVStages;
        const bool landed = warp_wait(&bars->v_full[st], (j / kVStages) & 1, bars, p.err, lane);
        if (landed && (j0 + j) * 128 + r >= key_end) {
          uint4* v0 = reinterpret_cast<uint4*>(smem + kOffV + st * kTile + r * 128);
          uint4* v1 = reinterpret_cast<uint4*>(smem + kOffV + st * kTile + kHalf + r * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            v0[c] = make_uint4(0u, 0u, 0u, 0u);
            v1[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
      }
      l += tile_sum;
      tc_fence_before();
      mbar_arrive(&bars->p_full[x]);
    }
    // ------------------------------------------------------------ epilogue
    // o_final: every MMA of the CTA has completed, so TMEM and the whole
    // shared memory may be reused.  Rows of a part that found an error are
    // zeros (not O * 0: O may hold non-finite values or was never written).
    const bool fin_ok = ok && (n_tiles == 0 || warp_wait(&bars->o_final, 0, bars, p.err, lane));
    tc_fence_after();
    const bool part_err = !fin_ok || bad_blk;
    const bool have = !part_err && n_tiles > 0 && l > 0.f;
    const float inv = have ? 1.f / l : 0.f;
    // this part's O / l, columns [32c, 32c + 32)
    auto own_chunk = [&](int c, float (&o)[32]) {
      uint32_t v[32];
      tmem_ld32(o_addr + c * 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = have ? __uint_as_float(v[i]) * inv : 0.f;
    };
    // write the tile's final rows
    auto emit = [&](auto&& chunk) {
      if (use_tma_store && valid_tokens == 2 * TQ) {
        // Both tiles are full: each row goes into four 32-column boxes with
        // the 128-byte swizzle (conflict-free), then one thread per tile
        // stores them with TMA.
        uint8_t* stage = smem + x * 65536;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          chunk(c, o);
          uint8_t* box = stage + c * 16384;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<float4*>(box + swz128(r, q4)) =
                make_float4(o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2], o[4 * q4 + 3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + x, 128);
        if (r == 0) {
          const int z = b * q_tokens + t0 + x * TQ;
          for (int c = 0; c < 4; ++c) tma_store_3d(&tmO, stage + c * 16384, c * 32, kvh * G, z);
          bulk_commit();
          bulk_wait_read_all();
        }
      } else {
        float* orow = p.out + ((int64_t(b) * q_tokens + tok) * p.H + kvh * G + g) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          chunk(c, o);
          if (row_valid) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(orow + c * 32 + i) =
                  make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
          }
        }
      }
    };
    if (split_k == 1) {
      emit(own_chunk);
    } else {
      // A part of a split unit publishes its normalised O rows and (m, l) --
      // l < 0 marks a part that failed -- then takes a ticket; the part that
      // takes the last ticket merges all parts with the log-sum-exp rule:
      // out = sum_q w_q O_q / l_q, w_q = l_q 2^(m_q - M) / sum_q' l_q' 2^(m_q' - M).
      const int us = u - pl.first_split;
      const int64_t slot0 = int64_t(us) * split_k;
      // a part's O tile is stored as [32 column quads][128 rows][4]: a warp
      // moves 512 contiguous bytes per access
      auto part_o = [&](int q) {
        return reinterpret_cast<float4*>(p.split_o + ((slot0 + q) * 2 + x) * (128 * 128)) + r;
      };
      auto part_ml = [&](int q) {
        return reinterpret_cast<float2*>(p.split_ml) + ((slot0 + q) * 2 + x) * 128 + r;
      };
      {
        float4* dst = part_o(part);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          own_chunk(c, o);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[(c * 8 + i) * 128] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
        *part_ml(part) = make_float2(m_ref, part_err ? -1.f : (have ? l : 0.f));
      }
      __threadfence();
      named_bar_sync(1 + x, 128);
      if (r == 0) {
        int32_t* tk = p.tickets + us * 2 + x;
        const int t = atomicAdd(tk, 1);
        if (t == split_k - 1) *tk = 0;                 // every part is in: reset
        bars->ticket[x] = t;
        __threadfence();
      }
      named_bar_sync(1 + x, 128);
      if (bars->ticket[x] == split_k - 1) {
        float w[kMaxSplit], mq[kMaxSplit];
        float M = -INFINITY, L = 0.f;
        bool failed = false;
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q) {
          const float2 ml = q < split_k ? __ldcg(part_ml(q)) : make_float2(0.f, 0.f);
          failed |= ml.y < 0.f;
          w[q] = fmaxf(ml.y, 0.f);                     // l_q; 2^(m_q - M) below
          mq[q] = ml.x;
          if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q) {
          w[q] = w[q] > 0.f ? w[q] * ex2(mq[q] - M) : 0.f;
          L += w[q];
        }
        const float invL = (!failed && L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
        for (int q = 0; q < kMaxSplit; ++q) w[q] *= invL;
        emit([&](int c, float (&o)[32]) {
          // every part's loads first (one round trip to L2 per chunk)
          float4 v[kMaxSplit][8];
#pragma unroll
          for (int q = 0; q < kMaxSplit; ++q) {
            if (q < split_k) {
              const float4* src = part_o(q);
#pragma unroll
              for (int i = 0; i < 8; ++i) v[q][i] = __ldcg(src + (c * 8 + i) * 128);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
#pragma unroll
          for (int q = 0; q < kMaxSplit; ++q) {
            if (q < split_k && w[q] != 0.f) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                o[4 * i] = fmaf(w[q], v[q][i].x, o[4 * i]);
                o[4 * i + 1] = fmaf(w[q], v[q][i].y, o[4 * i + 1]);
                o[4 * i + 2] = fmaf(w[q], v[q][i].z, o[4 * i + 2]);
                o[4 * i + 3] = fmaf(w[q], v[q][i].w, o[4 * i + 3]);
              }
            }
          }
        });
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

cudaError_t launch_prefill_fast(const CUtensorMap* tmK, const CUtensorMap* tmV,
                                const PrefillArgs& a, int sms, cudaStream_t stream) {
  const int G = a.H / a.Hkv, TQ = 128 / G;
  // Q viewed as {head_dim, H, B * q_tokens}; one box = TQ tokens x G heads x 64
  CUtensorMap tmQ;
  auto fn = tensor_map_encoder();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {128, cuuint64_t(a.H), cuuint64_t(a.B) * a.q_tokens};
  const cuuint64_t strides[2] = {128 * 2, cuuint64_t(a.H) * 128 * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(G), cuuint32_t(TQ)};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (fn(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.q), dims, strides,
         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // O viewed as {head_dim, H, B * q_tokens} fp32; one box = 32 columns of
  // the tile's rows, 128-byte swizzle
  CUtensorMap tmO;
  int use_tma_store = 0;
  {
    const cuuint64_t odims[3] = {128, cuuint64_t(a.H), cuuint64_t(a.B) * a.q_tokens};
    const cuuint64_t ostr[2] = {128 * 4, cuuint64_t(a.H) * 128 * 4};
    const cuuint32_t obox[3] = {32, cuuint32_t(G), cuuint32_t(TQ)};
    if ((reinterpret_cast<uintptr_t>(a.out) & 15) == 0 &&
        fn(&tmO, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.out, odims, ostr, obox, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      use_tma_store = 1;
    else
      tmO = tmQ;   // never used
  }
  const size_t smem = 1024 + kDataBytes + sizeof(PfBars);
  static PerDeviceOnce attr;
  int dev = 0;
  cudaError_t ea = cudaGetDevice(&dev);
  if (ea != cudaSuccess) return ea;
  ea = static_cast<cudaError_t>(attr.run(dev, [&] {
    return int(cudaFuncSetAttribute(prefill_tc_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
  }));
  if (ea != cudaSuccess) return ea;
  PfPlan pl;
  pl.nq = (a.q_tokens + 2 * TQ - 1) / (2 * TQ);
  const int64_t units = int64_t(pl.nq) * a.Hkv * a.B;
  if (units > (int64_t(1) << 30)) return cudaErrorInvalidValue;
  pl.first_split = int(units);
  pl.k = 1;
  // The units of the last, partial wave (one CTA per SM) are split over
  // their keys so that the wave fills the GPU: k parts each, k * tail <= SMs.
  if (a.split_o && a.split_ml && a.tickets && a.max_splits != 1 && sms > 0) {
    const int64_t tail = units % sms;
    if (tail > 0) {
      int64_t k = sms / tail;
      k = std::min<int64_t>(k, a.max_splits > 1 ? std::min(a.max_splits, kMaxSplit) : kMaxSplit);
      if (k >= 2 && tail * k <= a.split_slots) {
        pl.first_split = int(units - tail);
        pl.k = int(k);
      }
    }
  }
  const int64_t ctas = pl.first_split + (units - pl.first_split) * pl.k;
  prefill_tc_kernel<<<unsigned(ctas), kPfThreads, smem, stream>>>(
      tmQ, *tmK, *tmV, tmO, a, pl, a.scale * 1.4426950408889634f, use_tma_store);
  return cudaGetLastError();
}

}  // namespace pa
