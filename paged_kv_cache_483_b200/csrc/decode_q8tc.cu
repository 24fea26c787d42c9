// Paged decode attention over an int8 or FP8 (E4M3) KV pool on the 5th-
// generation tensor cores: head_dim 128, block_size 16, GQA group G <= 4.
// One CTA per (partition, KV head, sequence).
//
// What it computes: the decode of "docs.rs ferrum-kv 0.4.0 src/attention.rs"
// (paged_attention, q_tokens = 1) on the K/V rows the pool holds, k_j =
// value(code_k[j]) * scale_k[j], v_j = value(code_v[j]) * scale_v[j] (the
// per-row absmax quantisation of "vladkulikov.com modern-llms module 9
// notebook", KV quantisation experiment, on the int8 grid or the E4M3 grid),
// with the one-pass (m, l, acc) update of "semidirectx cmu11-667 lecture19
// infer_world.py", section 3, taken over groups of 128 keys.
//
// B200 design.  The pool keeps one 4224-byte record per (block, head): K codes
// [16 tokens][128] with token t's 16-byte chunks pre-swizzled (chunk c at
// c ^ (t & 7)), V codes [128 d][16 tokens], 16 K scales, 16 V scales.  Work
// goes in groups of eight blocks (128 keys):
//  * warp 0 copies each block with two TMA boxes (lane i of the warp copies
//    block i of a group: one thread's copy-issue rate is too low for two
//    boxes per block): the K codes (16 rows of 128 B) into the group's K
//    tile, where eight blocks' K rows form one
//    128 x 128 operand in the 128-byte-swizzle K-major layout (the record's
//    own swizzle is that layout), and the V codes + scales (17 rows) into the
//    group's V tile, where block b's V rows sit 2176 B after block b - 1:
//    V^T [128 d x 128 keys] is a K-major operand without swizzle, core
//    matrices of 8 d-rows x 16 keys, 128 B apart along d and 2176 B along keys;
//  * warp 1 issues tcgen05.mma (kind::f8f6f4 for E4M3, kind::i8 for int8):
//    S^T[128 keys x N] = K Q~^T and, once the softmax has written P~,
//    O_g^T[128 d x N] = V^T P~^T, both straight from the codes in shared
//    memory, fp32 (s32) accumulators in tensor memory;
//  * two softmax warpgroups take alternate groups (one thread per key of the
//    group, and per d row in the fold): each reads S, forms the scores, takes
//    the group's max per head (warp max, then across its four warps through
//    shared memory), writes P, and folds the group's O_g into fp32 registers:
//    o = o * alpha + O_g * unit, alpha = 2^(m_old - m_new) -- the exact
//    online-softmax recurrence, no stale maximum, no rescale of tensor
//    memory; the two warpgroups' (m, l, o) are merged at the end;
//  * K tiles (two) are handed back when their QK completes, V tiles (four)
//    when their PV does; S, P and O have four buffers each, so QK runs up to
//    three groups ahead of the softmax.
// Groups of more than 4 heads go to the warp-level kernel (decode_q8.cu):
// the per-byte softmax work here grows with the group, while its 8-column
// MMA tiles are full at G = 8.
// Q and P enter the 8-bit MMA as sums of 8-bit terms (columns n = term * Gp +
// head of the B operands, Gp = G rounded up to a power of two):
//  * FP8: Q / sq (sq a power of two with max |Q / sq| <= 448) as three E4M3
//    terms q1 + q2 / 16 + q3 / 256, each the E4M3 rounding of the remainder of
//    the previous ones times 16 (relative error ~2^-12); P as three E4M3 terms
//    of 256 p scale_v / U, U the group's power-of-two V unit (> every live V
//    scale of the group), so the V dequantisation is folded into P;
//  * int8: Q / sq (sq = max|Q| / 127) as hi + lo / 254 (both int8, error <=
//    sq / 508 per element); P as 127 p scale_v / U = p1 + p2 / 254 (both
//    int8).  Per group the s32 sums stay far below 2^31.
// Slots past a sequence's end and blocks that are missing or out of range
// hold stale bytes; their scores are replaced by -inf and their p by 0, and
// for FP8 (whose codes include NaN) their V bytes are zeroed before PV.
#include <math.h>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "device_once.hpp"
#include "launch.hpp"
#include "tcgen05.cuh"

namespace pa {

namespace {

// Threads: a producer warp, an MMA warp and two softmax warpgroups that take
// alternate groups.
constexpr int kWG = 2;
constexpr int kGroupBlocks = 8;          // 128 keys per group = the MMA's M
constexpr uint32_t kKTile = kGroupBlocks * 2048;       // K codes of a group
constexpr uint32_t kVSlot = 2176;                     // one block's V codes + scales
constexpr uint32_t kVTile = kGroupBlocks * kVSlot;    // 17408
constexpr int kKStages = 2;              // K tiles: free again once their QK is done
constexpr int kMaxVStages = 4;           // V tiles: free again once their PV is done
constexpr int kBufs = 4;                 // S, P and O buffers (QK runs up to 3 groups ahead)
constexpr uint32_t kTmemCols = 256;      // S x 4, O x 4, 32 columns each
constexpr float kLog2e = 1.4426950408889634f;

struct TcTail {
  uint64_t kfull[kKStages], kempty[kKStages];
  uint64_t vfull[kMaxVStages], vempty[kMaxVStages];
  uint64_t s_full[kBufs], p_full[kBufs], o_full[kBufs];
  uint64_t q_ready;
  uint32_t tmem_base;
  int badmask[kMaxVStages];  // per V stage: bit i = block i of the group missing or unusable
  int any_bad;
  int abort;
  float qs[8];         // per head: sq * scale_log2
  float red[2][2][4][10];  // per iteration parity, warpgroup, warp: head maxima, V-scale max, ok
};

// Columns of the B operands (Q~ and P~): T terms of kGp heads, padded to the
// MMA's multiple of 16.
__host__ __device__ constexpr int q8tc_cols(bool fp8, int gp) {
  return ((gp * (fp8 ? 3 : 2) + 15) / 16) * 16;
}


// Shared-memory layout of a CTA for N columns (a multiple of 16) and vst V
// stages: K tiles [2][128 keys x 128 B] | V tiles [vst][8 blocks x 2176 B] |
// Q terms (N rows of 128 B, swizzled) | P terms x 4 (N rows of 128 keys, core
// matrices) | tail.
__host__ __device__ constexpr uint32_t v_off() { return uint32_t(kKStages) * kKTile; }
__host__ __device__ constexpr uint32_t q_off(int vst) { return v_off() + uint32_t(vst) * kVTile; }
__host__ __device__ constexpr uint32_t p_off(int vst, int N) { return q_off(vst) + uint32_t(N) * 128; }
__host__ __device__ constexpr uint32_t tail_off(int vst, int N) {
  return p_off(vst, N) + uint32_t(kBufs) * uint32_t(N / 8) * 1024u;
}

// 128-byte-swizzle-free K-major descriptor: core matrices of 8 rows x 16 B,
// lbo = byte step between core matrices along K, sbo = along M/N.
__device__ __forceinline__ uint64_t desc_kmajor_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t(lbo >> 4) << 16) |
         (uint64_t(sbo >> 4) << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor of an 8-bit MMA, M = 128, N columns, both operands
// K-major: FP8 = E4M3 x E4M3 -> f32, int8 = s8 x s8 -> s32.
__host__ __device__ constexpr uint32_t idesc_8bit(bool fp8, int N) {
  return (fp8 ? (1u << 4) : ((2u << 4) | (1u << 7) | (1u << 10))) |
         (uint32_t(N >> 3) << 17) | (uint32_t(128 >> 4) << 24);
}

template <bool kFp8>
__device__ __forceinline__ void umma_8bit(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  if constexpr (kFp8)
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Maximum over the warp (redux.sync on f32, sm_100a).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// E4M3 code of x (nearest, ties to even, saturating at +-448) and its value.
__device__ __forceinline__ uint32_t e4m3_of(float x) {
  return uint32_t(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}
__device__ __forceinline__ float e4m3_val(uint32_t c) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3)));
}

// Splits x into 8-bit terms (codes, low byte each): FP8 x ~ t0 + t1 / 16 +
// t2 / 256 (E4M3); int8 x ~ t0 + t1 / 254 (x in [-127.5, 127.5]).
template <bool kFp8>
__device__ __forceinline__ void split_terms(float x, uint32_t (&t)[3]) {
  if constexpr (kFp8) {
    t[0] = e4m3_of(x);
    const float r1 = (x - e4m3_val(t[0])) * 16.f;
    t[1] = e4m3_of(r1);
    const float r2 = (r1 - e4m3_val(t[1])) * 16.f;
    t[2] = e4m3_of(r2);
  } else {
    const float hi = rintf(fminf(fmaxf(x, -127.f), 127.f));
    t[0] = uint32_t(int32_t(hi)) & 0xFFu;
    t[1] = uint32_t(int32_t(rintf((x - hi) * 254.f))) & 0xFFu;
    t[2] = 0u;
  }
}

// N (16 or 32) consecutive 32-bit columns of this thread's TMEM lane.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 16)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
  else
    tmem_ld32(taddr, r);
}

// Columns [c, c + 4) of each of T terms (term k at column addr + k * stride)
// of this thread's TMEM lane, then one wait for all of them.
template <int T>
__device__ __forceinline__ void tmem_ld_terms(uint32_t addr, uint32_t stride,
                                              uint32_t (&r)[3][4]) {
  if constexpr (T == 3)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%12];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4,%5,%6,%7}, [%13];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8,%9,%10,%11}, [%14];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[1][0]),
          "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]), "=r"(r[2][0]), "=r"(r[2][1]),
          "=r"(r[2][2]), "=r"(r[2][3])
        : "r"(addr), "r"(addr + stride), "r"(addr + 2 * stride)
        : "memory");
  else
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%8];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4,%5,%6,%7}, [%9];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[1][0]),
          "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3])
        : "r"(addr), "r"(addr + stride)
        : "memory");
}

// The value a head's T accumulator columns stand for: FP8 t0 + t1 / 16 +
// t2 / 256 (f32 sums), int8 t0 + t1 / 254 (s32 sums).
template <bool kFp8>
__device__ __forceinline__ float terms_value(const uint32_t (&r)[3][4], int h) {
  if constexpr (kFp8)
    return __uint_as_float(r[0][h]) + __uint_as_float(r[1][h]) * 0.0625f +
           __uint_as_float(r[2][h]) * 0.00390625f;
  else
    return float(int32_t(r[0][h])) + float(int32_t(r[1][h])) * (1.f / 254.f);
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, TcTail* tail,
                                             int32_t* err) {
  if (mbar_wait(bar, parity)) return true;
  raise_err(err, PA_DEVERR_TIMEOUT);
  atomicExch(&tail->abort, 1);
  return false;
}

}  // namespace

template <bool kFp8, int kGp>
__global__ void __launch_bounds__(64 + 128 * kWG, 2) decode_q8tc_kernel(
    const __grid_constant__ CUtensorMap tmRK, const __grid_constant__ CUtensorMap tmRV,
    const DecodeArgs p, float scale_log2) {
  // kGp: the group size G rounded up to a power of two; B-operand column
  // n = term * kGp + head, so every register index is a compile-time one
  constexpr int T = kFp8 ? 3 : 2;          // 8-bit terms of Q and of P
  constexpr int N = q8tc_cols(kFp8, kGp);
  constexpr int kVStages = kMaxVStages;
  static_assert(N == 16, "G <= 4: 16 columns");
  extern __shared__ uint8_t tc_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~uintptr_t(1023));
  TcTail* tail = reinterpret_cast<TcTail*>(smem + tail_off(kVStages, N));
  uint8_t* vtile = smem + v_off();
  uint8_t* qterm = smem + q_off(kVStages);
  uint8_t* pterm = smem + p_off(kVStages, N);
  const uint32_t p_bytes = uint32_t(N / 8) * 1024u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x, kvh = blockIdx.y;
  const int b = p.order ? p.order[blockIdx.z] : int(blockIdx.z);
  const int G = p.H / p.Hkv;
  const int kv_len = p.kv_lens[b];
  const bool len_bad = kv_len < 0 || kv_len > p.MB * 16;
  const int nblk_seq = len_bad ? 0 : (kv_len + 15) >> 4;
  // Sink + recent window (window > 0): key j is visible iff j < sinks or
  // j >= lo; the CTAs walk the visible blocks only ([0, sb), then [lb,
  // nblk_seq)), numbered 0 .. nvis - 1.
  const int lo = (p.window > 0 && !len_bad) ? max(0, kv_len - p.window) : 0;
  const int sb = (min(p.sinks, kv_len) + 15) >> 4, lb = lo >> 4;
  const bool gap = lb > sb;
  const int nvis = gap ? sb + (nblk_seq - lb) : nblk_seq;
  auto vis_blk = [&](int v) { return (gap && v >= sb) ? lb + (v - sb) : v; };
  const int blk0 = part * p.part_blocks;
  const int nblk = max(0, min(blk0 + p.part_blocks, nvis) - blk0);
  const int ngroups = (nblk + kGroupBlocks - 1) / kGroupBlocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&tail->kfull[s], 1);
      mbar_init(&tail->kempty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&tail->vfull[s], 1);
      mbar_init(&tail->vempty[s], 1);
      tail->badmask[s] = 0;
    }
    for (int x = 0; x < kBufs; ++x) {
      mbar_init(&tail->s_full[x], 1);
      mbar_init(&tail->p_full[x], 128);
      mbar_init(&tail->o_full[x], 1);
    }
    mbar_init(&tail->q_ready, 128 * kWG);
    tail->any_bad = len_bad ? 1 : 0;
    tail->abort = 0;
    fence_barrier_init();
    if (len_bad && part == 0 && kvh == 0) raise_err(p.err, PA_DEVERR_KV_LEN);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tail->tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    // Lanes 0-7 each copy one block of a group (its K box and its V box): one
    // thread's copy-issue rate does not keep up with two boxes per block.
    if (ngroups > 0) {
      if (lane == 0) {
        prefetch_tensormap(&tmRK);
        prefetch_tensormap(&tmRV);
      }
      const uint64_t pol = policy_evict_first();
      const int32_t* trow = p.tables + int64_t(b) * p.MB;
      const bool copier = lane < kGroupBlocks;
      // a group's block ids are read one group ahead of its copies
      auto load_id = [&](int j) {
        const int v = j * kGroupBlocks + lane;
        return (copier && v < nblk) ? trow[vis_blk(blk0 + v)] : -1;
      };
      int cur = load_id(0);
      int issued = 0;
      for (int j = 0; j < ngroups; ++j) {
        const int nxt = j + 1 < ngroups ? load_id(j + 1) : -1;
        const int ks = j % kKStages, vs = j % kVStages;
        bool go = true;
        if (lane == 0) {
          go = (j < kKStages ||
                wait_or_flag(&tail->kempty[ks], ((j / kKStages) - 1) & 1, tail, p.err)) &&
               (j < kVStages ||
                wait_or_flag(&tail->vempty[vs], ((j / kVStages) - 1) & 1, tail, p.err)) &&
               !tail->abort;
        }
        if (!__shfl_sync(0xffffffffu, go ? 1 : 0, 0)) break;
        const int v = j * kGroupBlocks + lane;
        const bool bad = copier && v < nblk && (cur < 0 || cur >= p.NB);
        const bool valid = copier && v < nblk && !bad;
        const int mask = int(~__ballot_sync(0xffffffffu, valid) & 0xFFu);
        if (__any_sync(0xffffffffu, bad) && lane == 0) {
          tail->any_bad = 1;
          raise_err(p.err, PA_DEVERR_BLOCK_ID);
        }
        const uint32_t nvalid = uint32_t(__popc(~mask & 0xFF));
        if (lane == 0) {
          tail->badmask[vs] = mask;
          if (nvalid) {
            mbar_arrive_expect_tx(&tail->kfull[ks], nvalid * 2048u);
            mbar_arrive_expect_tx(&tail->vfull[vs], nvalid * kVSlot);
          } else {
            mbar_arrive(&tail->kfull[ks]);
            mbar_arrive(&tail->vfull[vs]);
          }
        }
        __syncwarp();                                  // the bytes are expected first
        if (valid) {
          const int z = cur * p.Hkv + kvh;
          tma_load_3d(smem + ks * kKTile + lane * 2048, &tmRK, &tail->kfull[ks], 0, 0, z, pol);
          tma_load_3d(vtile + vs * kVTile + lane * kVSlot, &tmRV, &tail->vfull[vs], 0, 16, z,
                      pol);
        }
        issued = j + 1;
        cur = nxt;
      }
      // drain: every issued copy has landed before the CTA may exit
      if (lane == 0) {
        for (int s = 0; s < kKStages && s < issued; ++s)
          mbar_wait(&tail->kfull[s], ((issued - 1 - s) / kKStages) & 1);
        for (int s = 0; s < kVStages && s < issued; ++s)
          mbar_wait(&tail->vfull[s], ((issued - 1 - s) / kVStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0 && ngroups > 0) {
      const uint32_t idesc = idesc_8bit(kFp8, N);
      const uint32_t qa = smem_u32(qterm);
      // Two queues, each in group order: QK(k) once group k has landed and
      // S buffer k & 1 is free (softmax(k - 2) has handed in P, i.e. PV(k - 2)
      // was issued; the tensor core runs this CTA's MMAs in issue order), and
      // PV(k) once the softmax has written P(k).  The thread issues whichever
      // is ready, so a stage is handed back as soon as its PV is done, not
      // after the next group's data has arrived.
      int nq = 0, npv = 0;
      bool ok = wait_or_flag(&tail->q_ready, 0, tail, p.err);
      uint64_t t0 = global_ns();
      uint32_t polls = 0;
      while (ok && npv < ngroups) {
        bool progressed = false;
        if (nq < ngroups && nq <= npv + kBufs - 1) {
          const int s = nq % kKStages, x = nq % kBufs;
          if (mbar_try_wait(&tail->kfull[s], (nq / kKStages) & 1)) {
            tc_fence_after();
            const uint32_t kb = smem_u32(smem + s * kKTile);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)             // S~_x = K(nq) Q~^T
              umma_8bit<kFp8>(tbase + 32 * x, desc_kmajor_sw128(kb + 32 * kk),
                              desc_kmajor_sw128(qa + 32 * kk), idesc, kk > 0 ? 1u : 0u);
            umma_commit(&tail->s_full[x]);
            umma_commit(&tail->kempty[s]);             // the K tile is done with
            ++nq;
            progressed = true;
          }
        }
        if (npv < nq) {
          const int s = npv % kVStages, x = npv % kBufs;
          if (mbar_try_wait(&tail->p_full[x], (npv / kBufs) & 1)) {
            tc_fence_after();
            const uint32_t vb = smem_u32(vtile + s * kVTile);
            const uint32_t pb = smem_u32(pterm + x * p_bytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)             // O_x = V^T(npv) P~(npv)^T
              umma_8bit<kFp8>(tbase + 32 * kBufs + 32 * x,
                              desc_kmajor_plain(vb + 2 * kk * kVSlot, kVSlot, 128),
                              desc_kmajor_plain(pb + 256 * kk, 128, 1024), idesc,
                              kk > 0 ? 1u : 0u);
            umma_commit(&tail->o_full[x]);
            umma_commit(&tail->vempty[s]);
            ++npv;
            progressed = true;
          }
        }
        if (progressed) {
          t0 = global_ns();
          polls = 0;
        } else if ((++polls & 255) == 0 && (global_ns() - t0 > kWaitLimitNs || tail->abort)) {
          if (!tail->abort) raise_err(p.err, PA_DEVERR_TIMEOUT);
          atomicExch(&tail->abort, 1);
          ok = false;
        }
      }
    }
  } else {
    // ------------------------------------------- softmax, fold, epilogue
    // Two warpgroups: warpgroup wg takes groups wg, wg + 2, ... (one group's
    // softmax runs while the other's waits on its MMAs).
    constexpr int kH = kGp;                           // heads per thread
    const int wg = (warp - 2) >> 2;
    const int sw = (warp - 2) & 3;                    // softmax warp of its warpgroup
    const int quarter = warp & 3;                     // its TMEM lane quarter
    const int tg = quarter * 32 + lane;               // key of the group, d row in the fold
    const int st = threadIdx.x - 64;                  // 0 .. 128 kWG - 1
    constexpr int kSm = 128 * kWG;                    // softmax threads
    const uint32_t bar_wg = 1 + wg;                   // named barrier of the warpgroup
    constexpr uint32_t kBarAll = 3;                   // every softmax thread
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    // Q rows and both P buffers start at zero: columns of heads >= G and
    // padding columns are never read, but the MMA reads their bytes
    for (int n = st >> 5; n < N; n += kSm / 32)
      reinterpret_cast<uint32_t*>(qterm + (n >> 3) * 1024 + (n & 7) * 128)[lane] = 0u;
    for (uint32_t o = st * 16; o < kBufs * p_bytes; o += kSm * 16)
      *reinterpret_cast<uint4*>(pterm + o) = make_uint4(0u, 0u, 0u, 0u);
    named_bar_sync(kBarAll, kSm);                     // zeros before the terms
    // ---- Q terms, one warp per head: lane covers d = 4 lane .. 4 lane + 3
    for (int h = warp - 2; h < G; h += 4 * kWG) {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(
                                static_cast<const __nv_bfloat16*>(p.q) +
                                (int64_t(b) * p.H + kvh * G + h) * 128) + lane);
      float x[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                    __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u)};
      float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
      amax = warp_max(amax);
      float sq;
      if constexpr (kFp8) {
        // the power of two at or above amax / 448: |Q / sq| <= 448
        sq = amax > 0.f ? fmaxf(exp2f(ceilf(log2f(amax / 448.f))), 0x1p-100f) : 1.f;
        while (amax / sq > 448.f) sq *= 2.f;
      } else {
        sq = amax > 0.f ? amax / 127.f : 1.f;
      }
      uint32_t word[3] = {0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t t[3];
        split_terms<kFp8>(x[e] / sq, t);
#pragma unroll
        for (int k = 0; k < T; ++k) word[k] |= t[k] << (8 * e);
      }
      const int c = lane >> 2;                        // 16-byte chunk of d
#pragma unroll
      for (int k = 0; k < T; ++k) {
        const int n = k * kGp + h;
        *reinterpret_cast<uint32_t*>(qterm + (n >> 3) * 1024 + (n & 7) * 128 +
                                     ((c ^ (n & 7)) << 4) + 4 * (lane & 3)) = word[k];
      }
      if (lane == 0) tail->qs[h] = sq * scale_log2;
    }
    fence_proxy_async_smem();
    named_bar_sync(kBarAll, kSm);                     // Q~ and qs[] of every head
    mbar_arrive(&tail->q_ready);
    float qs[kH];
#pragma unroll
    for (int h = 0; h < kH; ++h) qs[h] = h < G ? tail->qs[h] : 0.f;

    float m[kH], l[kH], o[kH];
#pragma unroll
    for (int h = 0; h < kH; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
      o[h] = 0.f;
    }
    // fold group jf's O_g into the registers (this thread's d row = tg):
    // o = o * alpha + O_g * unit; false if its wait gave up
    auto fold = [&](int jf, const float (&alpha)[kH], float unit_f) -> bool {
      const int xf = jf % kBufs;
      if (!__all_sync(0xffffffffu, mbar_wait(&tail->o_full[xf], (jf / kBufs) & 1))) {
        if (lane == 0) {
          raise_err(p.err, PA_DEVERR_TIMEOUT);
          atomicExch(&tail->abort, 1);
        }
        return false;
      }
      tc_fence_after();
      uint32_t v[3][4];
      tmem_ld_terms<T>(tbase + lane_off + 32 * kBufs + 32 * xf, kGp, v);
#pragma unroll
      for (int h = 0; h < kH; ++h)
        if (h < G) o[h] = fmaf(o[h], alpha[h], terms_value<kFp8>(v, h) * unit_f);
      return true;
    };

    // The four warps of a warpgroup leave the loop together: each group's
    // exchange carries every warp's "all waits succeeded" flag.
    bool ok = true, fold_ok = true;
    int it = -1;
    for (int j = wg; j < ngroups; j += kWG) {
      ++it;
      const int x = j % kBufs, s = j % kVStages;
      // S(j), and the group's V tile (its scales, its block mask)
      const bool mine = fold_ok &&
                        __all_sync(0xffffffffu, mbar_wait(&tail->s_full[x], (j / kBufs) & 1) &&
                                                    mbar_wait(&tail->vfull[s], (j / kVStages) & 1));
      tc_fence_after();
      uint32_t raw[3][4];
      if (mine) tmem_ld_terms<T>(tbase + lane_off + 32 * x, kGp, raw);
      const int mask = tail->badmask[s];
      const int i = tg >> 4, r = tg & 15;             // block of the group, key in the block
      const bool present = !((mask >> i) & 1);
      const int tok = vis_blk(blk0 + j * kGroupBlocks + i) * 16 + r;
      const bool live = mine && present && tok < kv_len && (tok >= lo || tok < p.sinks);
      uint8_t* vt = vtile + s * kVTile;
      const uint8_t* vs = vt + i * kVSlot;
      const float kscale = live ? reinterpret_cast<const float*>(vs + 2048)[r] : 0.f;
      const float vscale = live ? reinterpret_cast<const float*>(vs + 2112)[r] : 0.f;
      float sc[kH];
#pragma unroll
      for (int h = 0; h < kH; ++h)
        sc[h] = (live && h < G) ? terms_value<kFp8>(raw, h) * kscale * qs[h] : -INFINITY;
      // group maxima per head and of the live V scales: warp, then the 4 warps
      // exchange buffers alternate by this warpgroup's iteration, so a warp
      // ahead by one group never writes the slot another is still reading
      float* red = tail->red[it & 1][wg][sw];
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        if (h < G) {
          const float mx = warp_max(sc[h]);
          if (lane == 0) red[h] = mx;
        }
      }
      const float vmx = warp_max(vscale);
      if (lane == 0) {
        red[8] = vmx;
        red[9] = mine ? 1.f : 0.f;
      }
      named_bar_sync(bar_wg, 128);
      const float* rr = tail->red[it & 1][wg][0];
      ok = rr[9] != 0.f && rr[19] != 0.f && rr[29] != 0.f && rr[39] != 0.f;
      if (!ok) break;
      const float gv = fmaxf(fmaxf(rr[8], rr[18]), fmaxf(rr[28], rr[38]));
      // V unit: the power of two above the group's largest live V scale
      const float unit =
          gv > 0.f ? __uint_as_float(((__float_as_uint(gv) >> 23) + 1) << 23) : 1.f;
      const float v_over_unit = vscale * (1.f / unit);   // exact scaling by a power of two
      float alpha[kH];
      uint32_t pw[3][kH];
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        alpha[h] = 1.f;
        pw[0][h] = pw[1][h] = pw[2][h] = 0u;
        if (h < G) {
          const float gm = fmaxf(fmaxf(rr[h], rr[10 + h]), fmaxf(rr[20 + h], rr[30 + h]));
          const float mn = fmaxf(m[h], gm);
          alpha[h] = m[h] == -INFINITY ? 0.f : exp2f(m[h] - mn);
          m[h] = mn;
          const float pe = live ? exp2f(sc[h] - mn) : 0.f;      // live => mn finite
          l[h] = fmaf(l[h], alpha[h], pe);
          uint32_t t[3];
          split_terms<kFp8>(pe * v_over_unit * (kFp8 ? 256.f : 127.f), t);
          pw[0][h] = t[0];
          pw[1][h] = t[1];
          pw[2][h] = t[2];
        }
      }
      // P~ bytes: column n = term * G + head, key tg (core-matrix layout)
      uint8_t* pb = pterm + x * p_bytes + (tg >> 4) * 128 + (tg & 15);
#pragma unroll
      for (int k = 0; k < T; ++k)
#pragma unroll
        for (int h = 0; h < kH; ++h)
          if (h < G) {
            const int n = k * kGp + h;
            pb[(n >> 3) * 1024 + (n & 7) * 16] = uint8_t(pw[k][h]);
          }
      // only a group with a missing or bad block, or the sequence's partial
      // last block, holds stale V bytes
      const bool stale = mask != 0 || ((kv_len & 15) != 0 && j == ngroups - 1 &&
                                       blk0 + nblk == nvis);
      if (kFp8 && stale) {
        // stale V bytes may hold NaN codes: zero this thread's d row of them
#pragma unroll
        for (int bi = 0; bi < kGroupBlocks; ++bi) {
          const int keep = ((mask >> bi) & 1)
                               ? 0
                               : min(16, kv_len - vis_blk(blk0 + j * kGroupBlocks + bi) * 16);
          if (keep < 16) {
            uint32_t* row = reinterpret_cast<uint32_t*>(vt + bi * kVSlot + tg * 16);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int k4 = keep - 4 * q;            // bytes of this word to keep
              const uint32_t mk = k4 >= 4 ? 0xFFFFFFFFu : k4 <= 0 ? 0u : (0xFFFFFFFFu >> (32 - 8 * k4));
              row[q] &= mk;
            }
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&tail->p_full[x]);
      // fold now (the other warpgroup's softmax covers the wait for PV)
      fold_ok = fold(j, alpha, kFp8 ? unit * (1.f / 256.f) : unit * (1.f / 127.f));
    }
    ok = ok && fold_ok;

    // ------------------------------------------------------------ epilogue
    // l per head: sum over the warpgroup's 128 keys' partial sums; flags too
    float* er = tail->red[0][wg][sw];
    named_bar_sync(bar_wg, 128);                      // the last exchange's reads are done
#pragma unroll
    for (int h = 0; h < kH; ++h) {
      if (h < G) {
        float v = l[h];
#pragma unroll
        for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) er[h] = v;
      }
    }
    if (lane == 0) er[9] = ok ? 1.f : 0.f;
    named_bar_sync(bar_wg, 128);
    const float* rr = tail->red[0][wg][0];
    bool all_ok = rr[9] != 0.f && rr[19] != 0.f && rr[29] != 0.f && rr[39] != 0.f;
    float L[kH];
#pragma unroll
    for (int h = 0; h < kH; ++h)
      L[h] = h < G ? (rr[h] + rr[10 + h]) + (rr[20 + h] + rr[30 + h]) : 0.f;
    {
      // merge the two warpgroups' (m, l, o) through shared memory, in the K
      // tiles: once both warpgroups are past their loops every MMA of the CTA
      // has completed (each folded its last PV, and every QK precedes a PV)
      float* mo = reinterpret_cast<float*>(smem);     // [kH][128] o of warpgroup 1
      float* mml = mo + kH * 128;                    // [kH] m, [kH] l, ok
      named_bar_sync(kBarAll, kSm);
      if (wg == 1) {
#pragma unroll
        for (int h = 0; h < kH; ++h) mo[h * 128 + tg] = o[h];
        if (tg == 0) {
#pragma unroll
          for (int h = 0; h < kH; ++h) {
            mml[h] = m[h];
            mml[kH + h] = L[h];
          }
          mml[2 * kH] = all_ok ? 1.f : 0.f;
        }
      }
      named_bar_sync(kBarAll, kSm);
      if (wg == 0) {
        all_ok = all_ok && mml[2 * kH] != 0.f;
#pragma unroll
        for (int h = 0; h < kH; ++h) {
          const float m1 = mml[h];
          const float M = fmaxf(m[h], m1);
          const float w0 = m[h] == -INFINITY ? 0.f : exp2f(m[h] - M);
          const float w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
          o[h] = o[h] * w0 + mo[h * 128 + tg] * w1;
          L[h] = L[h] * w0 + mml[kH + h] * w1;
          m[h] = M;
        }
      }
    }
    if (wg == 0) {
      const bool zero = tail->any_bad != 0 || !all_ok || tail->abort;
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        if (h >= G) break;
        const float val = (L[h] > 0.f && !zero) ? o[h] / L[h] : 0.f;
        const int64_t bh = int64_t(b) * p.H + kvh * G + h;
        if (p.NP == 1) {
          p.out[bh * 128 + tg] = val;
        } else {
          const int64_t slot = bh * p.NP + part;
          float* ws_m = p.ws;
          float* ws_l = ws_m + int64_t(p.B) * p.H * p.NP;
          float* ws_o = ws_l + int64_t(p.B) * p.H * p.NP;
          ws_o[slot * 128 + tg] = val;
          if (tg == 0) {
            ws_m[slot] = zero ? -INFINITY : m[h];
            ws_l[slot] = zero ? -1.f : L[h];          // -1 poisons the whole row
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

namespace {

template <bool kFp8, int kGp>
cudaError_t launch_tc(const CUtensorMap* tmRK, const CUtensorMap* tmRV, const DecodeArgs& a,
                      cudaStream_t stream) {
  // two K tiles and four V tiles: two CTAs per SM
  constexpr int N = q8tc_cols(kFp8, kGp);
  const size_t smem = 1024 + tail_off(kMaxVStages, N) + sizeof(TcTail);
  static_assert(1024 + tail_off(kMaxVStages, N) + sizeof(TcTail) <= 113 * 1024,
                "two CTAs per SM");
  auto* kern = decode_q8tc_kernel<kFp8, kGp>;
  static PerDeviceOnce attr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = static_cast<cudaError_t>(attr.run(dev, [&] {
    return int(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(smem)));
  }));
  if (e != cudaSuccess) return e;
  dim3 grid(a.NP, a.Hkv, a.B);
  kern<<<grid, 64 + 128 * kWG, smem, stream>>>(*tmRK, *tmRV, a, a.scale * kLog2e);
  return cudaGetLastError();
}

template <bool kFp8>
cudaError_t launch_tc_g(const CUtensorMap* tmRK, const CUtensorMap* tmRV, const DecodeArgs& a,
                        int G, cudaStream_t stream) {
  if (G <= 1) return launch_tc<kFp8, 1>(tmRK, tmRV, a, stream);
  if (G <= 2) return launch_tc<kFp8, 2>(tmRK, tmRV, a, stream);
  return launch_tc<kFp8, 4>(tmRK, tmRV, a, stream);
}

}  // namespace

cudaError_t launch_decode_q8tc(const CUtensorMap* tmRK, const CUtensorMap* tmRV,
                               const DecodeArgs& a, bool fp8, cudaStream_t stream) {
  const int G = a.H / a.Hkv;
  if (G < 1 || G > 4) return cudaErrorInvalidValue;
  if (a.order) {
    cudaError_t eo = launch_decode_order(a.kv_lens, a.B, a.order, stream);
    if (eo != cudaSuccess) return eo;
  }
  cudaError_t e = fp8 ? launch_tc_g<true>(tmRK, tmRV, a, G, stream)
                      : launch_tc_g<false>(tmRK, tmRV, a, G, stream);
  if (e != cudaSuccess || a.NP == 1) return e;
  return launch_decode_combine(a.ws, a.B, a.H, a.NP, a.out, stream);
}

}  // namespace pa
