// Paged decode attention over an int8 KV pool: per-(token, head) rows of 128
// int8 codes with one float32 scale each, head_dim 128, block_size 16, GQA
// group G <= 8.  One CTA per (partition, KV head, sequence).
//
// What it computes: the decode of "docs.rs ferrum-kv 0.4.0 src/attention.rs"
// (paged_attention, q_tokens = 1) on the K/V rows the pool holds, i.e.
// k_j = code_k[j] * scale_k[j], v_j = code_v[j] * scale_v[j], the per-row
// absmax quantisation of "vladkulikov.com modern-llms module 9 notebook"
// (KV quantisation experiment, 8 bits), with the one-pass (m, l, acc) update
// of "semidirectx cmu11-667 lecture19 infer_world.py", section 3.
//
// Same machinery as the bf16 decode (producer warp + TMA ring, four consumer
// warps on tensor-core tiles, (m, l, O) merge, split partitions), with half
// the bytes per token:
//  * the pool keeps each (block, head) as one packed 4224-byte record
//    [K codes 2 KB | V codes 2 KB | 16 K scales | 16 V scales], staged with a
//    single TMA load (the records viewed as [NB * Hkv][33][128 bytes], one
//    33-row box per record; one copy instruction per block).  K rows
//    are token-major with their 16-byte chunks stored pre-swizzled (chunk k of
//    token t at k ^ (t & 7)); V is d-major (row d = the 16 tokens' codes);
//  * S^T = K Q^T runs on the int8 tensor-core MMA (m16n8k32, s32
//    accumulators) straight from the codes: Q is split per head into
//    int8 hi and lo parts, q = sq (hi + lo / 254) (error <= max|q| / 64516
//    per element), two MMAs per 32 columns, and
//    q.k_j = sq scale_k[j] (acc_hi + acc_lo / 254);
//  * O^T += V^T P^T runs on the fp16 MMA: two adjacent V codes become one
//    half2 with a byte permute and one subtraction (fp16 holds 1024 + u
//    exactly), and sum_j p_j v_j = 2^E sum_j (p_j scale_v[j] 2^-E) code_v[j]
//    with 2^E the block's largest V scale (a power of two, so the fp16 P
//    keeps its precision; O is rescaled by the ratio of successive 2^E
//    together with the online-softmax factor).  P goes in as fp16 hi + lo
//    parts; l sums the unscaled p_j.
// FP8 (E4M3) pools use the same record, with E4M3 codes and scales
// absmax / 448.  The fp8 instance runs both products on the fp16 MMA (every
// E4M3 value is exact in fp16).  V codes go through the E4M3 x2 -> f16 x2
// conversion; K codes, to spare that conversion unit, through integer ops:
// a code b in a 16-bit lane, (b + (b & 0x80)) << 7, is the fp16 pattern of
// value(b) * 2^-8 (sign to bit 15, exponent and mantissa bits shifted in
// place, subnormals included), taken as pairs (d0, d2) and (d1, d3) of each
// 4-byte word, with Q packed to match and the 2^8 folded into the score
// scale.  Q enters as fp16 with a power-of-two scale (exact for bf16
// inputs), so S = K Q^T is exact up to fp32 accumulation.  E4M3 has NaN
// codes, so the V bytes of dead tokens are zeroed before conversion.
// Token order: row r of a block's S^T tile holds token kPerm[r].  With it a
// thread's P^T fragment covers tokens 4c .. 4c + 3 (two per register), the
// four bytes of one 32-bit word of a V d-row, and the K rows a warp reads at
// once have distinct swizzle phases (no bank conflicts).
#include <math.h>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "device_once.hpp"
#include "launch.hpp"

namespace pa {

namespace {

constexpr int kQ8Threads = 160;     // 4 consumer warps + 1 producer warp
constexpr int kQ8Stages = 16;       // multiple of the 4 consumer warps
constexpr int kQ8StageBytes = kQ8RecordBytes;  // one packed (block, head) record
constexpr float kLog2e = 1.4426950408889634f;
// S^T row r of a block holds token kPerm[r] (see the file comment)
__constant__ int kPerm[16] = {0, 1, 4, 5, 10, 11, 14, 15, 2, 3, 6, 7, 8, 9, 12, 13};

struct Q8Tail {
  uint64_t full[kQ8Stages];
  uint64_t empty[kQ8Stages];
  int stage_bad[kQ8Stages];
  int any_bad;
};

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// D (s32) += A (16 x 32 s8, row) * B (32 x 8 s8, col)
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0,
                                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D (f32) += A (16 x 16 f16, row) * B (16 x 8 f16, col)
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two codes of the biased word u = w ^ 0x80808080 (bytes picked by sel,
// low then high) as an exact half2: the permute builds 0x64uu halves, i.e.
// 1024 + u, and 1152 = 1024 + 128 taken away leaves the signed code.
__device__ __forceinline__ uint32_t codes_half2(uint32_t u, uint32_t sel) {
  const uint32_t x = __byte_perm(u, 0x64646464u, sel);
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&x),
                            __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Two E4M3 codes (low byte, high byte of a 16-bit pair) as an exact half2
// (low byte -> low half).
__device__ __forceinline__ uint32_t e4m3x2_half2(uint32_t pair) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
      static_cast<__nv_fp8x2_storage_t>(pair & 0xFFFFu), __NV_E4M3);
  return uint32_t(h.x) | (uint32_t(h.y) << 16);
}

// Two E4M3 codes at bits 0-7 and 16-23 of y (other bits zero) as a half2
// of their values times 2^-8: y * 128 moves each code's magnitude bits to
// 7-13 (fp16 exponent and mantissa) and its sign to bit 14; adding that bit
// again carries it up to bit 15.
__device__ __forceinline__ uint32_t e4m3x2_half2_div256(uint32_t y) {
  const uint32_t z = y * 128u;
  return z + (z & 0x40004000u);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

template <bool kFp8>
__global__ void __launch_bounds__(kQ8Threads, 3) decode_q8_kernel(
    const __grid_constant__ CUtensorMap tmR, const DecodeArgs p, float scale_log2) {
  extern __shared__ uint8_t q8_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(q8_raw) + 127) & ~uintptr_t(127));
  Q8Tail* tail = reinterpret_cast<Q8Tail*>(smem + kQ8Stages * kQ8StageBytes);

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

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQ8Stages; ++s) {
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
      const uint64_t pol = policy_evict_first();
      const int32_t* trow = p.tables + int64_t(b) * p.MB;
      // Block ids in groups of 8, read one group ahead: an id read right
      // before its copy puts a table round trip on every block.
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
          const int s = i % kQ8Stages, round = i / kQ8Stages;
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
            uint8_t* st = smem + s * kQ8StageBytes;
            mbar_arrive_expect_tx(&tail->full[s], kQ8StageBytes);
            tma_load_3d(st, &tmR, &tail->full[s], 0, 0, blk * p.Hkv + kvh, pol);
          }
          issued = i + 1;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) cur[u] = nxt[u];
        load8(base + 16, nxt);
      }
      // drain: no copy may still be landing in shared memory at exit
      for (int s = 0; s < kQ8Stages && s < issued; ++s) {
        const int count = (issued - 1 - s) / kQ8Stages + 1;
        mbar_wait(&tail->full[s], (count - 1) & 1);
      }
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  const int g = lane >> 2, c = lane & 3;
  // int8: Q of head g as int8 hi + lo parts in the B-fragment order of
  // m16n8k32: word kk*2 + h covers d = 32 kk + 16 h + 4c .. + 3.
  // fp8: Q / sq as fp16 B fragments of m16n8k16 over d chunk 2 kk + h, with
  // MMA k (2c, 2c + 1) = d (4c, 4c + 2) in qh and k (2c + 8, 2c + 9) =
  // d (4c + 1, 4c + 3) in ql, the order in which the K words unpack.
  uint32_t qh[4][2], ql[4][2];
  float qs0, qs1;   // sq * scale_log2 of heads 2c and 2c + 1 (S^T columns)
  {
    const bool ok = g < G;
    const uint2* qrow = reinterpret_cast<const uint2*>(
        static_cast<const __nv_bfloat16*>(p.q) + (int64_t(b) * p.H + kvh * G + (ok ? g : 0)) * 128);
    float x[4][2][4];
    float amax = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint2 w = ok ? __ldg(qrow + 8 * kk + 4 * h + c) : make_uint2(0u, 0u);
        x[kk][h][0] = __uint_as_float(w.x << 16);
        x[kk][h][1] = __uint_as_float(w.x & 0xFFFF0000u);
        x[kk][h][2] = __uint_as_float(w.y << 16);
        x[kk][h][3] = __uint_as_float(w.y & 0xFFFF0000u);
#pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(x[kk][h][e]));
      }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    float sq;
    if constexpr (kFp8) {
      // sq = the power of two at or below amax: Q / sq is exact in fp16
      const uint32_t e = min(max((__float_as_uint(amax) >> 23) & 0xFFu, 1u), 253u);
      sq = __uint_as_float(e << 23);
      const float inv = __uint_as_float((254u - e) << 23);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          qh[kk][h] = pack_half2(x[kk][h][0] * inv, x[kk][h][2] * inv);
          ql[kk][h] = pack_half2(x[kk][h][1] * inv, x[kk][h][3] * inv);
        }
    } else {
    sq = amax > 0.f ? amax / 127.f : 1.f;
    const float inv = amax > 0.f ? 127.f / amax : 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t hw = 0, lw = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float t = fminf(fmaxf(x[kk][h][e] * inv, -127.f), 127.f);
          const float hi = rintf(t);
          const float lo = rintf((t - hi) * 254.f);
          hw |= (uint32_t(int32_t(hi)) & 0xFFu) << (8 * e);
          lw |= (uint32_t(int32_t(lo)) & 0xFFu) << (8 * e);
        }
        qh[kk][h] = hw;
        ql[kk][h] = lw;
      }
    }
    // fp8: K enters the MMA as value * 2^-8
    const float ks = kFp8 ? 256.f * scale_log2 : scale_log2;
    qs0 = __shfl_sync(0xffffffffu, sq, 8 * c) * ks;
    qs1 = __shfl_sync(0xffffffffu, sq, 8 * c + 4) * ks;
  }
  const int tokA = kPerm[g], tokB = kPerm[g + 8];       // tokens of S^T rows g, g + 8
  const uint32_t rowA = tokA * 128, rowB = tokB * 128;
  const uint32_t keyA = tokA & 7, keyB = tokB & 7;      // their swizzle phases
  // V^T A fragments: tokens kPerm[2c], kPerm[2c+1] are bytes (0,1) of word c
  // for c < 2 and bytes (2,3) otherwise; kPerm[2c+8], kPerm[2c+9] the others
  const uint32_t sel_a = c < 2 ? 0x4140u : 0x4342u;
  const uint32_t sel_b = c < 2 ? 0x4342u : 0x4140u;
  // fp8: the same pairs, as the low and high halves of the word rotated so
  // that the pair of A fragment a0 comes first
  const uint32_t vrot = c < 2 ? 0x3210u : 0x1032u;
  float o[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float unit = 0.f;    // 2^-E of the warp's O (0 before its first block)
  const int tok_end = kv_len;

  // Each warp takes its blocks two at a time (i and i + 4): one online-softmax
  // step over 32 tokens, and the two blocks' loads and MMAs interleaved.  A
  // missing or unusable block runs the same code with every token dead: its
  // scores are -inf and its V scales 0, so its (finite) codes add exactly 0.
  for (int i = warp; i < nblk; i += 8) {
    const int i2 = i + 4;
    const int sa = i % kQ8Stages, sb = i2 % kQ8Stages;
    const bool has2 = i2 < nblk;
    bool landed = mbar_wait(&tail->full[sa], (i / kQ8Stages) & 1);
    if (has2) landed = landed && mbar_wait(&tail->full[sb], (i2 / kQ8Stages) & 1);
    if (!__all_sync(0xffffffffu, landed)) {
      if (lane == 0) {
        raise_err(p.err, PA_DEVERR_TIMEOUT);
        tail->any_bad = 1;
      }
      break;
    }
    const bool use[2] = {!tail->stage_bad[sa], has2 && !tail->stage_bad[sb]};
    const uint32_t kb[2] = {smem_u32(smem + sa * kQ8StageBytes),
                            smem_u32(smem + sb * kQ8StageBytes)};
    const float* scl[2] = {reinterpret_cast<const float*>(smem + sa * kQ8StageBytes + 4096),
                           reinterpret_cast<const float*>(smem + sb * kQ8StageBytes + 4096)};
    const int tb[2] = {vis_blk(blk0 + i) * 16, vis_blk(blk0 + i2) * 16};
    // ---- S^T = K Q^T on int8 codes: hi and lo parts of Q
    int ih[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}}, il[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
    float fs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};   // fp8: S in fp32
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t c0 = 2 * kk, c1 = 2 * kk + 1;
      uint32_t a[2][4];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        a[x][0] = lds32(kb[x] + rowA + ((c0 ^ keyA) << 4) + 4 * c);
        a[x][2] = lds32(kb[x] + rowA + ((c1 ^ keyA) << 4) + 4 * c);
        a[x][1] = lds32(kb[x] + rowB + ((c0 ^ keyB) << 4) + 4 * c);
        a[x][3] = lds32(kb[x] + rowB + ((c1 ^ keyB) << 4) + 4 * c);
      }
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if constexpr (kFp8) {
          // chunk 2kk: rows A, B in a[x][0], a[x][1]; chunk 2kk + 1: a[x][2], a[x][3]
          // even bytes (d0, d2) -> MMA k (2c, 2c + 1); odd (d1, d3) -> (2c + 8, 2c + 9)
          mma_f16_16816(fs[x], e4m3x2_half2_div256(a[x][0] & 0x00FF00FFu),
                        e4m3x2_half2_div256(a[x][1] & 0x00FF00FFu),
                        e4m3x2_half2_div256((a[x][0] >> 8) & 0x00FF00FFu),
                        e4m3x2_half2_div256((a[x][1] >> 8) & 0x00FF00FFu), qh[kk][0], ql[kk][0]);
          mma_f16_16816(fs[x], e4m3x2_half2_div256(a[x][2] & 0x00FF00FFu),
                        e4m3x2_half2_div256(a[x][3] & 0x00FF00FFu),
                        e4m3x2_half2_div256((a[x][2] >> 8) & 0x00FF00FFu),
                        e4m3x2_half2_div256((a[x][3] >> 8) & 0x00FF00FFu), qh[kk][1], ql[kk][1]);
        } else {
          mma_s8_16832(ih[x], a[x][0], a[x][1], a[x][2], a[x][3], qh[kk][0], qh[kk][1]);
          mma_s8_16832(il[x], a[x][0], a[x][1], a[x][2], a[x][3], ql[kk][0], ql[kk][1]);
        }
      }
    }
    float sc[2][4], vA[2], vB[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int t0 = tb[x] + tokA, t1 = tb[x] + tokB;
      const bool live0 = use[x] && t0 < tok_end && (t0 >= lo || t0 < p.sinks);
      const bool live1 = use[x] && t1 < tok_end && (t1 >= lo || t1 < p.sinks);
      const float kA = scl[x][tokA], kB = scl[x][tokB];
      float dot[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        dot[k] = kFp8 ? fs[x][k] : fmaf(float(il[x][k]), 1.f / 254.f, float(ih[x][k]));
      sc[x][0] = live0 ? dot[0] * (kA * qs0) : -INFINITY;
      sc[x][1] = live0 ? dot[1] * (kA * qs1) : -INFINITY;
      sc[x][2] = live1 ? dot[2] * (kB * qs0) : -INFINITY;
      sc[x][3] = live1 ? dot[3] * (kB * qs1) : -INFINITY;
      vA[x] = live0 ? scl[x][16 + tokA] : 0.f;
      vB[x] = live1 ? scl[x][16 + tokB] : 0.f;
    }
    float x0 = fmaxf(fmaxf(sc[0][0], sc[0][2]), fmaxf(sc[1][0], sc[1][2]));
    float x1 = fmaxf(fmaxf(sc[0][1], sc[0][3]), fmaxf(sc[1][1], sc[1][3]));
    float vmax = fmaxf(fmaxf(vA[0], vB[0]), fmaxf(vA[1], vB[1]));
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    }
    if (x0 == -INFINITY) {          // nothing usable in the pair (bad blocks)
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tail->empty[sa]);
        if (has2) mbar_arrive(&tail->empty[sb]);
      }
      continue;
    }
    const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
    const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);
    float pp[2][4];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      pp[x][0] = exp2f(sc[x][0] - n0);
      pp[x][1] = exp2f(sc[x][1] - n1);
      pp[x][2] = exp2f(sc[x][2] - n0);
      pp[x][3] = exp2f(sc[x][3] - n1);
    }
    l0 = l0 * al0 + ((pp[0][0] + pp[0][2]) + (pp[1][0] + pp[1][2]));
    l1 = l1 * al1 + ((pp[0][1] + pp[0][3]) + (pp[1][1] + pp[1][3]));
    m0 = n0;
    m1 = n1;
    // power-of-two V unit 2^(E+1) > the largest live V scale of the pair
    const uint32_t e = min(max((__float_as_uint(vmax) >> 23) & 0xFFu, 1u), 252u);
    const float bunit = __uint_as_float((253u - e) << 23);   // 2^-(E + 1)
    const float ratio = unit == 0.f ? 1.f : bunit / unit;     // O in the new unit
    unit = bunit;
    const float r0 = al0 * ratio, r1 = al1 * ratio;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      o[j][0] *= r0;
      o[j][1] *= r1;
      o[j][2] *= r0;
      o[j][3] *= r1;
    }
    // P^T (times V scale and unit) as fp16 B fragments: hi + lo parts
    uint32_t fb[2][4];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const float q0 = pp[x][0] * (vA[x] * bunit), q1 = pp[x][1] * (vA[x] * bunit);
      const float q2 = pp[x][2] * (vB[x] * bunit), q3 = pp[x][3] * (vB[x] * bunit);
      const __half2 h01 = __floats2half2_rn(q0, q1), h23 = __floats2half2_rn(q2, q3);
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      fb[x][0] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h01));
      fb[x][1] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h23));
      fb[x][2] = movmatrix_trans(pack_half2(q0 - f01.x, q1 - f01.y));
      fb[x][3] = movmatrix_trans(pack_half2(q2 - f23.x, q3 - f23.y));
    }
    // fp8: byte mask of this thread's live tokens 4c .. 4c + 3 per block
    uint32_t vmask[2] = {0u, 0u};
    if constexpr (kFp8) {
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = tb[x] + 4 * c + u;
          if (use[x] && t < tok_end && (t >= lo || t < p.sinks)) vmask[x] |= 0xFFu << (8 * u);
        }
    }
    // ---- O^T += V^T P^T: d rows 16j + g and 16j + g + 8, tokens 4c .. 4c + 3
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t w[2][2];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        w[x][0] = lds32(kb[x] + 2048 + (16 * j + g) * 16 + 4 * c);
        w[x][1] = lds32(kb[x] + 2048 + (16 * j + g + 8) * 16 + 4 * c);
      }
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        uint32_t a0, a1, a2, a3;
        if constexpr (kFp8) {
          const uint32_t u0 = __byte_perm(w[x][0] & vmask[x], 0u, vrot);
          const uint32_t u1 = __byte_perm(w[x][1] & vmask[x], 0u, vrot);
          a0 = e4m3x2_half2(u0);
          a2 = e4m3x2_half2(u0 >> 16);
          a1 = e4m3x2_half2(u1);
          a3 = e4m3x2_half2(u1 >> 16);
        } else {
          const uint32_t b0 = w[x][0] ^ 0x80808080u, b1 = w[x][1] ^ 0x80808080u;
          a0 = codes_half2(b0, sel_a);
          a2 = codes_half2(b0, sel_b);
          a1 = codes_half2(b1, sel_a);
          a3 = codes_half2(b1, sel_b);
        }
        mma_f16_16816(o[j], a0, a1, a2, a3, fb[x][0], fb[x][1]);
        mma_f16_16816(o[j], a0, a1, a2, a3, fb[x][2], fb[x][3]);
      }
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&tail->empty[sa]);
      if (has2) mbar_arrive(&tail->empty[sb]);
    }
  }
  // O back to absolute units
  if (unit > 0.f) {
    const float back = 1.f / unit;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) o[j][k] *= back;
  }

  // ------------------------------------------- merge the four warps' states
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  named_bar_sync(1, 128);  // every consumer is done with the ring
  float* so = reinterpret_cast<float*>(smem);  // [4][8][128]
  float* sm = so + 4 * 8 * 128;                // [4][8]
  float* sl = sm + 32;                         // [4][8]
  {
    float* w0 = so + (warp * 8 + 2 * c) * 128;
    float* w1 = w0 + 128;
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
  const int t = threadIdx.x;  // d column
  const bool zero = tail->any_bad != 0;
  for (int n = 0; n < G; ++n) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w * 8 + n]);
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = sm[w * 8 + n];
        const float sc = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        num = fmaf(so[(w * 8 + n) * 128 + t], sc, num);
        den = fmaf(sl[w * 8 + n], sc, den);
      }
    }
    const float val = (den > 0.f && !zero) ? num / den : 0.f;
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
        ws_m[slot] = M;
        ws_l[slot] = zero ? -1.f : den;  // -1 poisons the whole row
      }
    }
  }
}

cudaError_t launch_decode_q8(const CUtensorMap* tmR, const DecodeArgs& a, bool fp8,
                             cudaStream_t stream) {
  if (a.order) {
    cudaError_t eo = launch_decode_order(a.kv_lens, a.B, a.order, stream);
    if (eo != cudaSuccess) return eo;
  }
  const size_t smem = 128 + kQ8Stages * kQ8StageBytes + sizeof(Q8Tail);
  auto* kern = fp8 ? decode_q8_kernel<true> : decode_q8_kernel<false>;
  static PerDeviceOnce attr[2];
  int dev = 0;
  cudaError_t ea = cudaGetDevice(&dev);
  if (ea != cudaSuccess) return ea;
  ea = static_cast<cudaError_t>(attr[fp8].run(dev, [&] {
    return int(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(smem)));
  }));
  if (ea != cudaSuccess) return ea;
  dim3 grid(a.NP, a.Hkv, a.B);
  kern<<<grid, kQ8Threads, smem, stream>>>(*tmR, a, a.scale * kLog2e);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.NP == 1) return e;
  return launch_decode_combine(a.ws, a.B, a.H, a.NP, a.out, stream);
}

}  // namespace pa
