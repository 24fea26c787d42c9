// Kernel launchers (host side), one per kernel family.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

struct pa_pool;

namespace pa {

// The device a pool's memory lives on (-1 for a host-only pool).
int pool_device(const pa_pool* p);

// Makes `dev` current for the lifetime of one entry-point call (when it is
// not already) and restores the caller's device afterwards; dev < 0 = no-op.
class DeviceScope {
 public:
  explicit DeviceScope(int dev) {
    if (dev >= 0 && cudaGetDevice(&prev_) == cudaSuccess && prev_ != dev)
      switched_ = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceScope() {
    if (switched_) cudaSetDevice(prev_);
  }
  DeviceScope(const DeviceScope&) = delete;
  DeviceScope& operator=(const DeviceScope&) = delete;

 private:
  int prev_ = -1;
  bool switched_ = false;
};

cudaError_t launch_reshape_and_cache(const void* key, const void* value,
                                     void* k_cache, void* v_cache,
                                     const int64_t* slots, int32_t T,
                                     int64_t row_bytes, int64_t num_slots,
                                     int32_t* err, int sms,
                                     cudaStream_t stream);

cudaError_t launch_cow_copy(void* k_cache, void* v_cache, const int32_t* src,
                            const int32_t* dst, int32_t n, int64_t block_bytes,
                            int32_t num_blocks, int32_t* err, int sms,
                            cudaStream_t stream);

// Up to four host -> device copies in one kernel launch: src is the mapped
// device address of pinned host memory, both ends 16-byte aligned, n16 the
// length in 16-byte units (0: unused).
constexpr int kUploadSegs = 4;
struct UploadSeg {
  const uint4* src = nullptr;
  uint4* dst = nullptr;
  int64_t n16 = 0;
};
struct UploadArgs {
  UploadSeg seg[kUploadSegs];
};
cudaError_t launch_upload(const UploadArgs& a, int sms, cudaStream_t stream);

// Table patches (row, index, value) x n applied to device tables [rows, width].
cudaError_t launch_table_patch(int32_t* tables, int32_t width, const int32_t* patches,
                               int32_t n, cudaStream_t stream);

// Generic CUDA-core paged attention: any dtype, head_dim <= 512, any block
// size and group size, q_tokens >= 1 (causal offset rule).
struct GenericArgs {
  const void* q;  // [B, q_tokens, H, d]
  const void* k_cache;
  const void* v_cache;
  const int32_t* tables;
  int32_t MB;
  const int32_t* kv_lens;
  int32_t B, q_tokens, H, Hkv, d, bs, NB;
  float scale;
  float* out;  // [B, q_tokens, H, d]
  int32_t* err;
  bool bf16;
  int32_t q8;     // 0: K/V arrays of the pool dtype; 1 / 2: int8 / FP8 records, bf16 q
  int32_t window = 0, sinks = 0;   // decode only: keys j < sinks or j >= kv_len - window
};
cudaError_t launch_attention_generic(const GenericArgs& a, cudaStream_t s);

// Tensor-core decode for bf16, head_dim 128, block_size 16, group <= 8.
struct DecodeArgs {
  const void* q;  // [B, H, 128] bf16
  const int32_t* tables;
  int32_t MB;
  const int32_t* kv_lens;
  int32_t B, H, Hkv, NB;
  float scale;
  int32_t part_blocks;  // blocks per partition
  int32_t NP;           // partitions per sequence (1 = no split)
  float* out;           // [B, H, 128]
  float* ws;            // split scratch (NP > 1)
  int32_t* err;
  int32_t* order;       // longest-first sequence order (device, [B]) or null
  // fused append (all null/0 when off): token kv_len-1 of sequence b is new;
  // its K/V rows new_k/new_v [B, Hkv, 128] go to pool slot new_slots[b]
  const void* new_k;
  const void* new_v;
  const int64_t* new_slots;
  void* k_cache;
  void* v_cache;
  // sink + recent window (window <= 0: every key): key j of a sequence is
  // visible iff j < sinks or j >= kv_len - window
  int32_t window;
  int32_t sinks;
};
bool decode_fast_supported(int dtype_bf16, int d, int bs, int G);
cudaError_t launch_decode_fast(const CUtensorMap* tmK, const CUtensorMap* tmV,
                               const DecodeArgs& a, int sms,
                               cudaStream_t stream);
size_t split_workspace_bytes(int32_t B, int32_t H, int32_t NP, int32_t d);
// Shared by the bf16 and int8 decodes: the longest-first order prepass and
// the log-sum-exp combine of split partitions.
cudaError_t launch_decode_order(const int32_t* kv_lens, int32_t B, int32_t* order,
                                cudaStream_t stream);
cudaError_t launch_decode_combine(const float* ws, int32_t B, int32_t H, int32_t NP,
                                  float* out, cudaStream_t stream);

// int8 pools: one packed record of kQ8RecordBytes per (block, head),
// [NB, Hkv, record]: K codes [16 tokens][128] with each token's 16-byte
// chunks stored swizzled (chunk k at k ^ (token & 7)), V codes [128 d][16
// tokens], 16 float32 K scales, 16 float32 V scales.
constexpr int kQ8RecordBytes = 4224;
// The same record holds int8 codes or FP8 (E4M3) codes.
// Append: key/value bf16 [T, Hkv, 128] are quantised per (token, head) row
// (int8: absmax / 127, round half to even; fp8: absmax / 448, nearest E4M3
// value, ties to even; decided in float64) into their slots.
cudaError_t launch_reshape_and_cache_q8(const void* key, const void* value, void* records,
                                        const int64_t* slots, int32_t T, int32_t Hkv,
                                        int64_t num_slots, bool fp8, int32_t* err, int sms,
                                        cudaStream_t stream);
// Decode over an int8 or FP8 pool (G <= 8; tmR maps the records as
// {128 bytes, 33 rows, NB * Hkv}), dequantising in the kernel.
cudaError_t launch_decode_q8(const CUtensorMap* tmR, const DecodeArgs& a, bool fp8,
                             cudaStream_t stream);
// The same decode on tcgen05 tensor cores straight from the codes: tmRK maps
// the records with a {128, 16, 1} box (K codes), tmRV with a {128, 17, 1}
// box (V codes and the two scale rows, read at row 16).
cudaError_t launch_decode_q8tc(const CUtensorMap* tmRK, const CUtensorMap* tmRV,
                               const DecodeArgs& a, bool fp8, cudaStream_t stream);
// Scratch for the longest-first order when the grid spans several waves.
bool decode_wants_order(int32_t B, int32_t Hkv, int32_t NP, int sms);
size_t order_workspace_bytes(int32_t B);

// Chunked prefill on tcgen05 tensor cores (bf16, head_dim 128, block 16).
struct PrefillArgs {
  const void* q;  // [B, q_tokens, H, 128] bf16
  const int32_t* tables;
  int32_t MB;
  const int32_t* kv_lens;
  int32_t B, q_tokens, H, Hkv, NB;
  float scale;
  float* out;  // [B, q_tokens, H, 128] fp32
  int32_t* err;
  // key-split scratch of the last wave (null = no split): split_slots slots
  // of 2 x 128 x 128 fp32 (split_o) and 2 x 128 (m, l) pairs (split_ml), and
  // 2 tickets per split unit (tickets, zero between calls)
  int32_t max_splits;  // 0 = automatic, 1 = never split, n = at most n parts
  float* split_o;
  float* split_ml;
  int32_t* tickets;
  int32_t split_slots;
};
bool prefill_fast_supported(int dtype_bf16, int d, int bs, int G);
cudaError_t launch_prefill_fast(const CUtensorMap* tmK, const CUtensorMap* tmV,
                                const PrefillArgs& a, int sms,
                                cudaStream_t stream);

}  // namespace pa
