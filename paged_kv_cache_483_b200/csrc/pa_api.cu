// C ABI of the paged-attention library (declared in include/pa.h).
//
// Argument checking, the host block manager, append staging and kernel
// dispatch.  No compute happens here: every step of the path runs in the
// kernels of kv_write.cu, attention_generic.cu, decode_mma.cu and
// prefill_tc.cu.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <memory>
#include <new>
#include <vector>

#include "../../include/pa.h"
#include "block_manager.hpp"
#include "common.cuh"
#include "launch.hpp"

using pa::BlockManager;
using pa::MgrStatus;

namespace {

constexpr int kRing = 4;  // append staging slots in flight

struct Staging {
  int64_t* host = nullptr;   // pinned: [slots (int64) | cow src,dst (int32)]
  void* dev = nullptr;       // device mirror
  size_t cap = 0;            // bytes
  cudaEvent_t done = nullptr;
  bool pending = false;
};

}  // namespace

struct pa_pool {
  // The host manager: owned by the pool that created it and shared by its
  // layer views (one block table per sequence serves every layer).
  std::unique_ptr<BlockManager> own_mgr;
  BlockManager* mgr = nullptr;
  int32_t num_blocks, block_size, num_kv_heads, head_dim;
  // multi-layer pools: caches [num_layers, ...]; a view addresses one layer
  int32_t num_layers = 1, layer = 0;
  int64_t layer_bytes = 0;        // bytes of one layer of one cache array
  pa_pool* owner = nullptr;       // set on views 1 .. num_layers - 1
  std::vector<pa_pool*> views;    // on the owner: views of layers 1 ..
  pa_dtype dtype;
  void* k_cache = nullptr;
  void* v_cache = nullptr;
  bool device = false;
  int dev_id = 0;
  int sms = 148;
  int32_t* d_err = nullptr;
  bool tmap_ok = false;
  CUtensorMap tmK, tmV;
  // int8 / FP8 pools: the records with a K-codes box and a V-codes + scales box
  CUtensorMap tmRK, tmRV;
  // tensor-core prefill: key-split scratch for one wave (one slot per SM)
  float* split_o = nullptr;
  float* split_ml = nullptr;
  int32_t* tickets = nullptr;
  Staging ring[kRing];
  int ring_next = 0;
  std::vector<int64_t> slots_tmp;
  std::vector<pa::CowPair> cow_tmp;

  pa_pool(int32_t nb, int32_t bs, const std::vector<int32_t>& order)
      : own_mgr(new BlockManager(nb, bs, order)), mgr(own_mgr.get()) {}
  pa_pool() = default;
  pa_pool* base() { return owner ? owner : this; }
};

int pa::pool_device(const pa_pool* p) { return (p && p->device) ? p->dev_id : -1; }

namespace {

pa_status from_mgr(MgrStatus s) {
  switch (s) {
    case MgrStatus::ok: return PA_OK;
    case MgrStatus::unknown_seq: return PA_ERR_UNKNOWN_SEQ;
    case MgrStatus::dup_seq: return PA_ERR_DUP_SEQ;
    case MgrStatus::exhausted: return PA_ERR_POOL_EXHAUSTED;
    default: return PA_ERR_INVALID_ARG;
  }
}

static_assert(pa::kQ8RecordBytes == PA_INT8_RECORD_BYTES, "int8 record size");

// int8 and FP8 pools share one packed record layout
bool is_q8(pa_dtype t) { return t == PA_INT8 || t == PA_FP8; }

size_t elem_bytes(pa_dtype t) { return is_q8(t) ? 1 : t == PA_BF16 ? 2 : 4; }

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() { return pa::tensor_map_encoder(); }

// The pool viewed as a 3-D tensor {head_dim, num_kv_heads, num_blocks *
// block_size}; one box = one block's 16 tokens x 64 columns of one KV head,
// written to shared memory with the 128-byte swizzle.
bool make_pool_map(CUtensorMap* map, void* base, const pa_pool* p) {
  auto fn = encode_fn();
  if (!fn) return false;
  // int8 pools: one box = the block's 16 rows of 128 codes (128 bytes)
  const bool q8 = is_q8(p->dtype);
  const cuuint64_t eb = q8 ? 1 : 2;
  const cuuint64_t dims[3] = {cuuint64_t(p->head_dim), cuuint64_t(p->num_kv_heads),
                              cuuint64_t(p->num_blocks) * p->block_size};
  const cuuint64_t strides[2] = {cuuint64_t(p->head_dim) * eb,
                                 cuuint64_t(p->head_dim) * p->num_kv_heads * eb};
  const cuuint32_t box[3] = {q8 ? 128u : 64u, 1, cuuint32_t(p->block_size)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, q8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  3, base, dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// int8 pools: the packed records viewed as {128 bytes, 33 rows, NB * Hkv};
// one box = `rows` rows of a record (33: the whole record).
bool make_record_map(CUtensorMap* map, void* base, const pa_pool* p, uint32_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, pa::kQ8RecordBytes / 128,
                              cuuint64_t(p->num_blocks) * p->num_kv_heads};
  const cuuint64_t strides[2] = {128, pa::kQ8RecordBytes};
  const cuuint32_t box[3] = {128, rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// All three record maps of an int8 / FP8 pool (or layer): the whole record,
// the K codes (rows 0-15), the V codes with the scale row (rows 16-32).
bool make_record_maps(pa_pool* p) {
  return make_record_map(&p->tmK, p->k_cache, p, pa::kQ8RecordBytes / 128) &&
         make_record_map(&p->tmRK, p->k_cache, p, 16) &&
         make_record_map(&p->tmRV, p->k_cache, p, 17);
}

// Blocks a decode walks per sequence at most: all of them, or with a sink +
// recent window the sink blocks plus the blocks the window can touch.
int32_t window_blocks(const pa_pool* p, int32_t max_blocks, int32_t window, int32_t sinks) {
  if (window <= 0) return max_blocks;
  const int64_t bs = p->block_size;
  const int64_t w = (sinks + bs - 1) / bs + (window + bs - 1) / bs + 1;
  return int32_t(std::min<int64_t>(max_blocks, w));
}

// Blocks per partition for the tensor-core decode.  partition_tokens > 0 is
// taken as given; 0 picks enough partitions for about two resident CTAs per
// SM when the batch has fewer (sequence, KV head) groups than that.
bool decode_partitions(const pa_pool* p, int32_t B, int32_t MB,
                       int32_t partition_tokens, int32_t* part_blocks,
                       int32_t* np) {
  if (partition_tokens > 0) {
    if (partition_tokens % p->block_size) return false;
    *part_blocks = partition_tokens / p->block_size;
  } else {
    const int64_t groups = int64_t(B) * p->num_kv_heads;
    const int64_t target = 2 * int64_t(p->sms);
    int64_t want = 1;
    if (groups > 0 && groups * 5 < target * 4) want = (target + groups - 1) / groups;
    const int64_t max_np = std::max<int64_t>(1, (MB + 15) / 16);
    want = std::min(want, max_np);
    *part_blocks = int32_t((MB + want - 1) / want);
  }
  if (*part_blocks < 1) *part_blocks = 1;
  *np = (MB + *part_blocks - 1) / *part_blocks;
  if (*np < 1) *np = 1;
  return true;
}

bool use_fast_decode(const pa_pool* p, int32_t H) {
  if (is_q8(p->dtype))   // packed records, no tensor maps
    return p->device && H % p->num_kv_heads == 0 && H / p->num_kv_heads <= 8;
  return p->tmap_ok && H % p->num_kv_heads == 0 &&
         pa::decode_fast_supported(p->dtype == PA_BF16, p->head_dim,
                                   p->block_size, H / p->num_kv_heads);
}

bool use_fast_prefill(const pa_pool* p, int32_t H) {
  return p->tmap_ok && H % p->num_kv_heads == 0 &&
         pa::prefill_fast_supported(p->dtype == PA_BF16, p->head_dim,
                                    p->block_size, H / p->num_kv_heads);
}

pa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

void free_split(pa_pool* p) {
  if (p->split_o) cudaFree(p->split_o);
  if (p->split_ml) cudaFree(p->split_ml);
  if (p->tickets) cudaFree(p->tickets);
  p->split_o = p->split_ml = nullptr;
  p->tickets = nullptr;
}

}  // namespace

extern "C" {

// int8 pools pass their packed records as k_cache and no v_cache.
static pa_status create_pool(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                             int32_t head_dim, pa_dtype kv_dtype, void* k_cache, void* v_cache,
                             const int32_t* alloc_order, pa_pool** out) {
  if (!out) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return PA_ERR_INVALID_ARG;
  if (!is_q8(kv_dtype) && (k_cache == nullptr) != (v_cache == nullptr))
    return PA_ERR_INVALID_ARG;
  if (k_cache && (!aligned16(k_cache) || (v_cache && !aligned16(v_cache))))
    return PA_ERR_INVALID_ARG;
  if (int64_t(num_blocks) * block_size > (int64_t(1) << 31) - 1)
    return PA_ERR_INVALID_ARG;
  std::vector<int32_t> order;
  if (alloc_order) {
    if (!BlockManager::is_permutation(alloc_order, num_blocks))
      return PA_ERR_INVALID_ARG;
    order.assign(alloc_order, alloc_order + num_blocks);
  }
  pa_pool* p = new (std::nothrow) pa_pool(num_blocks, block_size, order);
  if (!p) return PA_ERR_INVALID_ARG;
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  p->num_kv_heads = num_kv_heads;
  p->head_dim = head_dim;
  p->dtype = kv_dtype;
  p->k_cache = k_cache;
  p->v_cache = v_cache;
  if (k_cache) {
    p->device = true;
    if (cudaGetDevice(&p->dev_id) != cudaSuccess ||
        cudaDeviceGetAttribute(&p->sms, cudaDevAttrMultiProcessorCount,
                               p->dev_id) != cudaSuccess ||
        cudaMalloc(&p->d_err, sizeof(int32_t)) != cudaSuccess ||
        cudaMemset(p->d_err, 0, sizeof(int32_t)) != cudaSuccess) {
      if (p->d_err) cudaFree(p->d_err);
      delete p;
      return PA_ERR_CUDA;
    }
    if (kv_dtype == PA_BF16 && head_dim == 128 && block_size == 16)
      p->tmap_ok = make_pool_map(&p->tmK, k_cache, p) &&
                   make_pool_map(&p->tmV, v_cache, p);
    if (is_q8(kv_dtype) && !make_record_maps(p)) {
      cudaFree(p->d_err);
      delete p;
      return PA_ERR_CUDA;
    }
    if (p->tmap_ok) {
      // without it the prefill runs unsplit
      const size_t slots = size_t(p->sms);
      if (cudaMalloc(&p->split_o, slots * 2 * 128 * 128 * sizeof(float)) != cudaSuccess ||
          cudaMalloc(&p->split_ml, slots * 2 * 128 * 2 * sizeof(float)) != cudaSuccess ||
          cudaMalloc(&p->tickets, slots * 2 * sizeof(int32_t)) != cudaSuccess ||
          cudaMemset(p->tickets, 0, slots * 2 * sizeof(int32_t)) != cudaSuccess) {
        free_split(p);
        cudaGetLastError();
      }
    }
  }
  *out = p;
  return PA_OK;
}

// Views of layers 1 .. L - 1 of a device pool whose caches hold L layers:
// same manager, error word and prefill scratch; own base pointers, tensor
// maps and append staging.
static pa_status add_layer_views(pa_pool* p, int32_t num_layers) {
  const size_t eb = is_q8(p->dtype) ? 1 : p->dtype == PA_BF16 ? 2 : 4;
  p->num_layers = num_layers;
  p->layer_bytes = is_q8(p->dtype)
                       ? int64_t(p->num_blocks) * p->num_kv_heads * pa::kQ8RecordBytes
                       : int64_t(p->num_blocks) * p->block_size * p->num_kv_heads *
                             p->head_dim * int64_t(eb);
  for (int32_t l = 1; l < num_layers; ++l) {
    pa_pool* v = new (std::nothrow) pa_pool();
    if (!v) return PA_ERR_INVALID_ARG;
    p->views.push_back(v);
    v->mgr = p->mgr;
    v->owner = p;
    v->num_blocks = p->num_blocks;
    v->block_size = p->block_size;
    v->num_kv_heads = p->num_kv_heads;
    v->head_dim = p->head_dim;
    v->dtype = p->dtype;
    v->num_layers = num_layers;
    v->layer = l;
    v->layer_bytes = p->layer_bytes;
    v->device = p->device;
    v->dev_id = p->dev_id;
    v->sms = p->sms;
    v->d_err = p->d_err;
    v->split_o = p->split_o;
    v->split_ml = p->split_ml;
    v->tickets = p->tickets;
    v->k_cache = static_cast<char*>(p->k_cache) + l * p->layer_bytes;
    v->v_cache = p->v_cache ? static_cast<char*>(p->v_cache) + l * p->layer_bytes : nullptr;
    if (is_q8(p->dtype)) {
      if (!make_record_maps(v)) return PA_ERR_CUDA;
    } else if (p->tmap_ok) {
      v->tmap_ok = make_pool_map(&v->tmK, v->k_cache, v) && make_pool_map(&v->tmV, v->v_cache, v);
      if (!v->tmap_ok) return PA_ERR_CUDA;
    }
  }
  return PA_OK;
}

pa_status pa_pool_create_layers(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                                int32_t head_dim, pa_dtype kv_dtype, int32_t num_layers,
                                void* k_cache, void* v_cache, const int32_t* alloc_order,
                                pa_pool** out) {
  if (out) *out = nullptr;
  if (num_layers < 1 || !k_cache) return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_F32 && kv_dtype != PA_BF16 && !is_q8(kv_dtype)) return PA_ERR_INVALID_ARG;
  if (is_q8(kv_dtype) && (block_size != 16 || head_dim != 128)) return PA_ERR_UNSUPPORTED;
  if (is_q8(kv_dtype) && v_cache) return PA_ERR_INVALID_ARG;
  pa_status st = create_pool(num_blocks, block_size, num_kv_heads, head_dim, kv_dtype, k_cache,
                             v_cache, alloc_order, out);
  if (st != PA_OK) return st;
  st = add_layer_views(*out, num_layers);
  if (st != PA_OK) {
    pa_free(*out);
    *out = nullptr;
  }
  return st;
}

pa_status pa_pool_layer(pa_pool* p, int32_t layer, pa_pool** view) {
  if (!p || !view) return PA_ERR_INVALID_ARG;
  *view = nullptr;
  pa_pool* o = p->base();
  if (layer < 0 || layer >= o->num_layers) return PA_ERR_INVALID_ARG;
  *view = layer == 0 ? o : o->views[size_t(layer - 1)];
  return PA_OK;
}

pa_status pa_pool_create(int32_t num_blocks, int32_t block_size,
                         int32_t num_kv_heads, int32_t head_dim,
                         pa_dtype kv_dtype, void* k_cache, void* v_cache,
                         const int32_t* alloc_order, pa_pool** out) {
  if (kv_dtype != PA_F32 && kv_dtype != PA_BF16) {
    if (out) *out = nullptr;
    return PA_ERR_INVALID_ARG;
  }
  return create_pool(num_blocks, block_size, num_kv_heads, head_dim, kv_dtype, k_cache,
                     v_cache, alloc_order, out);
}

pa_status pa_pool_create_int8(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                              int32_t head_dim, void* kv_records, const int32_t* alloc_order,
                              pa_pool** out) {
  if (out) *out = nullptr;
  if (block_size != 16 || head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (!kv_records) return PA_ERR_INVALID_ARG;
  return create_pool(num_blocks, block_size, num_kv_heads, head_dim, PA_INT8, kv_records,
                     nullptr, alloc_order, out);
}

pa_status pa_pool_create_fp8(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                             int32_t head_dim, void* kv_records, const int32_t* alloc_order,
                             pa_pool** out) {
  if (out) *out = nullptr;
  if (block_size != 16 || head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (!kv_records) return PA_ERR_INVALID_ARG;
  return create_pool(num_blocks, block_size, num_kv_heads, head_dim, PA_FP8, kv_records,
                     nullptr, alloc_order, out);
}

static void free_ring(pa_pool* p) {
  for (auto& r : p->ring) {
    if (r.host) cudaFreeHost(r.host);
    if (r.dev) cudaFree(r.dev);
    if (r.done) cudaEventDestroy(r.done);
  }
}

pa_status pa_free(pa_pool* p) {
  if (!p) return PA_OK;
  if (p->owner) return PA_ERR_INVALID_ARG;   // a layer view: freed with its pool
  pa::DeviceScope on_pool_device(pa::pool_device(p));
  if (p->device) {
    cudaDeviceSynchronize();
    for (pa_pool* v : p->views) free_ring(v);
    free_ring(p);
    if (p->d_err) cudaFree(p->d_err);
    free_split(p);
  }
  for (pa_pool* v : p->views) delete v;
  delete p;
  return PA_OK;
}

pa_status pa_seq_create(pa_pool* p, int32_t seq) {
  if (!p) return PA_ERR_INVALID_ARG;
  return from_mgr(p->mgr->create(seq));
}

pa_status pa_seq_fork(pa_pool* p, int32_t parent, int32_t child,
                      int32_t prefix_tokens) {
  if (!p || prefix_tokens < -1) return PA_ERR_INVALID_ARG;
  return from_mgr(p->mgr->share_prefix(parent, child, prefix_tokens));
}

pa_status pa_seq_release(pa_pool* p, int32_t seq) {
  if (!p) return PA_ERR_INVALID_ARG;
  return from_mgr(p->mgr->release(seq));
}

pa_status pa_seq_truncate(pa_pool* p, const int32_t* seqs, const int32_t* lengths,
                          int32_t n) {
  if (!p) return PA_ERR_INVALID_ARG;
  return from_mgr(p->mgr->truncate(seqs, lengths, n));
}

pa_status pa_seq_create_cached(pa_pool* p, int32_t seq, uint64_t scope,
                               uint64_t revision, const int32_t* tokens,
                               int32_t n_tokens, int32_t* hit_tokens) {
  if (!p) return PA_ERR_INVALID_ARG;
  int64_t hit = 0;
  pa_status st = from_mgr(p->mgr->create_cached(seq, scope, revision, tokens, n_tokens, &hit));
  if (st == PA_OK && hit_tokens) *hit_tokens = int32_t(hit);
  return st;
}

pa_status pa_prefix_publish(pa_pool* p, int32_t seq, uint64_t scope,
                            uint64_t revision, const int32_t* tokens,
                            int32_t n_tokens, int32_t* added_blocks) {
  if (!p) return PA_ERR_INVALID_ARG;
  int64_t added = 0;
  pa_status st = from_mgr(p->mgr->publish(seq, scope, revision, tokens, n_tokens, &added));
  if (st == PA_OK && added_blocks) *added_blocks = int32_t(added);
  return st;
}

pa_status pa_prefix_clear(pa_pool* p, int32_t* freed_blocks) {
  if (!p) return PA_ERR_INVALID_ARG;
  const int64_t freed = p->mgr->prefix_clear();
  if (freed_blocks) *freed_blocks = int32_t(freed);
  return PA_OK;
}

int64_t pa_prefix_entries(const pa_pool* p) { return p ? p->mgr->prefix_entries() : 0; }

pa_status pa_seq_table(const pa_pool* p, int32_t seq, int32_t* blocks_out,
                       int32_t cap, int32_t* n_blocks, int32_t* length) {
  if (!p) return PA_ERR_INVALID_ARG;
  const std::vector<int32_t>* t = p->mgr->table(seq);
  if (!t) return PA_ERR_UNKNOWN_SEQ;
  if (n_blocks) *n_blocks = int32_t(t->size());
  if (length) *length = int32_t(p->mgr->length(seq));
  if (blocks_out) {
    if (cap < int32_t(t->size())) return PA_ERR_INVALID_ARG;
    std::copy(t->begin(), t->end(), blocks_out);
  }
  return PA_OK;
}

pa_status pa_block_tables(const pa_pool* p, const int32_t* seqs, int32_t n,
                          int32_t width, int32_t* tables_out,
                          int32_t* kv_lens_out) {
  if (!p || n < 0 || width <= 0 || (n > 0 && !seqs)) return PA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const std::vector<int32_t>* t = p->mgr->table(seqs[i]);
    if (!t) return PA_ERR_UNKNOWN_SEQ;
    if (int32_t(t->size()) > width) return PA_ERR_INVALID_ARG;
  }
  for (int32_t i = 0; i < n; ++i) {
    const std::vector<int32_t>* t = p->mgr->table(seqs[i]);
    if (tables_out) {
      int32_t* row = tables_out + int64_t(i) * width;
      std::fill(row, row + width, 0);
      std::copy(t->begin(), t->end(), row);
    }
    if (kv_lens_out) kv_lens_out[i] = int32_t(p->mgr->length(seqs[i]));
  }
  return PA_OK;
}

pa_status pa_plan_append(pa_pool* p, const int32_t* seqs, const int32_t* n_new,
                         int32_t n_seqs, int64_t* slot_mapping_out,
                         int32_t* cow_src_out, int32_t* cow_dst_out,
                         int32_t cow_cap, int32_t* n_cow_out) {
  if (!p || n_seqs < 0 || (n_seqs > 0 && (!seqs || !n_new)))
    return PA_ERR_INVALID_ARG;
  if ((cow_src_out || cow_dst_out) && cow_cap < n_seqs) return PA_ERR_INVALID_ARG;
  p->slots_tmp.clear();
  p->cow_tmp.clear();
  pa_status st = from_mgr(p->mgr->append(seqs, n_new, n_seqs, &p->slots_tmp, &p->cow_tmp));
  if (st != PA_OK) return st;
  if (slot_mapping_out)
    std::copy(p->slots_tmp.begin(), p->slots_tmp.end(), slot_mapping_out);
  for (size_t i = 0; i < p->cow_tmp.size(); ++i) {
    if (cow_src_out) cow_src_out[i] = p->cow_tmp[i].src;
    if (cow_dst_out) cow_dst_out[i] = p->cow_tmp[i].dst;
  }
  if (n_cow_out) *n_cow_out = int32_t(p->cow_tmp.size());
  return PA_OK;
}

pa_status pa_pool_stats(const pa_pool* p, pa_stats* out) {
  if (!p || !out) return PA_ERR_INVALID_ARG;
  pa::Snapshot s = p->mgr->snapshot();
  out->allocated_blocks = s.allocated;
  out->free_blocks = s.free;
  out->physical_capacity_tokens = s.capacity;
  out->physical_payload_tokens = s.payload;
  out->logical_tokens = s.logical;
  out->internal_waste_tokens = s.waste;
  out->sharing_savings_tokens = s.savings;
  out->live_sequences = s.live;
  return PA_OK;
}

pa_status pa_refcounts(const pa_pool* p, int32_t* out) {
  if (!p || !out) return PA_ERR_INVALID_ARG;
  const auto& r = p->mgr->refcounts();
  std::copy(r.begin(), r.end(), out);
  return PA_OK;
}

pa_status pa_validate(const pa_pool* p) {
  if (!p) return PA_ERR_INVALID_ARG;
  return p->mgr->validate() ? PA_OK : PA_ERR_INTERNAL;
}

// K2 for any pool: whole blocks of codes/values (and, for int8 pools, of
// their scales).
static cudaError_t cow_blocks(pa_pool* p, const int32_t* d_src, const int32_t* d_dst, int32_t n,
                              cudaStream_t s) {
  // the tables are shared by every layer: a copied block is copied in all
  pa_pool* o = p->base();
  cudaError_t e = cudaSuccess;
  for (int32_t l = 0; l < o->num_layers && e == cudaSuccess; ++l) {
    char* kc = static_cast<char*>(o->k_cache) + l * o->layer_bytes;
    char* vc = o->v_cache ? static_cast<char*>(o->v_cache) + l * o->layer_bytes : nullptr;
    if (is_q8(o->dtype))   // one array of packed records
      e = pa::launch_cow_copy(kc, nullptr, d_src, d_dst, n,
                              int64_t(o->num_kv_heads) * pa::kQ8RecordBytes, o->num_blocks,
                              o->d_err, o->sms, s);
    else
      e = pa::launch_cow_copy(kc, vc, d_src, d_dst, n,
                              int64_t(o->block_size) * o->num_kv_heads * o->head_dim *
                                  elem_bytes(o->dtype),
                              o->num_blocks, o->d_err, o->sms, s);
  }
  return e;
}

// K1 for any pool: copies rows, or quantises bf16 rows into an int8 or FP8
// pool.
static cudaError_t write_rows(pa_pool* p, const void* key, const void* value,
                              const int64_t* d_slots, int32_t T, cudaStream_t s) {
  const int64_t num_slots = int64_t(p->num_blocks) * p->block_size;
  if (is_q8(p->dtype))
    return pa::launch_reshape_and_cache_q8(key, value, p->k_cache, d_slots, T,
                                           p->num_kv_heads, num_slots, p->dtype == PA_FP8,
                                           p->d_err, p->sms, s);
  return pa::launch_reshape_and_cache(key, value, p->k_cache, p->v_cache, d_slots, T,
                                      int64_t(p->num_kv_heads) * p->head_dim *
                                          elem_bytes(p->dtype),
                                      num_slots, p->d_err, p->sms, s);
}

pa_status pa_append_kv(pa_pool* p, const int32_t* seqs, const int32_t* n_new,
                       int32_t n_seqs, const void* key, const void* value,
                       int64_t* slot_mapping_out, void* stream) {
  if (!p) return PA_ERR_INVALID_ARG;
  if (!p->device) return PA_ERR_NO_DEVICE;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (n_seqs < 0 || (n_seqs > 0 && (!seqs || !n_new))) return PA_ERR_INVALID_ARG;
  int64_t T = 0;
  for (int32_t i = 0; i < n_seqs; ++i) T += std::max<int32_t>(0, n_new[i]);
  if (T > 0 && (!key || !value)) return PA_ERR_INVALID_ARG;
  if (T > INT32_MAX) return PA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // staging slot: wait until the kernels of its previous use are done
  Staging& r = p->ring[p->ring_next];
  if (r.pending && cudaEventSynchronize(r.done) != cudaSuccess) return PA_ERR_CUDA;
  r.pending = false;
  const size_t need = size_t(T) * sizeof(int64_t) + size_t(n_seqs) * 2 * sizeof(int32_t);
  if (need > r.cap) {
    size_t cap = std::max<size_t>(need, 4096);
    cap = std::max(cap, r.cap * 2);
    if (r.host) cudaFreeHost(r.host);
    if (r.dev) cudaFree(r.dev);
    r.host = nullptr;
    r.dev = nullptr;
    r.cap = 0;
    if (cudaMallocHost(reinterpret_cast<void**>(&r.host), cap) != cudaSuccess)
      return PA_ERR_CUDA;
    if (cudaMalloc(&r.dev, cap) != cudaSuccess) return PA_ERR_CUDA;
    r.cap = cap;
    if (!r.done && cudaEventCreateWithFlags(&r.done, cudaEventDisableTiming) != cudaSuccess)
      return PA_ERR_CUDA;
  }

  // host plan (step a1): all-or-nothing
  p->slots_tmp.clear();
  p->cow_tmp.clear();
  pa_status st = from_mgr(p->mgr->append(seqs, n_new, n_seqs, &p->slots_tmp, &p->cow_tmp));
  if (st != PA_OK) return st;
  if (slot_mapping_out)
    std::copy(p->slots_tmp.begin(), p->slots_tmp.end(), slot_mapping_out);
  const int32_t n_cow = int32_t(p->cow_tmp.size());
  int64_t* hs = r.host;
  std::copy(p->slots_tmp.begin(), p->slots_tmp.end(), hs);
  int32_t* hc = reinterpret_cast<int32_t*>(hs + T);
  for (int32_t i = 0; i < n_cow; ++i) {
    hc[i] = p->cow_tmp[i].src;
    hc[n_cow + i] = p->cow_tmp[i].dst;
  }
  const size_t bytes = size_t(T) * sizeof(int64_t) + size_t(n_cow) * 2 * sizeof(int32_t);
  if (bytes && cudaMemcpyAsync(r.dev, r.host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return PA_ERR_CUDA;
  const int64_t* d_slots = static_cast<const int64_t*>(r.dev);
  const int32_t* d_cow = reinterpret_cast<const int32_t*>(d_slots + T);
  cudaError_t e = cow_blocks(p, d_cow, d_cow + n_cow, n_cow, s);
  if (e == cudaSuccess) e = write_rows(p, key, value, d_slots, int32_t(T), s);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  if (cudaEventRecord(r.done, s) != cudaSuccess) return PA_ERR_CUDA;
  r.pending = true;
  p->ring_next = (p->ring_next + 1) % kRing;
  return PA_OK;
}

pa_status pa_reshape_and_cache(pa_pool* p, const void* key, const void* value,
                               const int64_t* d_slot_mapping, int32_t T,
                               void* stream) {
  if (!p) return PA_ERR_INVALID_ARG;
  if (!p->device) return PA_ERR_NO_DEVICE;
  if (T < 0 || (T > 0 && (!key || !value || !d_slot_mapping))) return PA_ERR_INVALID_ARG;
  pa::DeviceScope on_pool_device(p->dev_id);
  return cuda_status(write_rows(p, key, value, d_slot_mapping, T,
                                static_cast<cudaStream_t>(stream)));
}

pa_status pa_cow_copy(pa_pool* p, const int32_t* d_src, const int32_t* d_dst,
                      int32_t n, void* stream) {
  if (!p) return PA_ERR_INVALID_ARG;
  if (!p->device) return PA_ERR_NO_DEVICE;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (n < 0 || (n > 0 && (!d_src || !d_dst))) return PA_ERR_INVALID_ARG;
  return cuda_status(cow_blocks(p, d_src, d_dst, n, static_cast<cudaStream_t>(stream)));
}

size_t pa_decode_workspace_bytes(const pa_pool* p, int32_t B, int32_t H,
                                 int32_t max_blocks, int32_t partition_tokens) {
  if (!p || B <= 0 || H <= 0 || max_blocks <= 0) return 0;
  if (!use_fast_decode(p, H)) return 0;
  int32_t pb = 0, np = 1;
  if (!decode_partitions(p, B, max_blocks, partition_tokens, &pb, &np)) return 0;
  size_t bytes = pa::split_workspace_bytes(B, H, np, p->head_dim);
  if (pa::decode_wants_order(B, p->num_kv_heads, np, p->sms))
    bytes += pa::order_workspace_bytes(B);
  return bytes;
}

int32_t pa_decode_path(const pa_pool* p, int32_t H) {
  return (p && use_fast_decode(p, H)) ? 1 : 0;
}

int32_t pa_prefill_path(const pa_pool* p, int32_t H) {
  return (p && use_fast_prefill(p, H)) ? 1 : 0;
}

// The CUDA-core path: any pool dtype (int8 / FP8 records dequantised element
// by element, bf16 queries), any head_dim <= 512, block or group size.
static pa::GenericArgs generic_args(const pa_pool* p, const void* q, int32_t B,
                                    int32_t q_tokens, int32_t H, const int32_t* tables,
                                    int32_t max_blocks, const int32_t* kv_lens, float scale,
                                    float* out) {
  pa::GenericArgs g{q, p->k_cache, p->v_cache, tables, max_blocks,
                    kv_lens, B, q_tokens, H, p->num_kv_heads, p->head_dim,
                    p->block_size, p->num_blocks, scale, out, p->d_err,
                    p->dtype == PA_BF16, 0};
  if (is_q8(p->dtype)) g.q8 = p->dtype == PA_FP8 ? 2 : 1;
  return g;
}

static pa_status decode_fast(pa_pool* p, const void* q, int32_t B, int32_t H,
                             const int32_t* d_block_tables, int32_t max_blocks,
                             const int32_t* d_kv_lens, float scale, int32_t partition_tokens,
                             void* workspace, size_t workspace_bytes, float* out,
                             void* stream, const void* new_k, const void* new_v,
                             const int64_t* new_slots, int32_t window = 0, int32_t sinks = 0) {
  if (!aligned16(q)) return PA_ERR_INVALID_ARG;
  pa::DecodeArgs a{};
  // partitions split the walked (visible) blocks
  const int32_t walk = window_blocks(p, max_blocks, window, sinks);
  if (!decode_partitions(p, B, walk, partition_tokens, &a.part_blocks, &a.NP))
    return PA_ERR_INVALID_ARG;
  const size_t split_bytes = pa::split_workspace_bytes(B, H, a.NP, p->head_dim);
  const bool order = pa::decode_wants_order(B, p->num_kv_heads, a.NP, p->sms);
  const size_t need = split_bytes + (order ? pa::order_workspace_bytes(B) : 0);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return PA_ERR_INVALID_ARG;
  a.order = order ? reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + split_bytes)
                  : nullptr;
  a.q = q;
  a.tables = d_block_tables;
  a.MB = max_blocks;
  a.kv_lens = d_kv_lens;
  a.B = B;
  a.H = H;
  a.Hkv = p->num_kv_heads;
  a.NB = p->num_blocks;
  a.scale = scale;
  a.out = out;
  a.ws = static_cast<float*>(workspace);
  a.err = p->d_err;
  a.new_k = new_k;
  a.new_v = new_v;
  a.new_slots = new_slots;
  a.k_cache = p->k_cache;
  a.v_cache = p->v_cache;
  a.window = window;
  a.sinks = sinks;
  if (is_q8(p->dtype)) {
    // Groups of up to 4 heads: tcgen05 MMAs straight from the codes (a 128-key
    // group per MMA; the per-byte softmax work grows with the group).  Larger
    // groups: the warp-level kernel, whose 8-column MMA tiles they fill.
    const bool fp8 = p->dtype == PA_FP8;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return cuda_status(H / p->num_kv_heads <= 4
                           ? pa::launch_decode_q8tc(&p->tmRK, &p->tmRV, a, fp8, s)
                           : pa::launch_decode_q8(&p->tmK, a, fp8, s));
  }
  return cuda_status(pa::launch_decode_fast(&p->tmK, &p->tmV, a, p->sms,
                                            static_cast<cudaStream_t>(stream)));
}

static pa_status check_attention_args(const pa_pool* p, const void* q, int32_t B,
                                      int32_t H, const int32_t* tables,
                                      int32_t MB, const int32_t* kv_lens,
                                      const float* out) {
  if (!p) return PA_ERR_INVALID_ARG;
  if (!p->device) return PA_ERR_NO_DEVICE;
  if (B < 0 || H <= 0 || MB <= 0 || H % p->num_kv_heads) return PA_ERR_INVALID_ARG;
  if (B > 0 && (!q || !tables || !kv_lens || !out)) return PA_ERR_INVALID_ARG;
  if (int64_t(MB) * p->block_size > INT32_MAX) return PA_ERR_INVALID_ARG;
  if (p->head_dim > 512) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

pa_status pa_decode(pa_pool* p, const void* q, int32_t B, int32_t H,
                    const int32_t* d_block_tables, int32_t max_blocks,
                    const int32_t* d_kv_lens, float scale,
                    int32_t partition_tokens, void* workspace,
                    size_t workspace_bytes, float* out, void* stream) {
  pa_status st = check_attention_args(p, q, B, H, d_block_tables, max_blocks,
                                      d_kv_lens, out);
  if (st != PA_OK) return st;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (partition_tokens < 0) return PA_ERR_INVALID_ARG;
  if (B == 0) return PA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_fast_decode(p, H))
    return decode_fast(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, scale,
                       partition_tokens, workspace, workspace_bytes, out, stream, nullptr,
                       nullptr, nullptr);
  if (partition_tokens % p->block_size) return PA_ERR_INVALID_ARG;
  return cuda_status(pa::launch_attention_generic(
      generic_args(p, q, B, 1, H, d_block_tables, max_blocks, d_kv_lens, scale, out), s));
}

size_t pa_decode_window_workspace_bytes(const pa_pool* p, int32_t B, int32_t H,
                                        int32_t max_blocks, int32_t window, int32_t sinks,
                                        int32_t partition_tokens) {
  if (!p || window < 1 || sinks < 0) return 0;
  return pa_decode_workspace_bytes(p, B, H, window_blocks(p, max_blocks, window, sinks),
                                   partition_tokens);
}

pa_status pa_decode_window(pa_pool* p, const void* q, int32_t B, int32_t H,
                           const int32_t* d_block_tables, int32_t max_blocks,
                           const int32_t* d_kv_lens, float scale, int32_t window, int32_t sinks,
                           int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                           float* out, void* stream) {
  pa_status st = check_attention_args(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, out);
  if (st != PA_OK) return st;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (partition_tokens < 0 || window < 1 || sinks < 0) return PA_ERR_INVALID_ARG;
  if (B == 0) return PA_OK;
  if (!use_fast_decode(p, H)) {
    if (partition_tokens % p->block_size) return PA_ERR_INVALID_ARG;
    pa::GenericArgs g =
        generic_args(p, q, B, 1, H, d_block_tables, max_blocks, d_kv_lens, scale, out);
    g.window = window;
    g.sinks = sinks;
    return cuda_status(pa::launch_attention_generic(g, static_cast<cudaStream_t>(stream)));
  }
  return decode_fast(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, scale, partition_tokens,
                     workspace, workspace_bytes, out, stream, nullptr, nullptr, nullptr, window,
                     sinks);
}

pa_status pa_decode_append(pa_pool* p, const void* q, const void* key, const void* value,
                           const int64_t* d_slot_mapping, int32_t B, int32_t H,
                           const int32_t* d_block_tables, int32_t max_blocks,
                           const int32_t* d_kv_lens, float scale, int32_t partition_tokens,
                           void* workspace, size_t workspace_bytes, float* out, void* stream) {
  pa_status st = check_attention_args(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, out);
  if (st != PA_OK) return st;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (B > 0 && (!key || !value || !d_slot_mapping)) return PA_ERR_INVALID_ARG;
  if (partition_tokens < 0) return PA_ERR_INVALID_ARG;
  if (B == 0) return PA_OK;
  if (!use_fast_decode(p, H) || is_q8(p->dtype)) {
    // same result in two launches on the other paths
    st = pa_reshape_and_cache(p, key, value, d_slot_mapping, B, stream);
    if (st != PA_OK) return st;
    return pa_decode(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, scale,
                     partition_tokens, workspace, workspace_bytes, out, stream);
  }
  if (!aligned16(key) || !aligned16(value)) return PA_ERR_INVALID_ARG;
  return decode_fast(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, scale,
                     partition_tokens, workspace, workspace_bytes, out, stream, key, value,
                     d_slot_mapping);
}

pa_status pa_decode_window_append(pa_pool* p, const void* q, const void* key,
                                  const void* value, const int64_t* d_slot_mapping, int32_t B,
                                  int32_t H, const int32_t* d_block_tables, int32_t max_blocks,
                                  const int32_t* d_kv_lens, float scale, int32_t window,
                                  int32_t sinks, int32_t partition_tokens, void* workspace,
                                  size_t workspace_bytes, float* out, void* stream) {
  pa_status st = check_attention_args(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, out);
  if (st != PA_OK) return st;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (B > 0 && (!key || !value || !d_slot_mapping)) return PA_ERR_INVALID_ARG;
  if (partition_tokens < 0 || window < 1 || sinks < 0) return PA_ERR_INVALID_ARG;
  if (B == 0) return PA_OK;
  if (is_q8(p->dtype) || !use_fast_decode(p, H)) {
    // the quantising append is its own launch on an int8 / FP8 pool, and the
    // CUDA-core path decodes after a separate append
    st = pa_reshape_and_cache(p, key, value, d_slot_mapping, B, stream);
    if (st != PA_OK) return st;
    return pa_decode_window(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, scale, window,
                            sinks, partition_tokens, workspace, workspace_bytes, out, stream);
  }
  if (!aligned16(key) || !aligned16(value)) return PA_ERR_INVALID_ARG;
  // the newest key is always visible, so the CTA that walks the last
  // visible block is the one that writes and patches the new row
  return decode_fast(p, q, B, H, d_block_tables, max_blocks, d_kv_lens, scale, partition_tokens,
                     workspace, workspace_bytes, out, stream, key, value, d_slot_mapping, window,
                     sinks);
}

pa_status pa_prefill_chunk(pa_pool* p, const void* q, int32_t B,
                           int32_t q_tokens, int32_t H,
                           const int32_t* d_block_tables, int32_t max_blocks,
                           const int32_t* d_kv_lens, float scale,
                           int32_t max_kv_splits, float* out, void* stream) {
  pa_status st = check_attention_args(p, q, B, H, d_block_tables, max_blocks,
                                      d_kv_lens, out);
  if (st != PA_OK) return st;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (q_tokens <= 0 || q_tokens > 65535 || max_kv_splits < 0) return PA_ERR_INVALID_ARG;
  if (B == 0) return PA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!is_q8(p->dtype) && use_fast_prefill(p, H)) {
    if (!aligned16(q)) return PA_ERR_INVALID_ARG;
    pa::PrefillArgs a{q, d_block_tables, max_blocks, d_kv_lens, B, q_tokens, H,
                      p->num_kv_heads, p->num_blocks, scale, out, p->d_err,
                      max_kv_splits, p->split_o, p->split_ml, p->tickets,
                      p->split_o ? p->sms : 0};
    return cuda_status(pa::launch_prefill_fast(&p->tmK, &p->tmV, a, p->sms, s));
  }
  return cuda_status(pa::launch_attention_generic(
      generic_args(p, q, B, q_tokens, H, d_block_tables, max_blocks, d_kv_lens, scale, out),
      s));
}

}  // extern "C"

// ---- prepared decode batch ---------------------------------------------------
//
// One serving decode step per call.  The batch keeps, on the device, the
// block tables and scratch of a fixed list of sequences, and a host mirror of
// the tables; each step plans one new token per sequence on the host manager,
// finds the table entries that changed (the copied tail and a new block, at
// the end of each row), stages plan and patches in one pinned buffer, and
// queues: the uploads (plan, patches, q, new K/V) on an upload stream, the
// patch kernel, copy-on-write copies and the fused append + decode on the
// caller's stream, and the download of the output on a download stream.  Two
// sets of device buffers alternate between steps, so one step's transfers
// overlap the neighbouring steps' kernels.

namespace {

constexpr int kBatchSets = 2;
// Largest step upload that one kernel reads from host memory (above it, copies).
constexpr size_t kUploadKernelMaxBytes = size_t(1) << 20;

struct BatchSet {
  void* d_q = nullptr;       // [n, H, d] pool dtype (bf16 on int8 / FP8 pools)
  void* d_k = nullptr;       // [n, Hkv, d]
  void* d_v = nullptr;
  float* d_out = nullptr;    // [n, H, d]
  char* d_stage = nullptr;   // slots int64 [n] | lens [n] | cow src [n] | dst [n] | patches
  char* h_stage = nullptr;   // pinned mirror of d_stage
  const char* h_stage_dev = nullptr;   // its mapped device address (null: not mapped)
  cudaEvent_t up = nullptr, done = nullptr, down = nullptr;
  bool used = false;
};

}  // namespace

struct pa_batch {
  pa_pool* pool = nullptr;
  std::vector<int32_t> seqs, ones;
  int32_t n = 0, H = 0, MB = 0, part = 0;
  int32_t window = 0, sinks = 0;         // sink + recent window (0: full attention)
  size_t q_bytes = 0, kv_bytes = 0, out_bytes = 0, stage_bytes = 0;
  int32_t patch_cap = 0;                 // (row, index, value) triples per step
  int32_t* d_tables = nullptr;           // [n, MB]
  void* d_ws = nullptr;
  size_t ws_bytes = 0;
  cudaStream_t up = nullptr, down = nullptr;
  std::vector<int32_t> mirror;           // host copy of d_tables
  std::vector<int32_t> mirror_blocks;    // entries of each row the device holds
  std::vector<int64_t> mirror_len;       // sequence length the mirror reflects
  std::vector<int64_t> slots_tmp;
  std::vector<pa::CowPair> cow_tmp;
  std::vector<int32_t> patches;
  BatchSet set[kBatchSets];
  int64_t steps = 0;
  // The last step's output is downloaded by the next step call, after that
  // step's uploads, or by pa_batch_sync: the download waits for the step's
  // kernels, and when the two copy streams share one hardware queue a copy
  // queued ahead of the next uploads holds them up until those kernels end.
  int32_t pending = -1;                  // set of the step whose output is not queued yet
  float* pending_out = nullptr;
};

namespace {

// The device address of pinned host memory mapped into the current device's
// address space, or null (pageable memory, or not visible to this device).
const void* mapped_host(const void* h) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, h) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

// Queue the download of the output of set k's last step into h_out, after
// that step's kernels.
bool queue_download(pa_batch* b, int32_t k, float* h_out) {
  BatchSet& S = b->set[k];
  return cudaStreamWaitEvent(b->down, S.done, 0) == cudaSuccess &&
         cudaMemcpyAsync(h_out, S.d_out, b->out_bytes, cudaMemcpyDeviceToHost, b->down) ==
             cudaSuccess &&
         cudaEventRecord(S.down, b->down) == cudaSuccess;
}

bool flush_download(pa_batch* b) {
  if (b->pending < 0) return true;
  const bool ok = queue_download(b, b->pending, b->pending_out);
  b->pending = -1;
  return ok;
}

void free_batch(pa_batch* b) {
  for (auto& s : b->set) {
    cudaFree(s.d_q);
    cudaFree(s.d_k);
    cudaFree(s.d_v);
    cudaFree(s.d_out);
    cudaFree(s.d_stage);
    if (s.h_stage) cudaFreeHost(s.h_stage);
    if (s.up) cudaEventDestroy(s.up);
    if (s.done) cudaEventDestroy(s.done);
    if (s.down) cudaEventDestroy(s.down);
  }
  cudaFree(b->d_tables);
  cudaFree(b->d_ws);
  if (b->up) cudaStreamDestroy(b->up);
  if (b->down) cudaStreamDestroy(b->down);
  delete b;
}

}  // namespace

extern "C" {

pa_status pa_batch_create(pa_pool* p, const int32_t* seqs, int32_t n, int32_t H,
                          int32_t max_blocks, int32_t partition_tokens, pa_batch** out) {
  if (!out) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!p) return PA_ERR_INVALID_ARG;
  if (!p->device) return PA_ERR_NO_DEVICE;
  if (n <= 0 || !seqs || H <= 0 || H % p->num_kv_heads || max_blocks <= 0 ||
      partition_tokens < 0 || int64_t(max_blocks) * p->block_size > INT32_MAX)
    return PA_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const std::vector<int32_t>* t = p->mgr->table(seqs[i]);
    if (!t) return PA_ERR_UNKNOWN_SEQ;
    if (int32_t(t->size()) > max_blocks) return PA_ERR_INVALID_ARG;
    for (int32_t k = 0; k < i; ++k)
      if (seqs[k] == seqs[i]) return PA_ERR_INVALID_ARG;   // a sequence once
  }
  pa::DeviceScope on_pool_device(p->dev_id);
  pa_batch* b = new (std::nothrow) pa_batch();
  if (!b) return PA_ERR_INVALID_ARG;
  b->pool = p;
  b->seqs.assign(seqs, seqs + n);
  b->ones.assign(size_t(n), 1);
  b->n = n;
  b->H = H;
  b->MB = max_blocks;
  b->part = partition_tokens;
  const size_t eq = p->dtype == PA_F32 ? 4 : 2;   // queries and new rows: pool dtype, bf16 for codes
  b->q_bytes = size_t(n) * H * p->head_dim * eq;
  b->kv_bytes = size_t(n) * p->num_kv_heads * p->head_dim * eq;
  b->out_bytes = size_t(n) * H * p->head_dim * sizeof(float);
  b->patch_cap = 4 * n;
  b->stage_bytes = (size_t(n) * (8 + 4 + 8) + size_t(b->patch_cap) * 12 + 15) & ~size_t(15);
  b->ws_bytes = pa_decode_workspace_bytes(p, n, H, max_blocks, partition_tokens);
  // the upload stream at the greatest priority: its kernel takes the first SM
  // slot that frees up, ahead of the rest of a decode grid
  int least_prio = 0, greatest_prio = 0;
  cudaDeviceGetStreamPriorityRange(&least_prio, &greatest_prio);
  bool ok = cudaStreamCreateWithPriority(&b->up, cudaStreamNonBlocking, greatest_prio) ==
                cudaSuccess &&
            cudaStreamCreateWithFlags(&b->down, cudaStreamNonBlocking) == cudaSuccess &&
            cudaMalloc(&b->d_tables, size_t(n) * max_blocks * sizeof(int32_t)) == cudaSuccess &&
            (b->ws_bytes == 0 || cudaMalloc(&b->d_ws, b->ws_bytes) == cudaSuccess);
  for (auto& s : b->set) {
    ok = ok && cudaMalloc(&s.d_q, b->q_bytes) == cudaSuccess &&
         cudaMalloc(&s.d_k, b->kv_bytes) == cudaSuccess &&
         cudaMalloc(&s.d_v, b->kv_bytes) == cudaSuccess &&
         cudaMalloc(reinterpret_cast<void**>(&s.d_out), b->out_bytes) == cudaSuccess &&
         cudaMalloc(reinterpret_cast<void**>(&s.d_stage), b->stage_bytes) == cudaSuccess &&
         cudaMallocHost(reinterpret_cast<void**>(&s.h_stage), b->stage_bytes) == cudaSuccess &&
         cudaEventCreateWithFlags(&s.up, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&s.done, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&s.down, cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    free_batch(b);
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  for (auto& s : b->set) {
    void* dev = nullptr;
    if (cudaHostGetDevicePointer(&dev, s.h_stage, 0) == cudaSuccess)
      s.h_stage_dev = static_cast<const char*>(dev);
    else
      cudaGetLastError();                // not mapped: the step copies it
  }
  // the tables as they stand, uploaded once
  b->mirror.assign(size_t(n) * max_blocks, 0);
  b->mirror_blocks.assign(size_t(n), 0);
  b->mirror_len.assign(size_t(n), 0);
  for (int32_t i = 0; i < n; ++i) {
    const std::vector<int32_t>* t = p->mgr->table(seqs[i]);
    std::copy(t->begin(), t->end(), b->mirror.begin() + int64_t(i) * max_blocks);
    b->mirror_blocks[size_t(i)] = int32_t(t->size());
    b->mirror_len[size_t(i)] = p->mgr->length(seqs[i]);
  }
  if (cudaMemcpy(b->d_tables, b->mirror.data(), b->mirror.size() * sizeof(int32_t),
                 cudaMemcpyHostToDevice) != cudaSuccess) {
    free_batch(b);
    return PA_ERR_CUDA;
  }
  *out = b;
  return PA_OK;
}

pa_status pa_batch_step(pa_batch* b, const void* h_q, const void* h_key, const void* h_value,
                        float scale, float* h_out, void* stream) {
  if (!b || !h_q || !h_key || !h_value || !h_out) return PA_ERR_INVALID_ARG;
  pa_pool* p = b->pool;
  pa::DeviceScope on_pool_device(p->dev_id);
  const int32_t n = b->n, MB = b->MB;
  // every sequence must still be live and have room for one more token
  for (int32_t i = 0; i < n; ++i) {
    if (!p->mgr->table(b->seqs[size_t(i)])) return PA_ERR_UNKNOWN_SEQ;
    if (p->mgr->length(b->seqs[size_t(i)]) + 1 > int64_t(MB) * p->block_size)
      return PA_ERR_INVALID_ARG;
  }
  BatchSet& S = b->set[b->steps % kBatchSets];
  // the pinned staging of this set is rewritten only after its last upload ran
  if (S.used && cudaEventSynchronize(S.up) != cudaSuccess) return PA_ERR_CUDA;

  // step a1 on the host: one token per sequence, all-or-nothing
  b->slots_tmp.clear();
  b->cow_tmp.clear();
  pa_status st = from_mgr(p->mgr->append(b->seqs.data(), b->ones.data(), n, &b->slots_tmp,
                                         &b->cow_tmp));
  if (st != PA_OK) return st;

  // table entries that differ from the device copy: the changes of an append
  // (a copied tail, a new block) lie at the end of a row; a row whose length
  // moved by anything but this step (a rollback) is compared whole
  b->patches.clear();
  bool full_upload = false;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t seq = b->seqs[size_t(i)];
    const std::vector<int32_t>& t = *p->mgr->table(seq);
    const int64_t len = p->mgr->length(seq);
    const int32_t size = int32_t(t.size());
    int32_t from = 0;
    if (len - 1 == b->mirror_len[size_t(i)])
      from = std::max(0, std::min(b->mirror_blocks[size_t(i)], size) - 1);
    int32_t* row = b->mirror.data() + int64_t(i) * MB;
    for (int32_t j = from; j < size; ++j) {
      if (row[j] != t[size_t(j)]) {
        row[j] = t[size_t(j)];
        if (int32_t(b->patches.size()) < 3 * b->patch_cap) {
          b->patches.push_back(i);
          b->patches.push_back(j);
          b->patches.push_back(t[size_t(j)]);
        } else {
          full_upload = true;
        }
      }
    }
    b->mirror_blocks[size_t(i)] = size;
    b->mirror_len[size_t(i)] = len;
  }
  const int32_t ncow = int32_t(b->cow_tmp.size());
  const int32_t npatch = full_upload ? 0 : int32_t(b->patches.size() / 3);
  // staging: slots | lens | cow src | cow dst | patches
  int64_t* slots = reinterpret_cast<int64_t*>(S.h_stage);
  int32_t* lens = reinterpret_cast<int32_t*>(slots + n);
  int32_t* csrc = lens + n;
  int32_t* cdst = csrc + n;
  int32_t* pat = cdst + n;
  std::copy(b->slots_tmp.begin(), b->slots_tmp.end(), slots);
  for (int32_t i = 0; i < n; ++i) lens[i] = int32_t(b->mirror_len[size_t(i)]);
  for (int32_t c = 0; c < ncow; ++c) {
    csrc[c] = b->cow_tmp[size_t(c)].src;
    cdst[c] = b->cow_tmp[size_t(c)].dst;
  }
  std::copy(b->patches.begin(), b->patches.begin() + 3 * npatch, pat);
  const size_t staged = size_t(n) * 20 + size_t(npatch) * 12;
  const int64_t* d_slots = reinterpret_cast<const int64_t*>(S.d_stage);
  const int32_t* d_lens = reinterpret_cast<const int32_t*>(d_slots + n);
  const int32_t* d_csrc = d_lens + n;
  const int32_t* d_cdst = d_csrc + n;
  const int32_t* d_pat = d_cdst + n;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bool ok = true;
  // uploads, once this set's buffers are no longer read by its last step:
  // one kernel that reads the four host buffers where all are pinned and
  // mapped, 16-byte aligned and whole 16-byte units long; else four copies.
  // The kernel saves the copies' fixed costs, which dominate small uploads;
  // its CTAs hold SM slots for as long as the PCIe reads take, so large
  // uploads (and every upload on quantised pools, whose decode fills the SMs'
  // shared memory) go to the copy engines, which leave the decode alone.
  if (S.used) ok = cudaStreamWaitEvent(b->up, S.done, 0) == cudaSuccess;
  const size_t staged16 = (staged + 15) & ~size_t(15);
  const bool try_launch = !is_q8(p->dtype) &&
                          staged16 + b->q_bytes + 2 * b->kv_bytes <= kUploadKernelMaxBytes;
  const void* src[4] = {S.h_stage_dev, try_launch ? mapped_host(h_q) : nullptr,
                        try_launch ? mapped_host(h_key) : nullptr,
                        try_launch ? mapped_host(h_value) : nullptr};
  void* dst[4] = {S.d_stage, S.d_q, S.d_k, S.d_v};
  const size_t len[4] = {staged16, b->q_bytes, b->kv_bytes, b->kv_bytes};
  bool one_launch = try_launch;
  for (int i = 0; i < 4; ++i)
    one_launch = one_launch && src[i] && reinterpret_cast<uintptr_t>(src[i]) % 16 == 0 &&
                 reinterpret_cast<uintptr_t>(dst[i]) % 16 == 0 && len[i] % 16 == 0;
  if (ok && one_launch) {
    pa::UploadArgs ua;
    for (int i = 0; i < 4; ++i)
      ua.seg[i] = {static_cast<const uint4*>(src[i]), static_cast<uint4*>(dst[i]),
                   int64_t(len[i] / 16)};
    ok = pa::launch_upload(ua, p->sms, b->up) == cudaSuccess;
  } else if (ok) {
    ok = cudaMemcpyAsync(S.d_stage, S.h_stage, staged, cudaMemcpyHostToDevice, b->up) ==
             cudaSuccess &&
         cudaMemcpyAsync(S.d_q, h_q, b->q_bytes, cudaMemcpyHostToDevice, b->up) ==
             cudaSuccess &&
         cudaMemcpyAsync(S.d_k, h_key, b->kv_bytes, cudaMemcpyHostToDevice, b->up) ==
             cudaSuccess &&
         cudaMemcpyAsync(S.d_v, h_value, b->kv_bytes, cudaMemcpyHostToDevice, b->up) ==
             cudaSuccess;
  }
  ok = ok && cudaEventRecord(S.up, b->up) == cudaSuccess;
  // the previous step's download, now that this step's uploads are ahead of it
  ok = ok && flush_download(b);
  // kernels on the caller's stream, after the uploads and after the download
  // of this set's previous output
  ok = ok && cudaStreamWaitEvent(s, S.up, 0) == cudaSuccess;
  if (S.used) ok = ok && cudaStreamWaitEvent(s, S.down, 0) == cudaSuccess;
  if (ok && full_upload)          // many rows changed outside the batch: whole tables
    ok = cudaMemcpyAsync(b->d_tables, b->mirror.data(), b->mirror.size() * sizeof(int32_t),
                         cudaMemcpyHostToDevice, s) == cudaSuccess &&
         cudaStreamSynchronize(s) == cudaSuccess;
  if (ok) ok = pa::launch_table_patch(b->d_tables, MB, d_pat, npatch, s) == cudaSuccess;
  if (ok) ok = cow_blocks(p, d_csrc, d_cdst, ncow, s) == cudaSuccess;
  if (!ok) return PA_ERR_CUDA;
  st = b->window > 0
           ? pa_decode_window_append(p, S.d_q, S.d_k, S.d_v, d_slots, n, b->H, b->d_tables,
                                     MB, d_lens, scale, b->window, b->sinks, b->part, b->d_ws,
                                     b->ws_bytes, S.d_out, stream)
           : pa_decode_append(p, S.d_q, S.d_k, S.d_v, d_slots, n, b->H, b->d_tables, MB,
                              d_lens, scale, b->part, b->d_ws, b->ws_bytes, S.d_out, stream);
  if (st != PA_OK) return st;
  // the download goes on the download stream with the next call (or sync)
  if (cudaEventRecord(S.done, s) != cudaSuccess) return PA_ERR_CUDA;
  b->pending = int32_t(b->steps % kBatchSets);
  b->pending_out = h_out;
  S.used = true;
  ++b->steps;
  return PA_OK;
}

pa_status pa_batch_rollback(pa_batch* b) {
  if (!b) return PA_ERR_INVALID_ARG;
  pa_pool* p = b->pool;
  std::vector<int32_t> keep(b->seqs.size());
  for (size_t i = 0; i < b->seqs.size(); ++i) {
    if (!p->mgr->table(b->seqs[i])) return PA_ERR_UNKNOWN_SEQ;
    keep[i] = int32_t(std::max<int64_t>(0, p->mgr->length(b->seqs[i]) - 1));
  }
  pa_status st = from_mgr(p->mgr->truncate(b->seqs.data(), keep.data(), b->n));
  if (st != PA_OK) return st;
  // the mirror follows (entries past a row's end stay as they are, unused)
  for (size_t i = 0; i < b->seqs.size(); ++i) {
    b->mirror_len[i] = keep[i];
    b->mirror_blocks[i] = int32_t(p->mgr->table(b->seqs[i])->size());
  }
  return PA_OK;
}

pa_status pa_batch_set_window(pa_batch* b, int32_t window, int32_t sinks) {
  if (!b || window < 0 || sinks < 0 || (window == 0 && sinks > 0)) return PA_ERR_INVALID_ARG;
  pa_pool* p = b->pool;
  pa::DeviceScope on_pool_device(p->dev_id);
  const size_t need = window > 0 ? pa_decode_window_workspace_bytes(p, b->n, b->H, b->MB,
                                                                    window, sinks, b->part)
                                 : pa_decode_workspace_bytes(p, b->n, b->H, b->MB, b->part);
  if (need > b->ws_bytes) {
    // the scratch may still be read by queued steps
    if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
    void* ws = nullptr;
    if (cudaMalloc(&ws, need) != cudaSuccess) {
      cudaGetLastError();
      return PA_ERR_CUDA;
    }
    cudaFree(b->d_ws);
    b->d_ws = ws;
    b->ws_bytes = need;
  }
  b->window = window;
  b->sinks = sinks;
  return PA_OK;
}

pa_status pa_batch_sync(pa_batch* b) {
  if (!b) return PA_ERR_INVALID_ARG;
  pa::DeviceScope on_pool_device(b->pool->dev_id);
  if (!flush_download(b)) return PA_ERR_CUDA;
  for (auto& s : b->set)
    if (s.used && cudaEventSynchronize(s.down) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

pa_status pa_batch_free(pa_batch* b) {
  if (!b) return PA_OK;
  pa::DeviceScope on_pool_device(b->pool->dev_id);
  flush_download(b);
  cudaDeviceSynchronize();
  free_batch(b);
  return PA_OK;
}

pa_status pa_get_error(pa_pool* p, int32_t* device_code) {
  if (!p || !device_code) return PA_ERR_INVALID_ARG;
  *device_code = 0;
  if (!p->device) return PA_ERR_NO_DEVICE;
  pa::DeviceScope on_pool_device(p->dev_id);
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpy(device_code, p->d_err, sizeof(int32_t), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemset(p->d_err, 0, sizeof(int32_t)) != cudaSuccess) return PA_ERR_CUDA;
  return *device_code ? PA_ERR_DEVICE : PA_OK;
}

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNKNOWN_SEQ: return "unknown or released sequence";
    case PA_ERR_DUP_SEQ: return "duplicate sequence id";
    case PA_ERR_POOL_EXHAUSTED: return "physical KV pool exhausted";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_DEVICE: return "device error bits set";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PA_ERR_NO_DEVICE: return "host-only pool";
    case PA_ERR_INTERNAL: return "broken invariant";
    case PA_ERR_SCRATCH_LIMIT: return "request exceeds the fixed device scratch";
  }
  return "unknown status";
}

}  // extern "C"
