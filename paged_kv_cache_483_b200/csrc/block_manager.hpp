// Host block manager: free list, refcounts, block tables, copy-on-write plans.
//
// Semantics follow "abhik.ai examples/pagedattention.py" (KVPool: first free
// id in a fixed allocation order, copy-on-write of a shared partial tail,
// release) and "vladkulikov.com modern-llms module 9 notebook" (PagedKVPool:
// preflighted multi-token append, share_prefix, fill accounting, validate).
// Pure C++: no CUDA here, so every decision can be tested without a GPU.
#pragma once

#include <cstdint>
#include <cstddef>
#include <queue>
#include <unordered_map>
#include <vector>

namespace pa {

enum class MgrStatus { ok, unknown_seq, dup_seq, exhausted, invalid };

struct CowPair {
  int32_t src, dst;
};

struct Snapshot {
  int64_t allocated, free, capacity, payload, logical, waste, savings, live;
};

class BlockManager {
 public:
  // order: permutation of [0, num_blocks) or empty (identity).
  BlockManager(int32_t num_blocks, int32_t block_size,
               const std::vector<int32_t>& order);

  static bool is_permutation(const int32_t* order, int32_t n);

  MgrStatus create(int32_t seq);
  MgrStatus share_prefix(int32_t parent, int32_t child, int64_t prefix);
  MgrStatus release(int32_t seq);
  // Keep the first lengths[i] tokens of seqs[i] (distinct ids): blocks
  // wholly past them lose that sequence's reference, freed at zero -- the
  // release of "abhik.ai examples/pagedattention.py" applied to the dropped
  // tail.  All-or-nothing: every pair is checked before any change.
  MgrStatus truncate(const int32_t* seqs, const int32_t* lengths, int32_t n);

  // Batch append plan; all-or-nothing (preflight over the whole batch with
  // the refcount changes earlier members of the batch make).
  MgrStatus append(const int32_t* seqs, const int32_t* n_new, int32_t n,
                   std::vector<int64_t>* slots, std::vector<CowPair>* cow);

  const std::vector<int32_t>* table(int32_t seq) const;
  int64_t length(int32_t seq) const;
  Snapshot snapshot() const;
  const std::vector<int32_t>& refcounts() const { return refs_; }
  bool validate() const;

  int32_t num_blocks() const { return num_blocks_; }
  int32_t block_size() const { return block_size_; }

  // Prefix cache ("vladkulikov.com modern-llms module 9 notebook", the
  // prefix-hash trace): the block that ends at token `end` is identified by
  // (scope, revision, every token id before `end`), at full block boundaries.
  // create_cached: a new sequence starting with the longest run of leading
  // full blocks whose keys are cached (shared, refcount + 1 each).
  MgrStatus create_cached(int32_t seq, uint64_t scope, uint64_t revision,
                          const int32_t* tokens, int64_t n, int64_t* hit_tokens);
  // publish: key the sequence's full blocks among tokens[0, n) (n <= its
  // length); a key already cached keeps its block.  The cache holds one
  // reference per block it maps.
  MgrStatus publish(int32_t seq, uint64_t scope, uint64_t revision,
                    const int32_t* tokens, int64_t n, int64_t* added);
  // Drop every cache reference; returns the blocks that became free.
  int64_t prefix_clear();
  int64_t prefix_entries() const { return int64_t(pent_.size()); }

 private:
  struct Seq {
    int64_t length = 0;
    std::vector<int32_t> blocks;
    uint64_t batch = 0;   // the last append batch that named this sequence
  };
  int32_t take_block();            // first free id in the order
  void give_back(int32_t block);   // refcount reached zero
  std::vector<int64_t> fills() const;

  int32_t num_blocks_, block_size_;
  std::vector<int32_t> order_, rank_, refs_;
  std::vector<uint8_t> is_free_;
  int64_t n_free_;
  // min-heap of the free blocks' positions in the allocation order
  std::priority_queue<int32_t, std::vector<int32_t>, std::greater<int32_t>> free_heap_;
  std::unordered_map<int32_t, Seq> seqs_;
  // append scratch, reused by every call (no allocation per call once warm)
  uint64_t batch_ = 0;                  // stamp of the current append batch
  std::vector<Seq*> batch_seqs_;        // the batch's sequences, in order
  std::vector<int32_t> tail_drop_;      // per block: copies planned earlier in the batch
  std::vector<int32_t> tail_touched_;   // blocks whose tail_drop_ is non-zero

  // A key is stored as (its parent's entry, the block's own tokens): two
  // keys are equal exactly when their parents are and their last
  // block_size tokens are, so a chain of entries spells the whole prefix.
  struct PEntry {
    int32_t parent;        // entry of the previous block, -1 at the first
    uint64_t scope, revision;
    std::vector<int32_t> tokens;  // block_size ids
    int32_t block;
    uint64_t hash;
  };
  int32_t pfind(int32_t parent, uint64_t scope, uint64_t revision,
                const int32_t* tokens, uint64_t* hash_out) const;
  uint64_t phash(int32_t parent, uint64_t scope, uint64_t revision,
                 const int32_t* tokens) const;
  std::vector<PEntry> pent_;
  std::unordered_multimap<uint64_t, int32_t> pidx_;
  std::vector<int32_t> cache_refs_;  // per block: references the cache holds
};

}  // namespace pa
