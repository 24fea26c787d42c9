// Host block manager (see block_manager.hpp for the pages it follows).
#include "block_manager.hpp"

#include <algorithm>
#include <unordered_set>

namespace pa {

BlockManager::BlockManager(int32_t num_blocks, int32_t block_size,
                           const std::vector<int32_t>& order)
    : num_blocks_(num_blocks), block_size_(block_size),
      order_(order), rank_(num_blocks), refs_(num_blocks, 0),
      is_free_(num_blocks, 1), n_free_(num_blocks), tail_drop_(num_blocks, 0),
      cache_refs_(num_blocks, 0) {
  if (order_.empty()) {
    order_.resize(num_blocks);
    for (int32_t i = 0; i < num_blocks; ++i) order_[i] = i;
  }
  for (int32_t r = 0; r < num_blocks; ++r) {
    rank_[order_[r]] = r;
    free_heap_.push(r);
  }
}

bool BlockManager::is_permutation(const int32_t* order, int32_t n) {
  std::vector<uint8_t> seen(n, 0);
  for (int32_t i = 0; i < n; ++i) {
    int32_t b = order[i];
    if (b < 0 || b >= n || seen[b]) return false;
    seen[b] = 1;
  }
  return true;
}

// The first free id in the allocation order ("abhik.ai examples/pagedattention.py", KVPool._allocate).
int32_t BlockManager::take_block() {
  int32_t r = free_heap_.top();
  free_heap_.pop();
  int32_t b = order_[r];
  is_free_[b] = 0;
  --n_free_;
  refs_[b] = 1;
  return b;
}

void BlockManager::give_back(int32_t b) {
  is_free_[b] = 1;
  ++n_free_;
  free_heap_.push(rank_[b]);
}

MgrStatus BlockManager::create(int32_t seq) {
  if (seqs_.count(seq)) return MgrStatus::dup_seq;
  seqs_.emplace(seq, Seq{});
  return MgrStatus::ok;
}

// Share the blocks of the first `prefix` tokens ("vladkulikov.com modern-llms module 9 notebook",
// PagedKVPool.share_prefix; fork is the whole length, "abhik.ai examples/pagedattention.py").
MgrStatus BlockManager::share_prefix(int32_t parent, int32_t child,
                                     int64_t prefix) {
  auto it = seqs_.find(parent);
  if (it == seqs_.end()) return MgrStatus::unknown_seq;
  if (prefix < 0) prefix = it->second.length;  // fork: the whole parent
  if (prefix > it->second.length) return MgrStatus::invalid;
  if (seqs_.count(child)) return MgrStatus::dup_seq;
  Seq s;
  s.length = prefix;
  int64_t nb = (prefix + block_size_ - 1) / block_size_;
  s.blocks.assign(it->second.blocks.begin(), it->second.blocks.begin() + nb);
  for (int32_t b : s.blocks) ++refs_[b];
  seqs_.emplace(child, std::move(s));
  return MgrStatus::ok;
}

// One reference less per block; zero-reference blocks become free ("abhik.ai examples/pagedattention.py",
// KVPool.release).
MgrStatus BlockManager::release(int32_t seq) {
  auto it = seqs_.find(seq);
  if (it == seqs_.end()) return MgrStatus::unknown_seq;
  for (int32_t b : it->second.blocks)
    if (--refs_[b] == 0) give_back(b);
  seqs_.erase(it);
  return MgrStatus::ok;
}

// A rollback of each sequence's newest tokens; equal to share_prefix of the
// kept tokens into a new sequence followed by release of the old one.
MgrStatus BlockManager::truncate(const int32_t* seqs, const int32_t* lengths, int32_t n) {
  if (n < 0 || (n > 0 && (!seqs || !lengths))) return MgrStatus::invalid;
  const uint64_t stamp = ++batch_;
  for (int32_t i = 0; i < n; ++i) {
    auto it = seqs_.find(seqs[i]);
    if (it == seqs_.end()) return MgrStatus::unknown_seq;
    if (lengths[i] < 0 || lengths[i] > it->second.length) return MgrStatus::invalid;
    if (it->second.batch == stamp) return MgrStatus::invalid;   // named twice
    it->second.batch = stamp;
  }
  for (int32_t i = 0; i < n; ++i) {
    Seq& s = seqs_.find(seqs[i])->second;
    const size_t keep = size_t((int64_t(lengths[i]) + block_size_ - 1) / block_size_);
    for (size_t j = keep; j < s.blocks.size(); ++j)
      if (--refs_[s.blocks[j]] == 0) give_back(s.blocks[j]);
    if (keep < s.blocks.size()) s.blocks.resize(keep);
    s.length = lengths[i];
  }
  return MgrStatus::ok;
}

// Preflight ("vladkulikov.com modern-llms module 9 notebook", PagedKVPool._blocks_needed_for_append), then
// the copy of a shared partial tail and token placement ("abhik.ai examples/pagedattention.py",
// KVPool.append and copy_on_write).
MgrStatus BlockManager::append(const int32_t* seqs, const int32_t* n_new,
                               int32_t n, std::vector<int64_t>* slots,
                               std::vector<CowPair>* cow) {
  // -- preflight: nothing below this block changes state until it passes.
  // A sequence named twice in the batch is caught by its batch stamp; a
  // shared tail copied earlier in the batch holds one reference less for the
  // sequences after it (tail_drop_, reset before returning).
  ++batch_;
  batch_seqs_.clear();
  tail_touched_.clear();
  MgrStatus verdict = MgrStatus::ok;
  int64_t need = 0, total_tokens = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = seqs_.find(seqs[i]);
    if (it == seqs_.end()) {
      verdict = MgrStatus::unknown_seq;
      break;
    }
    Seq& s = it->second;
    if (n_new[i] < 0 || s.batch == batch_) {
      verdict = MgrStatus::invalid;
      break;
    }
    s.batch = batch_;
    batch_seqs_.push_back(&s);
    int64_t cnt = n_new[i];
    total_tokens += cnt;
    if (cnt == 0) continue;
    int64_t used = s.length % block_size_, room = 0;
    if (!s.blocks.empty() && used) {
      room = block_size_ - used;
      const int32_t tail = s.blocks.back();
      if (refs_[tail] - tail_drop_[tail] > 1) {
        need += 1;
        if (tail_drop_[tail]++ == 0) tail_touched_.push_back(tail);
      }
    }
    int64_t beyond = std::max<int64_t>(0, cnt - room);
    need += (beyond + block_size_ - 1) / block_size_;
  }
  for (int32_t b : tail_touched_) tail_drop_[b] = 0;
  if (verdict != MgrStatus::ok) return verdict;
  if (need > n_free_) return MgrStatus::exhausted;

  // -- apply: per sequence, copy a shared partial tail, then place tokens.
  if (slots) slots->reserve(slots->size() + total_tokens);
  for (int32_t i = 0; i < n; ++i) {
    Seq& s = *batch_seqs_[size_t(i)];
    int64_t cnt = n_new[i];
    if (cnt == 0) continue;
    if (!s.blocks.empty() && (s.length % block_size_) &&
        refs_[s.blocks.back()] > 1) {
      int32_t old = s.blocks.back();
      int32_t fresh = take_block();
      s.blocks.back() = fresh;
      --refs_[old];
      if (cow) cow->push_back({old, fresh});
    }
    for (int64_t t = 0; t < cnt; ++t) {
      int64_t pos = s.length;
      int64_t logical = pos / block_size_, off = pos % block_size_;
      if (off == 0) s.blocks.push_back(take_block());
      if (slots)
        slots->push_back(int64_t(s.blocks[logical]) * block_size_ + off);
      s.length = pos + 1;
    }
  }
  return MgrStatus::ok;
}

const std::vector<int32_t>* BlockManager::table(int32_t seq) const {
  auto it = seqs_.find(seq);
  return it == seqs_.end() ? nullptr : &it->second.blocks;
}

int64_t BlockManager::length(int32_t seq) const {
  auto it = seqs_.find(seq);
  return it == seqs_.end() ? -1 : it->second.length;
}

// Live slots per block: the largest fill any sharer gives it ("vladkulikov.com modern-llms module 9 notebook",
// PagedKVPool._refresh_fills); a block the prefix cache maps counts as full.
std::vector<int64_t> BlockManager::fills() const {
  std::vector<int64_t> fill(num_blocks_, 0);
  for (int32_t b = 0; b < num_blocks_; ++b)
    if (cache_refs_[b]) fill[b] = block_size_;   // cached blocks are full
  for (const auto& kv : seqs_) {
    const Seq& s = kv.second;
    for (size_t j = 0; j < s.blocks.size(); ++j) {
      int64_t f = std::min<int64_t>(block_size_, s.length - int64_t(j) * block_size_);
      fill[s.blocks[j]] = std::max(fill[s.blocks[j]], f);
    }
  }
  return fill;
}

// The state summary of "vladkulikov.com modern-llms module 9 notebook", PagedKVPool.snapshot.
Snapshot BlockManager::snapshot() const {
  Snapshot r{};
  std::vector<int64_t> fill = fills();
  r.free = n_free_;
  r.allocated = num_blocks_ - n_free_;
  r.capacity = r.allocated * block_size_;
  for (int32_t b = 0; b < num_blocks_; ++b)
    if (refs_[b]) r.payload += fill[b];
  for (const auto& kv : seqs_) r.logical += kv.second.length;
  r.waste = r.capacity - r.payload;
  r.savings = r.logical - r.payload;
  r.live = int64_t(seqs_.size());
  return r;
}

// The invariants of "vladkulikov.com modern-llms module 9 notebook", PagedKVPool.validate.
bool BlockManager::validate() const {
  if (int64_t(free_heap_.size()) != n_free_) return false;
  std::vector<int32_t> expect(num_blocks_, 0);
  for (const auto& kv : seqs_) {
    const Seq& s = kv.second;
    if (s.length < 0) return false;
    if (int64_t(s.blocks.size()) != (s.length + block_size_ - 1) / block_size_)
      return false;
    std::unordered_set<int32_t> uniq(s.blocks.begin(), s.blocks.end());
    if (uniq.size() != s.blocks.size()) return false;
    for (int32_t b : s.blocks) {
      if (b < 0 || b >= num_blocks_) return false;
      ++expect[b];
    }
  }
  std::vector<uint8_t> in_seq(num_blocks_, 0);
  for (const auto& kv : seqs_)
    for (int32_t b : kv.second.blocks) in_seq[b] = 1;
  int64_t cache_only = 0;
  for (int32_t b = 0; b < num_blocks_; ++b) {
    expect[b] += cache_refs_[b];
    if (cache_refs_[b] && !in_seq[b]) cache_only += block_size_;
  }
  std::vector<int64_t> fill = fills();
  int64_t nfree = 0;
  for (int32_t b = 0; b < num_blocks_; ++b) {
    if (refs_[b] != expect[b]) return false;
    if (refs_[b] == 0) {
      if (!is_free_[b] || fill[b] != 0) return false;
      ++nfree;
    } else {
      if (is_free_[b]) return false;
      if (fill[b] < 1 || fill[b] > block_size_) return false;
    }
  }
  if (nfree != n_free_) return false;
  Snapshot s = snapshot();
  return s.logical + cache_only >= s.payload;
}

uint64_t BlockManager::phash(int32_t parent, uint64_t scope, uint64_t revision,
                             const int32_t* tokens) const {
  // FNV-1a over the entry's identity (parent entry, scope, revision, ids)
  uint64_t h = 1469598103934665603ull;
  auto mix = [&h](uint64_t v) {
    for (int i = 0; i < 8; ++i) {
      h ^= (v >> (8 * i)) & 0xFF;
      h *= 1099511628211ull;
    }
  };
  mix(uint64_t(int64_t(parent)));
  mix(scope);
  mix(revision);
  for (int32_t i = 0; i < block_size_; ++i) mix(uint64_t(uint32_t(tokens[i])));
  return h;
}

int32_t BlockManager::pfind(int32_t parent, uint64_t scope, uint64_t revision,
                            const int32_t* tokens, uint64_t* hash_out) const {
  const uint64_t h = phash(parent, scope, revision, tokens);
  if (hash_out) *hash_out = h;
  auto range = pidx_.equal_range(h);
  for (auto it = range.first; it != range.second; ++it) {
    const PEntry& e = pent_[it->second];
    if (e.parent == parent && e.scope == scope && e.revision == revision &&
        std::equal(e.tokens.begin(), e.tokens.end(), tokens))
      return it->second;
  }
  return -1;
}

// Prefix reuse ("vladkulikov.com modern-llms module 9 notebook", prefix-hash trace): the new sequence starts
// with the longest run of cached leading full blocks.
MgrStatus BlockManager::create_cached(int32_t seq, uint64_t scope, uint64_t revision,
                                      const int32_t* tokens, int64_t n,
                                      int64_t* hit_tokens) {
  if (n < 0 || (n > 0 && !tokens)) return MgrStatus::invalid;
  if (seqs_.count(seq)) return MgrStatus::dup_seq;
  Seq s;
  int32_t parent = -1;
  for (int64_t end = block_size_; end <= n; end += block_size_) {
    const int32_t e = pfind(parent, scope, revision, tokens + end - block_size_, nullptr);
    if (e < 0) break;
    s.blocks.push_back(pent_[e].block);
    parent = e;
  }
  s.length = int64_t(s.blocks.size()) * block_size_;
  for (int32_t b : s.blocks) ++refs_[b];
  if (hit_tokens) *hit_tokens = s.length;
  seqs_.emplace(seq, std::move(s));
  return MgrStatus::ok;
}

// Key every full block of a sequence; the first publisher of a key wins.
MgrStatus BlockManager::publish(int32_t seq, uint64_t scope, uint64_t revision,
                                const int32_t* tokens, int64_t n, int64_t* added) {
  auto it = seqs_.find(seq);
  if (it == seqs_.end()) return MgrStatus::unknown_seq;
  if (n < 0 || (n > 0 && !tokens) || n > it->second.length) return MgrStatus::invalid;
  const Seq& s = it->second;
  int64_t count = 0;
  int32_t parent = -1;
  for (int64_t end = block_size_; end <= n; end += block_size_) {
    const int32_t* blk_tokens = tokens + end - block_size_;
    uint64_t h = 0;
    int32_t e = pfind(parent, scope, revision, blk_tokens, &h);
    if (e < 0) {
      PEntry pe{parent, scope, revision,
                std::vector<int32_t>(blk_tokens, blk_tokens + block_size_),
                s.blocks[size_t(end / block_size_ - 1)], h};
      e = int32_t(pent_.size());
      pent_.push_back(std::move(pe));
      pidx_.emplace(h, e);
      ++refs_[pent_[e].block];
      ++cache_refs_[pent_[e].block];
      ++count;
    }
    parent = e;
  }
  if (added) *added = count;
  return MgrStatus::ok;
}

int64_t BlockManager::prefix_clear() {
  int64_t freed = 0;
  for (const PEntry& e : pent_) {
    --cache_refs_[e.block];
    if (--refs_[e.block] == 0) {
      give_back(e.block);
      ++freed;
    }
  }
  pent_.clear();
  pidx_.clear();
  return freed;
}

}  // namespace pa
