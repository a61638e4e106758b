// Host block manager: free list, reference counts, block tables, copy-on-write.
//
// P1 = "Paged Attention：大模型推理显存优化的核心方案", P2 = "PagedAttention：操作系统级 KV
// 缓存虚拟内存管理".
//   P1 "Paged Attention 的工作原理" / P2 §3.2.2 steps 2-3: a block is taken only
//     when the sequence's last block is full; the new token goes to (block, offset).
//   P1 "块表（Block Table）" / P2 §2.3: per-sequence logical -> physical table.
//   P2 §3.2.1: a prompt of n tokens takes ceil(n / block_size) blocks.
//   P2 §3.3: a finished sequence's blocks return to the free pool.
//   P2 §3.4: shared blocks are reference counted; writing into one copies it
//     first, remaps the writer's table and drops one reference from the original.
//   P2 §3.4 (prefix block pool) / P3: prompts' whole blocks can be listed in a
//     prefix cache keyed by their full token prefix; a later prompt with the
//     same prefix maps its first blocks onto them. The cache holds one
//     reference per listed block; a listed block held only by the cache is
//     evictable and is reclaimed, least recently released first, when the free
//     list runs dry.
//   P2 §五 (page replacement) / §八: a sequence's blocks can be swapped out to
//     host blocks (own FIFO free list) and back in, to relieve the device pool.
// The free list is a FIFO ring over a fixed array (front = next allocation,
// back = most recently freed); evictable blocks sit on an intrusive LRU list;
// every operation is O(blocks touched).
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "../../include/pagedattn.h"

namespace {

struct Seq {
  std::vector<int32_t> table;
  int64_t len = 0;
  // dry run of a batched append (valid while batch == the manager's batch number)
  uint64_t batch = 0;
  int64_t shadow_len = 0, shadow_bi = -1;
};

// Prefix-cache key of a prompt block: a 64-bit hash chained over every token
// of the prompt up to the block's end. The entry keeps the parent's chain hash
// and the block's own tokens, which a hit must match exactly.
uint64_t mix64(uint64_t x) {
  x ^= x >> 30;
  x *= 0xbf58476d1ce4e5b9ull;
  x ^= x >> 27;
  x *= 0x94d049bb133111ebull;
  x ^= x >> 31;
  return x;
}
constexpr uint64_t kChainSeed = 0x6a09e667f3bcc909ull;
uint64_t chain_hash(uint64_t parent, const int32_t* tok, int32_t n) {
  uint64_t h = mix64(parent ^ 0x9e3779b97f4a7c15ull);
  for (int32_t i = 0; i < n; ++i) h = mix64(h ^ (static_cast<uint64_t>(static_cast<uint32_t>(tok[i])) + 0x632be59bd9b4e019ull));
  return h;
}

struct CacheEntry {
  int32_t block;
  uint64_t parent;
  std::vector<int32_t> tokens;
};

struct Swapped {
  std::vector<int32_t> host;  // host block of each logical block
  int64_t len = 0;
};

class BlockManager {
 public:
  BlockManager(int64_t num_blocks, int32_t block_size)
      : nb_(num_blocks),
        bs_(block_size),
        ring_(num_blocks),
        ref_(num_blocks, 0),
        key_of_(num_blocks, 0),
        cached_(num_blocks, 0),
        lru_prev_(num_blocks, -1),
        lru_next_(num_blocks, -1),
        in_lru_(num_blocks, 0) {}

  bool init_order(const int32_t* order) {
    std::vector<uint8_t> seen(nb_, 0);
    for (int64_t i = 0; i < nb_; ++i) {
      int32_t b = order ? order[i] : static_cast<int32_t>(i);
      if (b < 0 || b >= nb_ || seen[b]) return false;
      seen[b] = 1;
      ring_[i] = b;
    }
    head_ = 0;
    count_ = nb_;
    return true;
  }

  int64_t free_count() const { return count_; }

  pa_status add_seq(int64_t id, int32_t n, int64_t* slots) {
    if (n < 0) return PA_ERR_INVALID_ARG;
    if (seqs_.count(id) || swapped_.count(id)) return PA_ERR_SEQ_EXISTS;
    int64_t need = (static_cast<int64_t>(n) + bs_ - 1) / bs_;
    if (need > available()) return PA_ERR_NO_FREE_BLOCKS;
    Seq s;
    s.table.reserve(need);
    for (int64_t i = 0; i < need; ++i) {
      int32_t b = pop();
      ref_[b] = 1;
      s.table.push_back(b);
    }
    s.len = n;
    if (slots)
      for (int32_t t = 0; t < n; ++t) slots[t] = slot_of(s.table, t);
    seqs_.emplace(id, std::move(s));
    return PA_OK;
  }

  pa_status fork(int64_t parent, int64_t child) {
    auto it = seqs_.find(parent);
    if (it == seqs_.end()) return PA_ERR_UNKNOWN_SEQ;
    if (seqs_.count(child) || swapped_.count(child)) return PA_ERR_SEQ_EXISTS;
    Seq c = it->second;  // copy of table and length
    for (int32_t b : c.table) ++ref_[b];
    seqs_.emplace(child, std::move(c));
    return PA_OK;
  }

  // Blocks the next append of `s` takes: 1 if its last block is full or
  // shared, else 0.
  int blocks_needed(const Seq& s) const {
    if (s.len % bs_ == 0) return 1;
    return ref_[s.table[s.len / bs_]] > 1 ? 1 : 0;
  }

  pa_status append(int64_t id, int64_t* slot, int32_t* pair) {
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return PA_ERR_UNKNOWN_SEQ;
    Seq& s = it->second;
    if (blocks_needed(s) > available()) return PA_ERR_NO_FREE_BLOCKS;
    do_append(s, slot, pair);
    return PA_OK;
  }

  pa_status append_many(int32_t n, const int64_t* ids, int64_t* slots, int32_t* pairs, int32_t* n_pairs) {
    // Dry run on shadow lengths and counts so that the batch is all or nothing.
    // After an append at length L the block at logical index L / bs is private
    // to the sequence (fresh, copied, or already held once), and counts only
    // fall during a batch, so a later append into the same index copies nothing.
    // The shadow state lives in the sequences (tagged with this batch's
    // number) and the count changes in a per-block array reset afterwards:
    // no allocation per call once the scratch vectors have grown.
    ++batch_no_;
    batch_.resize(static_cast<size_t>(n));
    if (static_cast<int64_t>(dref_.size()) != nb_) dref_.assign(static_cast<size_t>(nb_), 0);
    dref_touched_.clear();
    int64_t need = 0;
    pa_status err = PA_OK;
    for (int32_t i = 0; i < n; ++i) {
      auto it = seqs_.find(ids[i]);
      if (it == seqs_.end()) {
        err = PA_ERR_UNKNOWN_SEQ;
        break;
      }
      Seq& s = it->second;
      batch_[i] = &s;
      if (s.batch != batch_no_) {
        s.batch = batch_no_;
        s.shadow_len = s.len;
        s.shadow_bi = -1;
      }
      const int64_t bi = s.shadow_len / bs_;
      if (s.shadow_len % bs_ == 0) {
        ++need;
      } else if (bi != s.shadow_bi) {
        const int32_t b = s.table[bi];
        if (ref_[b] + dref_[b] > 1) {
          ++need;
          if (dref_[b] == 0) dref_touched_.push_back(b);
          dref_[b] -= 1;
        }
      }
      s.shadow_bi = bi;
      s.shadow_len += 1;
    }
    for (int32_t b : dref_touched_) dref_[b] = 0;
    if (err != PA_OK) return err;
    if (need > available()) return PA_ERR_NO_FREE_BLOCKS;
    int32_t np = 0;
    for (int32_t i = 0; i < n; ++i) {
      int32_t pr[2];
      do_append(*batch_[i], &slots[i], pr);
      if (pr[0] >= 0) {
        if (pairs) {
          pairs[2 * np] = pr[0];
          pairs[2 * np + 1] = pr[1];
        }
        ++np;
      }
    }
    if (n_pairs) *n_pairs = np;
    return PA_OK;
  }

  pa_status free_seq(int64_t id) {
    auto sw = swapped_.find(id);
    if (sw != swapped_.end()) {
      for (int32_t h : sw->second.host) hpush(h);
      swapped_.erase(sw);
      return PA_OK;
    }
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return PA_ERR_UNKNOWN_SEQ;
    for (int32_t b : it->second.table) {
      if (--ref_[b] == 0)
        push(b);
      else if (ref_[b] == 1 && cached_[b])
        lru_push_back(b);  // only the cache holds it now
    }
    seqs_.erase(it);
    return PA_OK;
  }

  // Prefill with prefix reuse (see pa_bm_add_seq_cached).
  pa_status add_seq_cached(int64_t id, const int32_t* tok, int32_t n, int64_t* slots, int32_t* n_cached) {
    if (n < 0 || (n > 0 && !tok)) return PA_ERR_INVALID_ARG;
    if (seqs_.count(id) || swapped_.count(id)) return PA_ERR_SEQ_EXISTS;
    const int32_t nfull = n / bs_;
    const int64_t nblocks = (static_cast<int64_t>(n) + bs_ - 1) / bs_;
    std::vector<int32_t> hits;
    std::vector<uint64_t> keys(nfull);
    uint64_t parent = kChainSeed;
    bool missed = false;
    int64_t evictable_hits = 0;
    for (int32_t i = 0; i < nfull; ++i) {
      const int32_t* bt = tok + static_cast<int64_t>(i) * bs_;
      keys[i] = chain_hash(parent, bt, bs_);
      if (!missed) {
        auto it = cache_.find(keys[i]);
        if (it != cache_.end() && it->second.parent == parent &&
            std::memcmp(it->second.tokens.data(), bt, sizeof(int32_t) * bs_) == 0) {
          hits.push_back(it->second.block);
          if (in_lru_[it->second.block]) ++evictable_hits;
        } else {
          missed = true;
        }
      }
      parent = keys[i];
    }
    const int64_t need = nblocks - static_cast<int64_t>(hits.size());
    if (need > available() - evictable_hits) return PA_ERR_NO_FREE_BLOCKS;
    Seq s;
    s.table.reserve(nblocks);
    for (int32_t b : hits) {
      if (in_lru_[b]) lru_remove(b);
      ++ref_[b];
      s.table.push_back(b);
    }
    for (int64_t i = static_cast<int64_t>(hits.size()); i < nblocks; ++i) {
      int32_t b = pop();
      ref_[b] = 1;
      s.table.push_back(b);
      if (i < nfull && !cache_.count(keys[i])) {
        CacheEntry e;
        e.block = b;
        e.parent = i == 0 ? kChainSeed : keys[i - 1];
        e.tokens.assign(tok + i * bs_, tok + (i + 1) * bs_);
        cache_.emplace(keys[i], std::move(e));
        key_of_[b] = keys[i];
        cached_[b] = 1;
        ++ref_[b];  // the cache's own reference
      }
    }
    s.len = n;
    const int32_t nc = static_cast<int32_t>(hits.size()) * bs_;
    hit_tokens_ += nc;
    if (slots)
      for (int32_t t = 0; t < n; ++t) slots[t] = t < nc ? -1 : slot_of(s.table, t);
    if (n_cached) *n_cached = nc;
    seqs_.emplace(id, std::move(s));
    return PA_OK;
  }

  pa_status set_host_blocks(int64_t n) {
    if (n < 0 || n > INT32_MAX || !swapped_.empty()) return PA_ERR_INVALID_ARG;
    hring_.assign(n, 0);
    for (int64_t i = 0; i < n; ++i) hring_[i] = static_cast<int32_t>(i);
    hhead_ = 0;
    hcount_ = n;
    return PA_OK;
  }

  pa_status swap_out(int64_t id, int32_t* pairs, int32_t cap, int32_t* n_out) {
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return PA_ERR_UNKNOWN_SEQ;
    const int64_t nb = static_cast<int64_t>(it->second.table.size());
    if (nb > cap || (nb > 0 && !pairs)) return PA_ERR_INVALID_ARG;
    if (nb > hcount_) return PA_ERR_NO_FREE_BLOCKS;
    Swapped sw;
    sw.len = it->second.len;
    sw.host.reserve(nb);
    for (int64_t i = 0; i < nb; ++i) {
      const int32_t h = hpop();
      sw.host.push_back(h);
      pairs[2 * i] = it->second.table[i];
      pairs[2 * i + 1] = h;
    }
    free_seq(id);  // one reference per device block
    swapped_.emplace(id, std::move(sw));
    if (n_out) *n_out = static_cast<int32_t>(nb);
    return PA_OK;
  }

  pa_status swap_in(int64_t id, int32_t* pairs, int32_t cap, int32_t* n_out) {
    auto sw = swapped_.find(id);
    if (sw == swapped_.end()) return PA_ERR_UNKNOWN_SEQ;
    const int64_t nb = static_cast<int64_t>(sw->second.host.size());
    if (nb > cap || (nb > 0 && !pairs)) return PA_ERR_INVALID_ARG;
    if (nb > available()) return PA_ERR_NO_FREE_BLOCKS;
    Seq s;
    s.len = sw->second.len;
    s.table.reserve(nb);
    for (int64_t i = 0; i < nb; ++i) {
      const int32_t b = pop();
      ref_[b] = 1;
      s.table.push_back(b);
      pairs[2 * i] = sw->second.host[i];
      pairs[2 * i + 1] = b;
    }
    for (int32_t h : sw->second.host) hpush(h);
    swapped_.erase(sw);
    seqs_.emplace(id, std::move(s));
    if (n_out) *n_out = static_cast<int32_t>(nb);
    return PA_OK;
  }

  int64_t host_free() const { return hcount_; }

  void prefix_stats(int64_t* cached, int64_t* evictable, int64_t* hit_tokens) const {
    if (cached) *cached = static_cast<int64_t>(cache_.size());
    if (evictable) *evictable = lru_size_;
    if (hit_tokens) *hit_tokens = hit_tokens_;
  }

  const Seq* find(int64_t id) const {
    auto it = seqs_.find(id);
    return it == seqs_.end() ? nullptr : &it->second;
  }

  int32_t ref(int32_t b) const { return ref_[b]; }
  int64_t num_blocks() const { return nb_; }
  int32_t block_size() const { return bs_; }

  void stats(int64_t* free_blocks, int64_t* used, int64_t* allocated) const {
    // fill of each block = max over the tables that hold it
    std::unordered_map<int32_t, int32_t> fill;
    for (const auto& kv : seqs_) {
      const Seq& s = kv.second;
      for (size_t i = 0; i < s.table.size(); ++i) {
        int64_t n = s.len - static_cast<int64_t>(i) * bs_;
        int32_t f = static_cast<int32_t>(n < bs_ ? n : bs_);
        int32_t& cur = fill[s.table[i]];
        if (f > cur) cur = f;
      }
    }
    int64_t u = 0;
    for (const auto& kv : fill) u += kv.second;
    if (free_blocks) *free_blocks = count_;
    if (used) *used = u;
    if (allocated) *allocated = (nb_ - count_) * bs_;
  }

  void free_list(int32_t* out, int64_t cap, int64_t* n) const {
    for (int64_t i = 0; i < count_ && i < cap; ++i) out[i] = ring_[(head_ + i) % nb_];
    if (n) *n = count_;
  }

 private:
  int64_t slot_of(const std::vector<int32_t>& table, int64_t t) const {
    return static_cast<int64_t>(table[t / bs_]) * bs_ + t % bs_;
  }
  // Blocks an allocation can draw on: the free list plus evictable cached blocks.
  int64_t available() const { return count_ + lru_size_; }

  void lru_push_back(int32_t b) {
    lru_prev_[b] = lru_tail_;
    lru_next_[b] = -1;
    if (lru_tail_ >= 0)
      lru_next_[lru_tail_] = b;
    else
      lru_head_ = b;
    lru_tail_ = b;
    in_lru_[b] = 1;
    ++lru_size_;
  }
  void lru_remove(int32_t b) {
    if (lru_prev_[b] >= 0)
      lru_next_[lru_prev_[b]] = lru_next_[b];
    else
      lru_head_ = lru_next_[b];
    if (lru_next_[b] >= 0)
      lru_prev_[lru_next_[b]] = lru_prev_[b];
    else
      lru_tail_ = lru_prev_[b];
    in_lru_[b] = 0;
    --lru_size_;
  }
  // Free list empty: drop the least recently released evictable block from
  // the cache and put it on the free list.
  void evict_one() {
    const int32_t b = lru_head_;
    lru_remove(b);
    cache_.erase(key_of_[b]);
    cached_[b] = 0;
    ref_[b] = 0;
    push(b);
  }
  int32_t hpop() {
    const int32_t h = hring_[hhead_];
    hhead_ = (hhead_ + 1) % static_cast<int64_t>(hring_.size());
    --hcount_;
    return h;
  }
  void hpush(int32_t h) {
    hring_[(hhead_ + hcount_) % static_cast<int64_t>(hring_.size())] = h;
    ++hcount_;
  }
  int32_t pop() {
    if (count_ == 0) evict_one();
    int32_t b = ring_[head_];
    head_ = (head_ + 1) % nb_;
    --count_;
    return b;
  }
  void push(int32_t b) {
    ring_[(head_ + count_) % nb_] = b;
    ++count_;
  }
  void do_append(Seq& s, int64_t* slot, int32_t* pair) {
    int64_t t = s.len;
    int64_t i = t / bs_;
    if (pair) pair[0] = pair[1] = -1;
    if (t % bs_ == 0) {
      int32_t b = pop();
      ref_[b] = 1;
      s.table.push_back(b);
    } else {
      int32_t src = s.table[i];
      if (ref_[src] > 1) {
        int32_t dst = pop();
        --ref_[src];
        ref_[dst] = 1;
        s.table[i] = dst;
        if (pair) {
          pair[0] = src;
          pair[1] = dst;
        }
      }
    }
    s.len = t + 1;
    if (slot) *slot = slot_of(s.table, t);
  }

  int64_t nb_;
  int32_t bs_;
  std::vector<int32_t> ring_;
  int64_t head_ = 0, count_ = 0;
  std::vector<int32_t> ref_;
  std::unordered_map<int64_t, Seq> seqs_;
  // batched-append scratch (see append_many)
  uint64_t batch_no_ = 0;
  std::vector<Seq*> batch_;
  std::vector<int32_t> dref_, dref_touched_;
  // prefix cache
  std::unordered_map<uint64_t, CacheEntry> cache_;
  std::vector<uint64_t> key_of_;
  std::vector<uint8_t> cached_;
  std::vector<int32_t> lru_prev_, lru_next_;
  std::vector<uint8_t> in_lru_;
  int32_t lru_head_ = -1, lru_tail_ = -1;
  int64_t lru_size_ = 0;
  int64_t hit_tokens_ = 0;
  // host blocks for swapped-out sequences
  std::vector<int32_t> hring_;
  int64_t hhead_ = 0, hcount_ = 0;
  std::unordered_map<int64_t, Swapped> swapped_;
};

}  // namespace

struct pa_bm {
  BlockManager m;
  pa_bm(int64_t nb, int32_t bs) : m(nb, bs) {}
};

extern "C" {

pa_status pa_bm_create(int64_t num_blocks, int32_t block_size, const int32_t* free_order, pa_bm** out) {
  if (!out || num_blocks <= 0 || num_blocks > INT32_MAX || block_size <= 0) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  pa_bm* bm = new (std::nothrow) pa_bm(num_blocks, block_size);
  if (!bm) return PA_ERR_INVALID_ARG;
  if (!bm->m.init_order(free_order)) {
    delete bm;
    return PA_ERR_INVALID_ARG;
  }
  *out = bm;
  return PA_OK;
}

void pa_bm_destroy(pa_bm* bm) { delete bm; }

pa_status pa_bm_add_seq(pa_bm* bm, int64_t seq_id, int32_t num_tokens, int64_t* slots_out) {
  if (!bm) return PA_ERR_INVALID_ARG;
  return bm->m.add_seq(seq_id, num_tokens, slots_out);
}

pa_status pa_bm_add_seq_cached(pa_bm* bm, int64_t seq_id, const int32_t* tokens, int32_t num_tokens,
                               int64_t* slots_out, int32_t* n_cached_out) {
  if (!bm) return PA_ERR_INVALID_ARG;
  return bm->m.add_seq_cached(seq_id, tokens, num_tokens, slots_out, n_cached_out);
}

pa_status pa_bm_prefix_stats(const pa_bm* bm, int64_t* cached_blocks, int64_t* evictable_blocks,
                             int64_t* hit_tokens) {
  if (!bm) return PA_ERR_INVALID_ARG;
  bm->m.prefix_stats(cached_blocks, evictable_blocks, hit_tokens);
  return PA_OK;
}

pa_status pa_bm_set_host_blocks(pa_bm* bm, int64_t num_host_blocks) {
  if (!bm) return PA_ERR_INVALID_ARG;
  return bm->m.set_host_blocks(num_host_blocks);
}

pa_status pa_bm_swap_out(pa_bm* bm, int64_t seq_id, int32_t* pairs_out, int32_t cap, int32_t* n_pairs_out) {
  if (!bm || cap < 0) return PA_ERR_INVALID_ARG;
  return bm->m.swap_out(seq_id, pairs_out, cap, n_pairs_out);
}

pa_status pa_bm_swap_in(pa_bm* bm, int64_t seq_id, int32_t* pairs_out, int32_t cap, int32_t* n_pairs_out) {
  if (!bm || cap < 0) return PA_ERR_INVALID_ARG;
  return bm->m.swap_in(seq_id, pairs_out, cap, n_pairs_out);
}

pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child) {
  if (!bm) return PA_ERR_INVALID_ARG;
  return bm->m.fork(parent, child);
}

pa_status pa_bm_append_slot(pa_bm* bm, int64_t seq_id, int64_t* slot_out, int32_t* cow_pair_out) {
  if (!bm || !slot_out) return PA_ERR_INVALID_ARG;
  return bm->m.append(seq_id, slot_out, cow_pair_out);
}

pa_status pa_bm_append_slots(pa_bm* bm, int32_t n, const int64_t* seq_ids, int64_t* slots_out,
                             int32_t* cow_pairs_out, int32_t* n_pairs_out) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !slots_out))) return PA_ERR_INVALID_ARG;
  return bm->m.append_many(n, seq_ids, slots_out, cow_pairs_out, n_pairs_out);
}

pa_status pa_bm_free_seq(pa_bm* bm, int64_t seq_id) {
  if (!bm) return PA_ERR_INVALID_ARG;
  return bm->m.free_seq(seq_id);
}

pa_status pa_bm_block_table(const pa_bm* bm, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n_out,
                            int64_t* len_out) {
  if (!bm || cap < 0 || (cap > 0 && !out)) return PA_ERR_INVALID_ARG;
  const Seq* s = bm->m.find(seq_id);
  if (!s) return PA_ERR_UNKNOWN_SEQ;
  int32_t n = static_cast<int32_t>(s->table.size());
  for (int32_t i = 0; i < n && i < cap; ++i) out[i] = s->table[i];
  if (n_out) *n_out = n;
  if (len_out) *len_out = s->len;
  return PA_OK;
}

pa_status pa_bm_block_tables(const pa_bm* bm, int32_t n, const int64_t* seq_ids, int32_t* out, int32_t cap,
                             int32_t pad, int32_t* lens_out) {
  if (!bm || n < 0 || cap < 0 || (n > 0 && (!seq_ids || !out || !lens_out))) return PA_ERR_INVALID_ARG;
  // every id is checked before any row is written; the lookups of a batch of
  // up to kKeep sequences are kept for the copy pass
  constexpr int32_t kKeep = 512;
  const Seq* kept[kKeep];
  for (int32_t i = 0; i < n; ++i) {
    const Seq* s = bm->m.find(seq_ids[i]);
    if (!s) return PA_ERR_UNKNOWN_SEQ;
    if (static_cast<int64_t>(s->table.size()) > cap || s->len > INT32_MAX) return PA_ERR_INVALID_ARG;
    if (i < kKeep) kept[i] = s;
  }
  for (int32_t i = 0; i < n; ++i) {
    const Seq* s = i < kKeep ? kept[i] : bm->m.find(seq_ids[i]);
    int32_t* row = out + static_cast<int64_t>(i) * cap;
    int32_t m = static_cast<int32_t>(s->table.size());
    if (m) std::memcpy(row, s->table.data(), sizeof(int32_t) * m);
    for (int32_t j = m; j < cap; ++j) row[j] = pad;
    lens_out[i] = static_cast<int32_t>(s->len);
  }
  return PA_OK;
}

// Shared-prefix groups of a decode batch (P2 §3.4: sequences that share a
// prefix hold the same physical blocks; P1 "跨请求的内存共享": the samples of
// one prompt). Sequences are keyed by the physical id of their first block
// (only those with at least one whole block take part), keys in order of first
// appearance in the batch; each key's sequences, in batch order, are cut into
// groups of at most max_group_size. A group's prefix is the longest run of
// leading table entries that every member holds identically, counted over the
// whole blocks of its shortest member and cut down to a multiple of
// align_tokens; a group of one member, or with a prefix of zero tokens, is
// dropped and its sequences get no prefix.
pa_status pa_bm_longest_first(const pa_bm* bm, int32_t n, const int64_t* seq_ids, const int32_t* skip_tokens,
                              int32_t* order) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !order))) return PA_ERR_INVALID_ARG;
  std::vector<int64_t> span(n);
  for (int32_t i = 0; i < n; ++i) {
    const Seq* q = bm->m.find(seq_ids[i]);
    if (!q) return PA_ERR_UNKNOWN_SEQ;
    span[i] = q->len - (skip_tokens ? skip_tokens[i] : 0);
  }
  for (int32_t i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order, order + n, [&](int32_t x, int32_t y) { return span[x] > span[y]; });
  return PA_OK;
}

pa_status pa_bm_prefix_groups(const pa_bm* bm, int32_t n, const int64_t* seq_ids, int32_t max_group_size,
                              int32_t align_tokens, int32_t* group_offsets, int32_t* group_members,
                              int32_t* group_prefix_tokens, int32_t* seq_prefix_tokens, int32_t* n_groups_out,
                              int32_t* max_prefix_out) {
  if (!bm || n < 0 || max_group_size < 1 || align_tokens < 1 || !group_offsets || !n_groups_out ||
      (n > 0 && (!seq_ids || !group_members || !group_prefix_tokens || !seq_prefix_tokens)))
    return PA_ERR_INVALID_ARG;
  const int32_t bs = bm->m.block_size();
  std::vector<const Seq*> seqs(n);
  for (int32_t i = 0; i < n; ++i) {
    seqs[i] = bm->m.find(seq_ids[i]);
    if (!seqs[i]) return PA_ERR_UNKNOWN_SEQ;
  }
  std::unordered_map<int32_t, std::vector<int32_t>> by_first;
  std::vector<int32_t> keys;
  for (int32_t i = 0; i < n; ++i) {
    if (seqs[i]->len < bs) continue;
    auto it = by_first.find(seqs[i]->table[0]);
    if (it == by_first.end()) {
      keys.push_back(seqs[i]->table[0]);
      by_first.emplace(seqs[i]->table[0], std::vector<int32_t>{i});
    } else {
      it->second.push_back(i);
    }
  }
  int32_t ng = 0, nm = 0, maxp = 0;
  group_offsets[0] = 0;
  for (int32_t i = 0; i < n; ++i) seq_prefix_tokens[i] = 0;
  for (int32_t key : keys) {
    const std::vector<int32_t>& rows = by_first[key];
    for (size_t c0 = 0; c0 < rows.size(); c0 += max_group_size) {
      const size_t c1 = std::min(rows.size(), c0 + static_cast<size_t>(max_group_size));
      if (c1 - c0 < 2) continue;
      int64_t full = INT64_MAX;
      for (size_t u = c0; u < c1; ++u) full = std::min(full, seqs[rows[u]]->len / bs);
      const std::vector<int32_t>& t0 = seqs[rows[c0]]->table;
      int64_t k = 0;
      for (; k < full; ++k) {
        bool same = true;
        for (size_t u = c0 + 1; u < c1 && same; ++u) same = seqs[rows[u]]->table[k] == t0[k];
        if (!same) break;
      }
      const int64_t ptok = k * bs / align_tokens * align_tokens;
      if (ptok == 0) continue;
      if (ptok > INT32_MAX) return PA_ERR_UNSUPPORTED;
      for (size_t u = c0; u < c1; ++u) {
        group_members[nm++] = rows[u];
        seq_prefix_tokens[rows[u]] = static_cast<int32_t>(ptok);
      }
      group_prefix_tokens[ng] = static_cast<int32_t>(ptok);
      group_offsets[++ng] = nm;
      maxp = std::max(maxp, static_cast<int32_t>(ptok));
    }
  }
  *n_groups_out = ng;
  if (max_prefix_out) *max_prefix_out = maxp;
  return PA_OK;
}

pa_status pa_bm_refcount(const pa_bm* bm, int32_t block, int32_t* out) {
  if (!bm || !out || block < 0 || block >= bm->m.num_blocks()) return PA_ERR_INVALID_ARG;
  *out = bm->m.ref(block);
  return PA_OK;
}

pa_status pa_bm_stats(const pa_bm* bm, int64_t* free_blocks, int64_t* used_slots, int64_t* allocated_slots) {
  if (!bm) return PA_ERR_INVALID_ARG;
  bm->m.stats(free_blocks, used_slots, allocated_slots);
  return PA_OK;
}

pa_status pa_bm_free_list(const pa_bm* bm, int32_t* out, int64_t cap, int64_t* n_out) {
  if (!bm || cap < 0 || (cap > 0 && !out)) return PA_ERR_INVALID_ARG;
  bm->m.free_list(out, cap, n_out);
  return PA_OK;
}

}  // extern "C"
