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
// The free list is a FIFO ring over a fixed array (front = next allocation,
// back = most recently freed), so every operation is O(blocks touched).
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pagedattn.h"

namespace {

struct Seq {
  std::vector<int32_t> table;
  int64_t len = 0;
};

class BlockManager {
 public:
  BlockManager(int64_t num_blocks, int32_t block_size)
      : nb_(num_blocks), bs_(block_size), ring_(num_blocks), ref_(num_blocks, 0) {}

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
    if (seqs_.count(id)) return PA_ERR_SEQ_EXISTS;
    int64_t need = (static_cast<int64_t>(n) + bs_ - 1) / bs_;
    if (need > count_) return PA_ERR_NO_FREE_BLOCKS;
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
    if (seqs_.count(child)) return PA_ERR_SEQ_EXISTS;
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
    if (blocks_needed(s) > count_) return PA_ERR_NO_FREE_BLOCKS;
    do_append(s, slot, pair);
    return PA_OK;
  }

  pa_status append_many(int32_t n, const int64_t* ids, int64_t* slots, int32_t* pairs, int32_t* n_pairs) {
    // Dry run on shadow lengths and counts so that the batch is all or nothing.
    // After an append at length L the block at logical index L / bs is private
    // to the sequence (fresh, copied, or already held once), and counts only
    // fall during a batch, so a later append into the same index copies nothing.
    struct Shadow {
      int64_t len;
      int64_t private_bi;
    };
    std::unordered_map<int64_t, Shadow> sh;
    std::unordered_map<int32_t, int32_t> dref;
    int64_t need = 0;
    for (int32_t i = 0; i < n; ++i) {
      auto it = seqs_.find(ids[i]);
      if (it == seqs_.end()) return PA_ERR_UNKNOWN_SEQ;
      const Seq& s = it->second;
      auto ins = sh.emplace(ids[i], Shadow{s.len, -1});
      Shadow& st = ins.first->second;
      int64_t bi = st.len / bs_;
      if (st.len % bs_ == 0) {
        ++need;
      } else if (bi != st.private_bi) {
        int32_t b = s.table[bi];
        if (ref_[b] + dref[b] > 1) {
          ++need;
          dref[b] -= 1;
        }
      }
      st.private_bi = bi;
      st.len += 1;
    }
    if (need > count_) return PA_ERR_NO_FREE_BLOCKS;
    int32_t np = 0;
    for (int32_t i = 0; i < n; ++i) {
      int32_t pr[2];
      do_append(seqs_.find(ids[i])->second, &slots[i], pr);
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
    auto it = seqs_.find(id);
    if (it == seqs_.end()) return PA_ERR_UNKNOWN_SEQ;
    for (int32_t b : it->second.table)
      if (--ref_[b] == 0) push(b);
    seqs_.erase(it);
    return PA_OK;
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
  int32_t pop() {
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
  for (int32_t i = 0; i < n; ++i) {
    const Seq* s = bm->m.find(seq_ids[i]);
    if (!s) return PA_ERR_UNKNOWN_SEQ;
    if (static_cast<int64_t>(s->table.size()) > cap || s->len > INT32_MAX) return PA_ERR_INVALID_ARG;
  }
  for (int32_t i = 0; i < n; ++i) {
    const Seq* s = bm->m.find(seq_ids[i]);
    int32_t* row = out + static_cast<int64_t>(i) * cap;
    int32_t m = static_cast<int32_t>(s->table.size());
    if (m) std::memcpy(row, s->table.data(), sizeof(int32_t) * m);
    for (int32_t j = m; j < cap; ++j) row[j] = pad;
    lens_out[i] = static_cast<int32_t>(s->len);
  }
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
