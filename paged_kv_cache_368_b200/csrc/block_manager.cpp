// Host-side block manager: the pool lifecycle of "PagedAttention：KV Cache 的分页革命"
// (section Runtime 如何管理 KV Block: initialise a pool of fixed-size blocks,
// take a free block when a step needs cache space, update the page table,
// return blocks when a request finishes) and of "【infra之路】10-PagedAttention 与
// KV Cache 管理" (section 3.3: one block table per request, a new physical
// block appended when the last one is full; section 4.3: requests sharing a
// prefix, or beams, point at the same physical blocks, copied on write;
// section 6: the scheduler admits work by the number of free blocks;
// preemption swaps a request's blocks to another pool).
//
// Policy choices the pages leave open:
//  * a free block is taken lowest id first (deterministic);
//  * a block shared by several sequences is copied before one of them
//    writes into it; the caller performs the copy with pa_copy_blocks using
//    the (src, dst) pair returned;
//  * running out of blocks is an error (PA_ERR_OUT_OF_BLOCKS), never a
//    silent reuse of block 0.
// Not thread-safe: one manager per scheduler thread.
#include <algorithm>
#include <cstdint>
#include <new>
#include <set>
#include <unordered_map>
#include <vector>

#include "paged.h"

struct pa_block_manager {
  int64_t num_blocks;
  int block_size;
  std::set<int64_t> free_blocks;
  std::vector<int32_t> refcount;
  struct Seq {
    std::vector<int64_t> blocks;
    int64_t len = 0;
  };
  std::unordered_map<int64_t, Seq> seqs;

  bool take(int64_t* out) {
    if (free_blocks.empty()) return false;
    auto it = free_blocks.begin();
    *out = *it;
    free_blocks.erase(it);
    refcount[*out] = 1;
    return true;
  }
  void release(int64_t b) {
    if (--refcount[b] == 0) free_blocks.insert(b);
  }
};

namespace {
int64_t blocks_for(int64_t tokens, int bs) { return (tokens + bs - 1) / bs; }
}  // namespace

extern "C" pa_block_manager* pa_bm_create(int64_t num_blocks, int block_size) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pa_block_manager* m = new (std::nothrow) pa_block_manager;
  if (!m) return nullptr;
  try {
    m->num_blocks = num_blocks;
    m->block_size = block_size;
    m->refcount.assign(static_cast<size_t>(num_blocks), 0);
    for (int64_t b = 0; b < num_blocks; ++b) m->free_blocks.insert(m->free_blocks.end(), b);
  } catch (...) {
    delete m;
    return nullptr;
  }
  return m;
}

extern "C" void pa_bm_destroy(pa_block_manager* m) { delete m; }

extern "C" int64_t pa_bm_num_free_blocks(const pa_block_manager* m) {
  return m ? static_cast<int64_t>(m->free_blocks.size()) : -1;
}

extern "C" pa_status pa_bm_add_sequence(pa_block_manager* m, int64_t seq_id, int64_t num_tokens) {
  if (!m || num_tokens < 0) return PA_ERR_INVALID;
  if (m->seqs.count(seq_id)) return PA_ERR_INVALID;
  const int64_t need = blocks_for(num_tokens, m->block_size);
  if (need > static_cast<int64_t>(m->free_blocks.size())) return PA_ERR_OUT_OF_BLOCKS;
  pa_block_manager::Seq s;
  s.len = num_tokens;
  s.blocks.reserve(static_cast<size_t>(need));
  for (int64_t i = 0; i < need; ++i) {
    int64_t b;
    m->take(&b);
    s.blocks.push_back(b);
  }
  m->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

extern "C" pa_status pa_bm_fork(pa_block_manager* m, int64_t parent, int64_t child) {
  if (!m || parent == child) return PA_ERR_INVALID;
  auto it = m->seqs.find(parent);
  if (it == m->seqs.end() || m->seqs.count(child)) return PA_ERR_INVALID;
  pa_block_manager::Seq s = it->second;  // copy the table, not the KV
  for (int64_t b : s.blocks) ++m->refcount[b];
  m->seqs.emplace(child, std::move(s));
  return PA_OK;
}

extern "C" pa_status pa_bm_append_slot(pa_block_manager* m, int64_t seq_id, int64_t* slot, int64_t* cow_src,
                                       int64_t* cow_dst) {
  if (!m || !slot) return PA_ERR_INVALID;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID;
  pa_block_manager::Seq& s = it->second;
  const int64_t pos = s.len;  // position of the new token
  const int bs = m->block_size;
  int64_t src = -1, dst = -1;
  if (pos % bs == 0) {  // the last block is full (or there is none): a new block
    int64_t b;
    if (!m->take(&b)) return PA_ERR_OUT_OF_BLOCKS;
    s.blocks.push_back(b);
  } else {
    int64_t& last = s.blocks.back();
    if (m->refcount[last] > 1) {  // shared: copy on write
      int64_t b;
      if (!m->take(&b)) return PA_ERR_OUT_OF_BLOCKS;
      src = last;
      dst = b;
      --m->refcount[last];
      last = b;
    }
  }
  s.len = pos + 1;
  *slot = s.blocks[static_cast<size_t>(pos / bs)] * bs + pos % bs;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_OK;
}

extern "C" pa_status pa_bm_free_sequence(pa_block_manager* m, int64_t seq_id) {
  if (!m) return PA_ERR_INVALID;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID;
  for (int64_t b : it->second.blocks) m->release(b);
  m->seqs.erase(it);
  return PA_OK;
}

extern "C" int64_t pa_bm_context_len(const pa_block_manager* m, int64_t seq_id) {
  if (!m) return -1;
  auto it = m->seqs.find(seq_id);
  return it == m->seqs.end() ? -1 : it->second.len;
}

extern "C" pa_status pa_bm_block_table(const pa_block_manager* m, int64_t seq_id, int32_t* table, int max_blocks,
                                       int* num_blocks) {
  if (!m || !num_blocks) return PA_ERR_INVALID;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_INVALID;
  const auto& b = it->second.blocks;
  *num_blocks = static_cast<int>(b.size());
  if (static_cast<int64_t>(b.size()) > max_blocks) return PA_ERR_INVALID;
  if (table) {
    for (size_t i = 0; i < b.size(); ++i) table[i] = static_cast<int32_t>(b[i]);
    for (int i = static_cast<int>(b.size()); i < max_blocks; ++i) table[i] = -1;
  }
  return PA_OK;
}

extern "C" int64_t pa_bm_blocks_needed_to_append(const pa_block_manager* m, const int64_t* seq_ids, int num_seqs) {
  if (!m || (num_seqs > 0 && !seq_ids)) return -1;
  // A full last block (or none) takes a new block.  A partly filled last
  // block held by r sequences is copied by each holder that writes while
  // others still hold it: k holders appending in one batch take min(k, r-1)
  // blocks, the last writer keeps the original.
  int64_t need = 0;
  std::unordered_map<int64_t, int32_t> copies;  // shared last block -> copies taken so far
  for (int i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end()) return -1;
    const auto& s = it->second;
    if (s.len % m->block_size == 0) {
      ++need;
      continue;
    }
    const int64_t last = s.blocks.back();
    int32_t& taken = copies[last];
    if (m->refcount[last] - taken > 1) {
      ++taken;
      ++need;
    }
  }
  return need;
}

extern "C" pa_status pa_bm_prepare_decode(pa_block_manager* m, const int64_t* seq_ids, int num_seqs,
                                          int max_blocks_per_seq, int32_t* block_tables, int32_t* context_lens,
                                          int64_t* slot_mapping, int64_t* cow_pairs, int64_t* num_cow_pairs) {
  if (!m || num_seqs < 0 || max_blocks_per_seq <= 0 || !num_cow_pairs) return PA_ERR_INVALID;
  if (num_seqs > 0 && (!seq_ids || !block_tables || !context_lens || !slot_mapping || !cow_pairs))
    return PA_ERR_INVALID;
  // Check everything first so that a failing call changes nothing.
  for (int i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end()) return PA_ERR_INVALID;
    for (int j = 0; j < i; ++j)
      if (seq_ids[j] == seq_ids[i]) return PA_ERR_INVALID;
    if (blocks_for(it->second.len + 1, m->block_size) > max_blocks_per_seq) return PA_ERR_INVALID;
  }
  const int64_t need = pa_bm_blocks_needed_to_append(m, seq_ids, num_seqs);
  if (need > static_cast<int64_t>(m->free_blocks.size())) return PA_ERR_OUT_OF_BLOCKS;
  int64_t ncow = 0;
  for (int i = 0; i < num_seqs; ++i) {
    int64_t src, dst;
    pa_bm_append_slot(m, seq_ids[i], &slot_mapping[i], &src, &dst);
    if (src >= 0) {
      cow_pairs[2 * ncow] = src;
      cow_pairs[2 * ncow + 1] = dst;
      ++ncow;
    }
    const auto& s = m->seqs.find(seq_ids[i])->second;
    context_lens[i] = static_cast<int32_t>(s.len);
    int nb = 0;
    pa_bm_block_table(m, seq_ids[i], block_tables + static_cast<int64_t>(i) * max_blocks_per_seq, max_blocks_per_seq,
                      &nb);
  }
  *num_cow_pairs = ncow;
  return PA_OK;
}

extern "C" pa_status pa_bm_swap_sequence(pa_block_manager* from, pa_block_manager* to, int64_t seq_id,
                                         int64_t* pairs, int64_t max_pairs, int64_t* num_pairs) {
  if (!from || !to || from == to || !num_pairs || from->block_size != to->block_size) return PA_ERR_INVALID;
  auto it = from->seqs.find(seq_id);
  if (it == from->seqs.end() || to->seqs.count(seq_id)) return PA_ERR_INVALID;
  const auto& src = it->second.blocks;
  const int64_t n = static_cast<int64_t>(src.size());
  if (n > max_pairs || (n > 0 && !pairs)) return PA_ERR_INVALID;
  if (n > static_cast<int64_t>(to->free_blocks.size())) return PA_ERR_OUT_OF_BLOCKS;
  pa_block_manager::Seq moved;
  moved.len = it->second.len;
  for (int64_t i = 0; i < n; ++i) {
    int64_t b;
    to->take(&b);
    moved.blocks.push_back(b);
    pairs[2 * i] = src[static_cast<size_t>(i)];
    pairs[2 * i + 1] = b;
  }
  for (int64_t b : src) from->release(b);
  from->seqs.erase(it);
  to->seqs.emplace(seq_id, std::move(moved));
  *num_pairs = n;
  return PA_OK;
}
