// pa_blockmgr.cpp -- host block manager that produces the metadata the
// kernels consume: block tables, slot mappings and copy-on-write pairs.
//
// Rules from "PagedAttention" (shubhamtatvamasi.com):
//  - "The idea: page the KV cache": a sequence takes a new physical block only
//    once its last one has no free slot (as an OS maps a page on first use),
//    and any free block will do, wherever it lies;
//  - "Sharing and copy-on-write": several tables may name one physical
//    block, which counts its holders; a block with no free slot left is
//    never written to again;
//  - "How does copy-on-write work for parallel sampling?": before a sequence
//    adds a token to a partially filled block that others also hold, it takes
//    a fresh block, gets the tokens already there duplicated into it, gives
//    up its hold on the old block and continues in the fresh one.
// The copy itself is the device's job (pa_copy_blocks); this manager returns
// the (src, dst) pair.
//
// Prefix caching ("Sharing and copy-on-write": requests that begin with one
// system prompt can hold the same blocks, and since a block with no free slot
// is not written to again, holding it together is safe while it lives): a
// full block added with its token ids is
// entered in an index under (the physical block before it, its tokens); a
// later request whose prompt starts with the same tokens finds its leading
// full blocks there and shares them.  The match is exact (the tokens are
// compared, not only hashed) and chained (a block matches only after its
// predecessor did).  An entry lives as long as its block is held.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pagedattn.h"

struct pa_block_manager {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::deque<int32_t> free_list;
  std::vector<int32_t> refcount;
  struct Seq {
    std::vector<int32_t> table;
    int64_t tokens = 0;
  };
  std::unordered_map<int64_t, Seq> seqs;
  // prefix cache: entry of a physical block (valid while the block is held)
  struct Cached {
    bool valid = false;
    uint64_t key = 0;
    int32_t parent = -1;          // the physical block before it in its table
    std::vector<int32_t> tokens;  // its block_size token ids
  };
  std::vector<Cached> cached;
  std::unordered_multimap<uint64_t, int32_t> prefix_index;  // key -> block
  int64_t num_cached = 0;

  static uint64_t key_of(int32_t parent, const int32_t* tokens, int32_t n) {
    uint64_t h = 1469598103934665603ull;  // FNV-1a over the parent id and the tokens
    auto mix = [&h](uint32_t v) {
      for (int b = 0; b < 4; ++b) {
        h ^= (v >> (8 * b)) & 0xffu;
        h *= 1099511628211ull;
      }
    };
    mix(static_cast<uint32_t>(parent));
    for (int32_t i = 0; i < n; ++i) mix(static_cast<uint32_t>(tokens[i]));
    return h;
  }
  // the held block whose entry is (parent, tokens), or -1
  int32_t find_cached(int32_t parent, const int32_t* tokens) const {
    const uint64_t key = key_of(parent, tokens, block_size);
    auto range = prefix_index.equal_range(key);
    for (auto it = range.first; it != range.second; ++it) {
      const Cached& c = cached[static_cast<size_t>(it->second)];
      if (c.parent == parent &&
          std::equal(c.tokens.begin(), c.tokens.end(), tokens))
        return it->second;
    }
    return -1;
  }
  void enter_cached(int32_t blk, int32_t parent, const int32_t* tokens) {
    Cached& c = cached[static_cast<size_t>(blk)];
    c.valid = true;
    c.key = key_of(parent, tokens, block_size);
    c.parent = parent;
    c.tokens.assign(tokens, tokens + block_size);
    prefix_index.emplace(c.key, blk);
    ++num_cached;
  }
  void forget_cached(int32_t blk) {
    Cached& c = cached[static_cast<size_t>(blk)];
    if (!c.valid) return;
    auto range = prefix_index.equal_range(c.key);
    for (auto it = range.first; it != range.second; ++it) {
      if (it->second == blk) {
        prefix_index.erase(it);
        break;
      }
    }
    c = Cached();
    --num_cached;
  }

  bool alloc(int32_t* out) {
    if (free_list.empty()) return false;
    *out = free_list.front();
    free_list.pop_front();
    refcount[*out] = 1;
    return true;
  }
  void release(int32_t blk) {
    if (--refcount[blk] == 0) {
      forget_cached(blk);
      free_list.push_back(blk);
    }
  }
};

extern "C" pa_status pa_bm_create(int32_t num_blocks, int32_t block_size,
                                  const int32_t* free_order, pa_block_manager** out) {
  if (out == nullptr || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  pa_block_manager* bm = new (std::nothrow) pa_block_manager();
  if (bm == nullptr) return PA_ERR_INVALID_ARG;
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->refcount.assign(num_blocks, 0);
  bm->cached.resize(static_cast<size_t>(num_blocks));
  if (free_order == nullptr) {
    for (int32_t i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
  } else {
    std::vector<char> seen(num_blocks, 0);
    for (int32_t i = 0; i < num_blocks; ++i) {
      const int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return PA_ERR_INVALID_ARG;  // not a permutation
      }
      seen[b] = 1;
      bm->free_list.push_back(b);
    }
  }
  *out = bm;
  return PA_OK;
}

extern "C" void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

extern "C" pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq, int64_t num_tokens) {
  if (bm == nullptr || num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (bm->seqs.count(seq)) return PA_ERR_INVALID_ARG;
  const int64_t need = (num_tokens + bm->block_size - 1) / bm->block_size;
  if (need > static_cast<int64_t>(bm->free_list.size())) return PA_ERR_OUT_OF_BLOCKS;
  pa_block_manager::Seq s;
  s.tokens = num_tokens;
  s.table.reserve(static_cast<size_t>(need));
  for (int64_t i = 0; i < need; ++i) {
    int32_t blk;
    bm->alloc(&blk);
    s.table.push_back(blk);
  }
  bm->seqs.emplace(seq, std::move(s));
  return PA_OK;
}

// A new request of num_tokens prompt tokens `token_ids`: its leading full
// blocks that match the prefix cache are shared (their key and value rows are
// already in the pool: *cached_tokens of them, a multiple of block_size), the
// rest are allocated, and its own full blocks are entered in the cache.  The
// caller writes the rows of tokens cached_tokens .. num_tokens - 1 before any
// attention reads them.  All or nothing.
extern "C" pa_status pa_bm_add_sequence_with_prefix(pa_block_manager* bm, int64_t seq,
                                                    const int32_t* token_ids,
                                                    int64_t num_tokens,
                                                    int64_t* cached_tokens) {
  if (bm == nullptr || num_tokens < 0 || cached_tokens == nullptr ||
      (num_tokens > 0 && token_ids == nullptr))
    return PA_ERR_INVALID_ARG;
  if (bm->seqs.count(seq)) return PA_ERR_INVALID_ARG;
  const int32_t bs = bm->block_size;
  const int64_t full = num_tokens / bs;
  const int64_t need_all = (num_tokens + bs - 1) / bs;
  // leading full blocks found in the cache
  std::vector<int32_t> hits;
  int32_t parent = -1;
  for (int64_t i = 0; i < full; ++i) {
    const int32_t blk = bm->find_cached(parent, token_ids + i * bs);
    if (blk < 0) break;
    hits.push_back(blk);
    parent = blk;
  }
  const int64_t fresh = need_all - static_cast<int64_t>(hits.size());
  if (fresh > static_cast<int64_t>(bm->free_list.size())) return PA_ERR_OUT_OF_BLOCKS;
  pa_block_manager::Seq s;
  s.tokens = num_tokens;
  s.table.reserve(static_cast<size_t>(need_all));
  for (int32_t blk : hits) {
    ++bm->refcount[static_cast<size_t>(blk)];
    s.table.push_back(blk);
  }
  for (int64_t i = static_cast<int64_t>(hits.size()); i < need_all; ++i) {
    int32_t blk;
    bm->alloc(&blk);
    if (i < full) bm->enter_cached(blk, s.table.empty() ? -1 : s.table.back(), token_ids + i * bs);
    s.table.push_back(blk);
  }
  bm->seqs.emplace(seq, std::move(s));
  *cached_tokens = static_cast<int64_t>(hits.size()) * bs;
  return PA_OK;
}

extern "C" pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child) {
  if (bm == nullptr) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
  if (bm->seqs.count(child)) return PA_ERR_INVALID_ARG;
  pa_block_manager::Seq s = it->second;
  for (int32_t blk : s.table) ++bm->refcount[blk];
  bm->seqs.emplace(child, std::move(s));
  return PA_OK;
}

extern "C" pa_status pa_bm_append_slot(pa_block_manager* bm, int64_t seq, int64_t* slot,
                                       int32_t* cow_src, int32_t* cow_dst) {
  if (bm == nullptr || slot == nullptr) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
  pa_block_manager::Seq& s = it->second;
  const int64_t pos = s.tokens;
  const int32_t bs = bm->block_size;
  int32_t src = -1, dst = -1;
  if (pos % bs == 0) {
    int32_t blk;
    if (!bm->alloc(&blk)) return PA_ERR_OUT_OF_BLOCKS;
    s.table.push_back(blk);
  } else {
    const int32_t last = s.table.back();
    if (bm->refcount[last] > 1) {
      int32_t blk;
      if (!bm->alloc(&blk)) return PA_ERR_OUT_OF_BLOCKS;
      --bm->refcount[last];
      s.table.back() = blk;
      src = last;
      dst = blk;
    }
  }
  *slot = static_cast<int64_t>(s.table[pos / bs]) * bs + pos % bs;
  s.tokens = pos + 1;
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_OK;
}

extern "C" pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq) {
  if (bm == nullptr) return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
  for (int32_t blk : it->second.table) bm->release(blk);
  bm->seqs.erase(it);
  return PA_OK;
}

extern "C" pa_status pa_bm_block_table(const pa_block_manager* bm, int64_t seq, int32_t* out,
                                       int32_t capacity, int32_t* num_blocks,
                                       int64_t* num_tokens) {
  if (bm == nullptr || capacity < 0 || (capacity > 0 && out == nullptr))
    return PA_ERR_INVALID_ARG;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
  const std::vector<int32_t>& t = it->second.table;
  const int32_t n = static_cast<int32_t>(t.size());
  for (int32_t i = 0; i < n && i < capacity; ++i) out[i] = t[i];
  if (num_blocks) *num_blocks = n;
  if (num_tokens) *num_tokens = it->second.tokens;
  return PA_OK;
}

// Sequences forked from one parent share the parent's leading blocks until
// they diverge ("Sharing and copy-on-write"); the count is read off the tables.
extern "C" pa_status pa_bm_shared_blocks(const pa_block_manager* bm, const int64_t* seqs,
                                         int32_t n, int32_t* out) {
  if (bm == nullptr || n < 0 || (n > 0 && (seqs == nullptr || out == nullptr)))
    return PA_ERR_INVALID_ARG;
  const std::vector<int32_t>* prev = nullptr;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
    const std::vector<int32_t>& t = it->second.table;
    if (prev != nullptr) {
      size_t k = 0;
      while (k < prev->size() && k < t.size() && (*prev)[k] == t[k]) ++k;
      out[i - 1] = static_cast<int32_t>(k);
    }
    prev = &t;
  }
  if (n > 0) out[n - 1] = 0;
  return PA_OK;
}

// A batch order that puts sequences holding the same leading blocks next to
// each other (the samples of one prompt, requests of one cached system
// prompt), so that pa_decode_attention_shared_prefix finds them in its
// windows: the sequences sorted by their block tables read as words (ties
// keep the given order).  order[i] = the index into seqs of the i-th
// sequence of the new order.
extern "C" pa_status pa_bm_order_by_prefix(const pa_block_manager* bm, const int64_t* seqs,
                                           int32_t n, int32_t* order) {
  if (bm == nullptr || n < 0 || (n > 0 && (seqs == nullptr || order == nullptr)))
    return PA_ERR_INVALID_ARG;
  std::vector<const std::vector<int32_t>*> tabs(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
    tabs[static_cast<size_t>(i)] = &it->second.table;
  }
  std::vector<int32_t> idx(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) idx[static_cast<size_t>(i)] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
    return std::lexicographical_compare(tabs[a]->begin(), tabs[a]->end(), tabs[b]->begin(),
                                        tabs[b]->end());
  });
  std::copy(idx.begin(), idx.end(), order);
  return PA_OK;
}

extern "C" int32_t pa_bm_refcount(const pa_block_manager* bm, int32_t block) {
  if (bm == nullptr || block < 0 || block >= bm->num_blocks) return -1;
  return bm->refcount[block];
}

extern "C" int32_t pa_bm_num_free(const pa_block_manager* bm) {
  return bm == nullptr ? -1 : static_cast<int32_t>(bm->free_list.size());
}

namespace {

// The sequences of a batch, checked: known, listed once, counts >= 0 (NULL
// counts = one token each).  *total gets the sum of the counts.
pa_status batch_rows(pa_block_manager* bm, const int64_t* seqs, int32_t n, const int32_t* counts,
                     std::vector<pa_block_manager::Seq*>* rows, int64_t* total) {
  rows->assign(static_cast<size_t>(n), nullptr);
  std::unordered_map<int64_t, int32_t> seen;
  *total = 0;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
    const int32_t c = counts ? counts[i] : 1;
    if (c < 0 || !seen.emplace(seqs[i], i).second) return PA_ERR_INVALID_ARG;
    (*rows)[static_cast<size_t>(i)] = &it->second;
    *total += c;
  }
  return PA_OK;
}

// Blocks the free list must give for the batch's appends, without changing
// anything: for each sequence in order, a copy when its first new token falls
// into a partial last block that some other sequence still holds (replaying
// the reference counts the earlier copies of the batch release: the last
// holder writes in place), then one block per block boundary its new tokens
// start.
int64_t blocks_needed(const pa_block_manager* bm,
                      const std::vector<pa_block_manager::Seq*>& rows, const int32_t* counts) {
  const int64_t bs = bm->block_size;
  std::unordered_map<int32_t, int32_t> drop;
  int64_t need = 0;
  for (size_t i = 0; i < rows.size(); ++i) {
    const int32_t c = counts ? counts[i] : 1;
    if (c == 0) continue;
    const pa_block_manager::Seq& s = *rows[i];
    if (s.tokens % bs != 0) {
      const int32_t last = s.table.back();
      if (bm->refcount[static_cast<size_t>(last)] - drop[last] > 1) {
        ++need;
        ++drop[last];
      }
    }
    need += (s.tokens + c + bs - 1) / bs - (s.tokens + bs - 1) / bs;
  }
  return need;
}

// The appends themselves, after the checks and the dry run.
void append_batch(pa_block_manager* bm, const int64_t* seqs, int32_t n, const int32_t* counts,
                  int32_t* slot_mapping, int32_t* q_start, int32_t* cow_pairs, int32_t* num_cow) {
  int32_t row = 0;
  for (int32_t i = 0; i < n; ++i) {
    if (q_start) q_start[i] = row;
    const int32_t c = counts ? counts[i] : 1;
    for (int32_t j = 0; j < c; ++j) {
      int64_t slot;
      int32_t src, dst;
      pa_bm_append_slot(bm, seqs[i], &slot, &src, &dst);  // cannot fail: the dry run
      slot_mapping[row++] = static_cast<int32_t>(slot);  // found every block
      if (src >= 0) {
        cow_pairs[2 * *num_cow] = src;
        cow_pairs[2 * *num_cow + 1] = dst;
        ++*num_cow;
      }
    }
  }
  if (q_start && n > 0) q_start[n] = row;
}

pa_status append_checked(pa_block_manager* bm, const int64_t* seqs, int32_t n,
                         const int32_t* counts, int32_t* slot_mapping, int32_t* q_start,
                         int32_t* cow_pairs, int32_t* num_cow) {
  if (bm == nullptr || n < 0 || num_cow == nullptr ||
      (n > 0 && (seqs == nullptr || cow_pairs == nullptr)))
    return PA_ERR_INVALID_ARG;
  *num_cow = 0;
  if (static_cast<int64_t>(bm->num_blocks) * bm->block_size - 1 > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  std::vector<pa_block_manager::Seq*> rows;
  int64_t total = 0;
  const pa_status st = batch_rows(bm, seqs, n, counts, &rows, &total);
  if (st != PA_OK) return st;
  if (total > INT32_MAX || (total > 0 && slot_mapping == nullptr)) return PA_ERR_INVALID_ARG;
  if (blocks_needed(bm, rows, counts) > static_cast<int64_t>(bm->free_list.size()))
    return PA_ERR_OUT_OF_BLOCKS;
  append_batch(bm, seqs, n, counts, slot_mapping, q_start, cow_pairs, num_cow);
  return PA_OK;
}

}  // namespace

// One step's appends for a batch: the slot of every listed sequence's next
// token and the copy-on-write pairs, in order, as pa_bm_append_slot would give
// them one by one; a batch that does not fit changes nothing.
extern "C" pa_status pa_bm_append_slots(pa_block_manager* bm, const int64_t* seqs, int32_t n,
                                        int32_t* slot_mapping, int32_t* cow_pairs,
                                        int32_t* num_cow) {
  return append_checked(bm, seqs, n, nullptr, slot_mapping, nullptr, cow_pairs, num_cow);
}

// Several new tokens per sequence (chunked prefill, speculative tokens): the
// slots of counts[i] consecutive tokens of seqs[i], for i in order, laid out
// as the query rows of pa_decode_attention_multi_query (sequence i's tokens
// at rows q_start[i] .. q_start[i + 1] - 1).  A sequence copies a shared
// partial last block at most once, on its first new token.
extern "C" pa_status pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seqs, int32_t n,
                                         const int32_t* counts, int32_t* slot_mapping,
                                         int32_t* q_start, int32_t* cow_pairs,
                                         int32_t* num_cow) {
  if (n > 0 && (counts == nullptr || q_start == nullptr)) return PA_ERR_INVALID_ARG;
  return append_checked(bm, seqs, n, counts, slot_mapping, q_start, cow_pairs, num_cow);
}

// What a scheduler asks before it admits a batch: the free blocks the appends
// would take (0 .. ), with no change to any table.
extern "C" pa_status pa_bm_blocks_needed(const pa_block_manager* bm, const int64_t* seqs,
                                         int32_t n, const int32_t* counts, int64_t* need) {
  if (bm == nullptr || n < 0 || need == nullptr || (n > 0 && seqs == nullptr))
    return PA_ERR_INVALID_ARG;
  std::vector<pa_block_manager::Seq*> rows;
  int64_t total = 0;
  const pa_status st =
      batch_rows(const_cast<pa_block_manager*>(bm), seqs, n, counts, &rows, &total);
  if (st != PA_OK) return st;
  *need = blocks_needed(bm, rows, counts);
  return PA_OK;
}

// The decode kernels' metadata for a batch: row i of `tables` (row stride
// `width`) is the block table of seqs[i] padded with -1, seq_lens[i] its
// length.  Nothing is written if a sequence is unknown, holds more than
// `width` blocks or more than INT32_MAX tokens.
extern "C" pa_status pa_bm_fill_tables(const pa_block_manager* bm, const int64_t* seqs,
                                       int32_t n, int32_t* tables, int32_t width,
                                       int32_t* seq_lens) {
  if (bm == nullptr || n < 0 || width < 0 ||
      (n > 0 && (seqs == nullptr || (width > 0 && tables == nullptr))))
    return PA_ERR_INVALID_ARG;
  std::vector<const pa_block_manager::Seq*> rows(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seqs[i]);
    if (it == bm->seqs.end()) return PA_ERR_NOT_FOUND;
    if (it->second.table.size() > static_cast<size_t>(width) || it->second.tokens > INT32_MAX)
      return PA_ERR_INVALID_ARG;
    rows[i] = &it->second;
  }
  for (int32_t i = 0; i < n; ++i) {
    const std::vector<int32_t>& t = rows[i]->table;
    int32_t* row = tables + static_cast<int64_t>(i) * width;
    std::copy(t.begin(), t.end(), row);
    std::fill(row + t.size(), row + width, -1);
    if (seq_lens) seq_lens[i] = static_cast<int32_t>(rows[i]->tokens);
  }
  return PA_OK;
}

// Memory the sequences hold ("PagedAttention", "The idea: page the KV cache":
// only a sequence's last block can be partly empty, so waste stays under one
// block per sequence; "Sharing and copy-on-write": a shared block is held
// once).  A slot counts as stored when some sequence holding the block has a
// token there.
extern "C" pa_status pa_bm_stats(const pa_block_manager* bm, pa_bm_stats_t* out) {
  if (bm == nullptr || out == nullptr) return PA_ERR_INVALID_ARG;
  const int64_t bs = bm->block_size;
  std::vector<int32_t> fill(static_cast<size_t>(bm->num_blocks), 0);  // max tokens per block
  pa_bm_stats_t st = {};
  st.num_blocks = bm->num_blocks;
  st.free_blocks = static_cast<int64_t>(bm->free_list.size());
  st.num_seqs = static_cast<int64_t>(bm->seqs.size());
  for (const auto& kv : bm->seqs) {
    const pa_block_manager::Seq& s = kv.second;
    const int64_t nb = static_cast<int64_t>(s.table.size());
    st.logical_blocks += nb;
    st.tokens += s.tokens;
    st.max_waste_per_seq = std::max(st.max_waste_per_seq, nb * bs - s.tokens);
    for (int64_t i = 0; i < nb; ++i) {
      const int32_t f = static_cast<int32_t>(std::min<int64_t>(bs, s.tokens - i * bs));
      int32_t& m = fill[static_cast<size_t>(s.table[static_cast<size_t>(i)])];
      m = std::max(m, f);
    }
  }
  for (int32_t b = 0; b < bm->num_blocks; ++b) {
    if (bm->refcount[b] > 0) {
      ++st.held_blocks;
      st.stored_slots += fill[static_cast<size_t>(b)];
    }
  }
  st.waste_slots = st.held_blocks * bs - st.stored_slots;
  st.cached_blocks = bm->num_cached;
  *out = st;
  return PA_OK;
}
