// pa_blockmgr.cpp -- host block manager that produces the metadata the
// kernels consume: block tables, slot mappings and copy-on-write pairs.
//
// Rules from "PagedAttention" (shubhamtatvamasi.com):
//  - "The idea: page the KV cache": a sequence gets a new physical block only
//    when its previous block is full (the OS analogy: a page is allocated when
//    first used), from a free list, from anywhere in memory;
//  - "Sharing and copy-on-write": tables may point at the same physical block;
//    each block keeps a reference count; a filled block is not written again;
//  - "How does copy-on-write work for parallel sampling?": a sequence that must
//    append into a shared, partially filled block allocates a new block, has
//    the old contents copied into it, decrements the old block's count and
//    writes into the copy.
// The copy itself is the device's job (pa_copy_blocks); this manager returns
// the (src, dst) pair.
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

  bool alloc(int32_t* out) {
    if (free_list.empty()) return false;
    *out = free_list.front();
    free_list.pop_front();
    refcount[*out] = 1;
    return true;
  }
  void release(int32_t blk) {
    if (--refcount[blk] == 0) free_list.push_back(blk);
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

extern "C" int32_t pa_bm_refcount(const pa_block_manager* bm, int32_t block) {
  if (bm == nullptr || block < 0 || block >= bm->num_blocks) return -1;
  return bm->refcount[block];
}

extern "C" int32_t pa_bm_num_free(const pa_block_manager* bm) {
  return bm == nullptr ? -1 : static_cast<int32_t>(bm->free_list.size());
}
