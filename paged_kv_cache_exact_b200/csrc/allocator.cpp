// Host-side page allocator for the paged KV cache (the bookkeeping half of
// PagedAttention; the kernels in kv_write.cu do the device writes).
//
// "FlashAttention and PagedAttention: Two Fixes for Two Different
// Bottlenecks", section "PagedAttention ... How it works": the cache is cut
// into fixed-size blocks; every sequence keeps a block table from logical
// block to physical block; blocks are allocated on demand, only when a
// sequence grows into one; sequences that share a prefix point at the same
// physical blocks and copy only when their contents diverge.  "Flash
// Attention: Fast, Memory-Efficient Attention for LLMs", section
// "PagedAttention (vLLM)": pages of finished sequences are freed and reused.
//
// Choices the pages leave open:
// * the free page handed out next is always the smallest free id (a fresh pool
//   gives consecutive requests consecutive pages, as the pages' example shows);
// * a physical page carries a reference count: sharing (fork) increments it,
//   freeing a sequence decrements it, the page returns to the pool at zero;
// * only a shared, partially filled last page is ever copied, right before the
//   sequence writes into it; full shared pages are read-only and stay shared.
//
// Not thread-safe: one allocator per scheduling thread.
#include <set>
#include <unordered_map>
#include <vector>

#include "../../include/pkv.h"

struct pkv_allocator {
  struct Seq {
    std::vector<int32_t> pages;
    int len = 0;
  };
  int num_pages, page_size, max_pages;
  std::vector<int> ref;
  std::set<int32_t> free_pages;
  std::unordered_map<int, Seq> seqs;

  pkv_allocator(int np, int ps, int mp) : num_pages(np), page_size(ps), max_pages(mp), ref(np, 0) {
    for (int i = 0; i < np; ++i) free_pages.insert(i);
  }
  int32_t take() {
    const int32_t p = *free_pages.begin();
    free_pages.erase(free_pages.begin());
    ref[p] = 1;
    return p;
  }
  void release(int32_t p) {
    if (--ref[p] == 0) free_pages.insert(p);
  }
};

extern "C" {

pkv_allocator* pkv_alloc_create(int num_pages, int page_size, int max_pages_per_seq) {
  if (num_pages < 1 || page_size < 1 || max_pages_per_seq < 1) return nullptr;
  try {
    return new pkv_allocator(num_pages, page_size, max_pages_per_seq);
  } catch (...) {
    return nullptr;
  }
}

void pkv_alloc_destroy(pkv_allocator* a) { delete a; }

int pkv_alloc_add_seq(pkv_allocator* a, int seq_id) {
  if (!a || a->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
  a->seqs.emplace(seq_id, pkv_allocator::Seq{});
  return PKV_OK;
}

int pkv_alloc_reserve(pkv_allocator* a, int seq_id, int n_tokens, int32_t* start_pos,
                      int32_t* cow_src, int32_t* cow_dst, int* n_cow) {
  if (!a || n_tokens < 0 || !start_pos || !cow_src || !cow_dst || !n_cow) return PKV_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
  pkv_allocator::Seq& s = it->second;
  const long long new_len = (long long)s.len + n_tokens;
  const long long need = (new_len + a->page_size - 1) / a->page_size;
  if (need > a->max_pages) return PKV_ERR_INVALID_ARG;
  const bool cow = n_tokens > 0 && s.len % a->page_size != 0 && a->ref[s.pages.back()] > 1;
  const long long extra = need - (long long)s.pages.size() + (cow ? 1 : 0);
  if (extra > (long long)a->free_pages.size()) return PKV_ERR_OUT_OF_PAGES;   // nothing changed
  *start_pos = s.len;
  *n_cow = 0;
  if (cow) {
    const int32_t shared = s.pages.back();
    const int32_t fresh = a->take();
    a->release(shared);                                 // stays >= 1: others still hold it
    s.pages.back() = fresh;
    *cow_src = shared;
    *cow_dst = fresh;
    *n_cow = 1;
  }
  while ((long long)s.pages.size() < need) s.pages.push_back(a->take());
  s.len = (int)new_len;
  return PKV_OK;
}

int pkv_alloc_fork(pkv_allocator* a, int parent_id, int child_id) {
  if (!a || a->seqs.count(child_id)) return PKV_ERR_INVALID_ARG;
  auto it = a->seqs.find(parent_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
  pkv_allocator::Seq child = it->second;               // same pages, same length
  for (int32_t p : child.pages) ++a->ref[p];
  a->seqs.emplace(child_id, std::move(child));
  return PKV_OK;
}

int pkv_alloc_free_seq(pkv_allocator* a, int seq_id) {
  if (!a) return PKV_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
  for (int32_t p : it->second.pages) a->release(p);
  a->seqs.erase(it);
  return PKV_OK;
}

int pkv_alloc_seq_len(const pkv_allocator* a, int seq_id, int* len) {
  if (!a || !len) return PKV_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
  *len = it->second.len;
  return PKV_OK;
}

int pkv_alloc_block_table(const pkv_allocator* a, const int* seq_ids, int n, int32_t* table,
                          int32_t* seq_lens) {
  if (!a || n < 0 || (n > 0 && (!seq_ids || !table || !seq_lens))) return PKV_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (!a->seqs.count(seq_ids[i])) return PKV_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const pkv_allocator::Seq& s = a->seqs.at(seq_ids[i]);
    int32_t* row = table + (size_t)i * a->max_pages;
    for (int k = 0; k < a->max_pages; ++k) row[k] = k < (int)s.pages.size() ? s.pages[k] : -1;
    seq_lens[i] = s.len;
  }
  return PKV_OK;
}

int pkv_alloc_num_free(const pkv_allocator* a) {
  return a ? (int)a->free_pages.size() : -1;
}

int pkv_alloc_page_refs(const pkv_allocator* a, int page) {
  return (a && page >= 0 && page < a->num_pages) ? a->ref[page] : -1;
}

}  // extern "C"
