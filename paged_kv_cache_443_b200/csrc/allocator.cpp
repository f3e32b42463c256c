// allocator.cpp -- host block manager behind pa_alloc_* / pa_seq_* / pa_build_tables.
//
// Follows "PagedAttention의 설계" and "블록 공유" of the supersilo.blog vLLM summary
// (the block manager hands out fixed-size blocks as a request grows, reclaims
// them, and lets samples of one prompt share blocks) and section 3 of the
// blog.aqudi.me write-up (a new block only when the current one is full;
// copy-on-write of shared blocks).  Conventions the pages leave open: a LIFO
// free stack; freeing in logical order; the copy-on-write block is taken
// before new blocks; all-or-nothing on OOM.
//
// Moving sequences between two managers (swap to host memory and back,
// "적용 범위와 관련 연구" of the supersilo.blog summary) keeps the sharing among
// the sequences moved together: a source block gets one destination block the
// first time it is met (sequences in caller order, blocks in logical order),
// and every later holder shares it.
//
// Storage: one flat refcount array, a free stack, and a hash map from sequence
// id to its block list.  Every operation is O(blocks touched).
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"
#include "pa_internal.h"

struct pa_allocator {
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t tokens = 0;
  };
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // back() is handed out next
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Seq> seqs;

  int32_t pop() {
    int32_t b = free_stack.back();
    free_stack.pop_back();
    refcount[b] = 1;
    return b;
  }
};

extern "C" pa_status pa_alloc_create(int num_blocks, int block_size,
                                     const int32_t* initial_free_order, pa_allocator** out) {
  if (!out) return pa::fail(PA_ERR_INVALID, "pa_alloc_create: out is NULL");
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0)
    return pa::fail(PA_ERR_INVALID, "pa_alloc_create: num_blocks and block_size must be > 0");
  pa_allocator* a = new (std::nothrow) pa_allocator();
  if (!a) return pa::fail(PA_ERR_OOM, "pa_alloc_create: host allocation failed");
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->refcount.assign(num_blocks, 0);
  a->free_stack.resize(num_blocks);
  if (initial_free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return pa::fail(PA_ERR_INVALID,
                        "pa_alloc_create: initial_free_order is not a permutation of 0..num_blocks-1");
      }
      seen[b] = 1;
      a->free_stack[i] = b;
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) a->free_stack[i] = num_blocks - 1 - i;
  }
  *out = a;
  return PA_OK;
}

extern "C" void pa_alloc_destroy(pa_allocator* a) { delete a; }

extern "C" int pa_alloc_num_free(const pa_allocator* a) {
  return a ? static_cast<int>(a->free_stack.size()) : -1;
}

extern "C" int pa_alloc_refcount(const pa_allocator* a, int32_t block) {
  if (!a || block < 0 || block >= a->num_blocks) return -1;
  return a->refcount[block];
}

extern "C" pa_status pa_alloc_free_stack(const pa_allocator* a, int32_t* out, int capacity,
                                         int* n_out) {
  if (!a || !n_out || capacity < 0 || (capacity > 0 && !out))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_free_stack: bad argument");
  const int n = static_cast<int>(a->free_stack.size());
  *n_out = n;
  const int m = n < capacity ? n : capacity;
  if (m > 0) std::memcpy(out, a->free_stack.data(), sizeof(int32_t) * m);
  return PA_OK;
}

extern "C" pa_status pa_seq_add(pa_allocator* a, int64_t seq_id) {
  if (!a) return pa::fail(PA_ERR_INVALID, "pa_seq_add: NULL handle");
  if (!a->seqs.emplace(seq_id, pa_allocator::Seq{}).second)
    return pa::fail(PA_ERR_INVALID, "pa_seq_add: sequence %lld exists", (long long)seq_id);
  return PA_OK;
}

extern "C" pa_status pa_seq_fork(pa_allocator* a, int64_t parent, int64_t child) {
  if (!a) return pa::fail(PA_ERR_INVALID, "pa_seq_fork: NULL handle");
  auto p = a->seqs.find(parent);
  if (p == a->seqs.end())
    return pa::fail(PA_ERR_INVALID, "pa_seq_fork: unknown parent %lld", (long long)parent);
  if (a->seqs.count(child))
    return pa::fail(PA_ERR_INVALID, "pa_seq_fork: child %lld exists", (long long)child);
  pa_allocator::Seq c = p->second;  // copy before emplace may rehash
  for (int32_t b : c.blocks) a->refcount[b] += 1;
  a->seqs.emplace(child, std::move(c));
  return PA_OK;
}

extern "C" pa_status pa_seq_append(pa_allocator* a, int64_t seq_id, int n_tokens,
                                   int64_t* slots_out, int64_t* cow_pair_out, int* n_cow) {
  if (!a) return pa::fail(PA_ERR_INVALID, "pa_seq_append: NULL handle");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_INVALID, "pa_seq_append: unknown sequence %lld", (long long)seq_id);
  if (n_tokens < 0) return pa::fail(PA_ERR_INVALID, "pa_seq_append: n_tokens < 0");
  if (n_tokens > 0 && !slots_out) return pa::fail(PA_ERR_INVALID, "pa_seq_append: slots_out NULL");
  if (!n_cow || !cow_pair_out)
    return pa::fail(PA_ERR_INVALID, "pa_seq_append: cow_pair_out / n_cow NULL");
  *n_cow = 0;
  if (n_tokens == 0) return PA_OK;
  pa_allocator::Seq& s = it->second;
  const int64_t bs = a->block_size;
  const int64_t have = static_cast<int64_t>(s.blocks.size());
  const int64_t want = (s.tokens + n_tokens + bs - 1) / bs;
  const bool tail_partial = (s.tokens % bs) != 0;
  const bool cow = tail_partial && a->refcount[s.blocks.back()] > 1;
  const int64_t need = (want - have) + (cow ? 1 : 0);
  if (need > static_cast<int64_t>(a->free_stack.size()))
    return pa::fail(PA_ERR_OOM, "pa_seq_append: need %lld blocks, %zu free", (long long)need,
                    a->free_stack.size());
  if (cow) {
    const int32_t old = s.blocks.back();
    const int32_t fresh = a->pop();
    a->refcount[old] -= 1;
    s.blocks.back() = fresh;
    cow_pair_out[0] = old;
    cow_pair_out[1] = fresh;
    *n_cow = 1;
  }
  for (int64_t i = have; i < want; ++i) s.blocks.push_back(a->pop());
  for (int64_t t = 0; t < n_tokens; ++t) {
    const int64_t pos = s.tokens + t;
    slots_out[t] = static_cast<int64_t>(s.blocks[pos / bs]) * bs + pos % bs;
  }
  s.tokens += n_tokens;
  return PA_OK;
}

extern "C" pa_status pa_seq_free(pa_allocator* a, int64_t seq_id) {
  if (!a) return pa::fail(PA_ERR_INVALID, "pa_seq_free: NULL handle");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_INVALID, "pa_seq_free: unknown sequence %lld", (long long)seq_id);
  for (int32_t b : it->second.blocks) {
    if (--a->refcount[b] == 0) a->free_stack.push_back(b);
  }
  a->seqs.erase(it);
  return PA_OK;
}

extern "C" pa_status pa_seq_move(pa_allocator* src, pa_allocator* dst, const int64_t* seq_ids,
                                 int num_seqs, int64_t* pairs_out, int pairs_capacity,
                                 int* n_pairs) {
  const char* fn = "pa_seq_move";
  if (!src || !dst || !n_pairs || num_seqs < 0 || pairs_capacity < 0 ||
      (num_seqs > 0 && !seq_ids))
    return pa::fail(PA_ERR_INVALID, "%s: bad argument", fn);
  if (src == dst) return pa::fail(PA_ERR_INVALID, "%s: source and destination are the same", fn);
  if (src->block_size != dst->block_size)
    return pa::fail(PA_ERR_INVALID, "%s: block sizes differ (%d vs %d)", fn, src->block_size,
                    dst->block_size);
  *n_pairs = 0;
  // validate and count distinct blocks first: a failure changes nothing
  std::unordered_map<int64_t, char> ids;
  std::unordered_map<int32_t, int32_t> map;
  int64_t distinct = 0;
  for (int i = 0; i < num_seqs; ++i) {
    auto it = src->seqs.find(seq_ids[i]);
    if (it == src->seqs.end())
      return pa::fail(PA_ERR_INVALID, "%s: unknown sequence %lld", fn, (long long)seq_ids[i]);
    if (dst->seqs.count(seq_ids[i]))
      return pa::fail(PA_ERR_INVALID, "%s: sequence %lld exists in the destination", fn,
                      (long long)seq_ids[i]);
    if (!ids.emplace(seq_ids[i], 1).second)
      return pa::fail(PA_ERR_INVALID, "%s: sequence %lld listed twice", fn, (long long)seq_ids[i]);
    for (int32_t b : it->second.blocks)
      if (map.emplace(b, -1).second) ++distinct;
  }
  if (distinct > static_cast<int64_t>(dst->free_stack.size()))
    return pa::fail(PA_ERR_OOM, "%s: need %lld blocks, %zu free", fn, (long long)distinct,
                    dst->free_stack.size());
  if (distinct > pairs_capacity || (distinct > 0 && !pairs_out))
    return pa::fail(PA_ERR_INVALID, "%s: pairs_out holds %d pairs, %lld needed", fn,
                    pairs_capacity, (long long)distinct);
  int64_t np = 0;
  for (int i = 0; i < num_seqs; ++i) {
    const pa_allocator::Seq& s = src->seqs.find(seq_ids[i])->second;
    pa_allocator::Seq d;
    d.tokens = s.tokens;
    d.blocks.reserve(s.blocks.size());
    for (int32_t b : s.blocks) {
      int32_t& m = map[b];
      if (m < 0) {
        m = dst->pop();
        pairs_out[2 * np] = b;
        pairs_out[2 * np + 1] = m;
        ++np;
      } else {
        dst->refcount[m] += 1;
      }
      d.blocks.push_back(m);
    }
    dst->seqs.emplace(seq_ids[i], std::move(d));
  }
  for (int i = 0; i < num_seqs; ++i) pa_seq_free(src, seq_ids[i]);
  *n_pairs = static_cast<int>(np);
  return PA_OK;
}

extern "C" pa_status pa_seq_num_tokens(const pa_allocator* a, int64_t seq_id, int* out) {
  if (!a || !out) return pa::fail(PA_ERR_INVALID, "pa_seq_num_tokens: bad argument");
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_INVALID, "pa_seq_num_tokens: unknown sequence %lld", (long long)seq_id);
  *out = static_cast<int>(it->second.tokens);
  return PA_OK;
}

extern "C" pa_status pa_build_tables(const pa_allocator* a, const int64_t* seq_ids, int num_seqs,
                                     int max_blocks_per_seq, int32_t* block_tables_out,
                                     int32_t* context_lens_out) {
  if (!a || num_seqs < 0 || max_blocks_per_seq <= 0 ||
      (num_seqs > 0 && (!seq_ids || !block_tables_out || !context_lens_out)))
    return pa::fail(PA_ERR_INVALID, "pa_build_tables: bad argument");
  // validate everything first so a failure writes nothing
  for (int b = 0; b < num_seqs; ++b) {
    auto it = a->seqs.find(seq_ids[b]);
    if (it == a->seqs.end())
      return pa::fail(PA_ERR_INVALID, "pa_build_tables: unknown sequence %lld",
                      (long long)seq_ids[b]);
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks_per_seq)
      return pa::fail(PA_ERR_INVALID, "pa_build_tables: sequence %lld has %zu blocks > %d",
                      (long long)seq_ids[b], it->second.blocks.size(), max_blocks_per_seq);
  }
  for (int b = 0; b < num_seqs; ++b) {
    const auto& s = a->seqs.find(seq_ids[b])->second;
    int32_t* row = block_tables_out + static_cast<int64_t>(b) * max_blocks_per_seq;
    const int n = static_cast<int>(s.blocks.size());
    for (int i = 0; i < n; ++i) row[i] = s.blocks[i];
    for (int i = n; i < max_blocks_per_seq; ++i) row[i] = -1;
    context_lens_out[b] = static_cast<int32_t>(s.tokens);
  }
  return PA_OK;
}
