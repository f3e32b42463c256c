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
// Prefix caching ("5. Prefix Caching", hjr-study-book Day 3; "prefix caching"
// in "4. 이 밖의 기법들", blog.aqudi.me: the KV blocks of a prompt prefix that
// repeats across requests are reused).  The pages give no mechanism; this one
// keys every full block by its content chain -- (key of the previous block,
// the block's token ids) -- interned as nodes of a trie, so a lookup compares
// token ids exactly and no hash collision can alias two prefixes.  A request
// takes the cached blocks of its longest cached chain of full blocks, leaving
// at least one token to compute.  A cached block whose count drops to zero is
// not freed but becomes evictable (least recently released first); blocks are
// taken from the free stack first and only then by evicting, which drops the
// block's key.
//
// Storage: one flat refcount array, a free stack, and a hash map from sequence
// id to its block list; with prefix caching a trie of keys, the block of each
// key, and an LRU list of evictable blocks.  Every operation is O(blocks
// touched).
#include <cstdint>
#include <cstring>
#include <functional>
#include <list>
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
  struct Key {  // a full block's content chain: parent node (-1 = none), token ids
    int64_t parent;
    std::vector<int32_t> tokens;
    bool operator==(const Key& o) const { return parent == o.parent && tokens == o.tokens; }
  };
  struct KeyHash {
    size_t operator()(const Key& k) const {
      uint64_t h = 1469598103934665603ull ^ static_cast<uint64_t>(k.parent);
      for (int32_t t : k.tokens) h = (h ^ static_cast<uint32_t>(t)) * 1099511628211ull;
      return static_cast<size_t>(h);
    }
  };
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // back() is handed out next
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Seq> seqs;
  // prefix cache
  bool prefix = false;
  std::unordered_map<Key, int64_t, KeyHash> nodes;  // content chain -> node id
  std::vector<int32_t> node_block;                  // node -> cached block or -1
  std::vector<int64_t> block_node;                  // block -> node or -1
  std::list<int32_t> evictable;                     // front is evicted first
  std::vector<std::list<int32_t>::iterator> evict_pos;

  size_t available() const { return free_stack.size() + evictable.size(); }

  int32_t pop() {
    int32_t b;
    if (!free_stack.empty()) {
      b = free_stack.back();
      free_stack.pop_back();
    } else {  // evict the least recently released cached block
      b = evictable.front();
      evictable.pop_front();
      node_block[block_node[b]] = -1;
      block_node[b] = -1;
    }
    refcount[b] = 1;
    return b;
  }

  // one reference fewer; at zero the block is freed, or kept evictable if cached
  void unref(int32_t b) {
    if (--refcount[b] != 0) return;
    if (prefix && block_node[b] >= 0) {
      evictable.push_back(b);
      evict_pos[b] = std::prev(evictable.end());
    } else {
      free_stack.push_back(b);
    }
  }

  // one reference more to a cached block (taken back from the evictable list at zero)
  void ref_cached(int32_t b) {
    if (refcount[b] == 0) evictable.erase(evict_pos[b]);
    refcount[b] += 1;
  }

  int64_t find_node(int64_t parent, const int32_t* tokens) const {
    Key k{parent, std::vector<int32_t>(tokens, tokens + block_size)};
    auto it = nodes.find(k);
    return it == nodes.end() ? -1 : it->second;
  }

  int64_t intern(int64_t parent, const int32_t* tokens) {
    Key k{parent, std::vector<int32_t>(tokens, tokens + block_size)};
    auto it = nodes.find(k);
    if (it != nodes.end()) return it->second;
    const int64_t id = static_cast<int64_t>(node_block.size());
    nodes.emplace(std::move(k), id);
    node_block.push_back(-1);
    return id;
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
  return a ? static_cast<int>(a->available()) : -1;
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

extern "C" pa_status pa_alloc_enable_prefix_cache(pa_allocator* a) {
  if (!a) return pa::fail(PA_ERR_INVALID, "pa_alloc_enable_prefix_cache: NULL handle");
  if (!a->prefix) {
    a->prefix = true;
    a->block_node.assign(a->num_blocks, -1);
    a->evict_pos.resize(a->num_blocks);
  }
  return PA_OK;
}

extern "C" pa_status pa_alloc_evictable(const pa_allocator* a, int32_t* out, int capacity,
                                        int* n_out) {
  if (!a || !n_out || capacity < 0 || (capacity > 0 && !out))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_evictable: bad argument");
  const int n = static_cast<int>(a->evictable.size());
  *n_out = n;
  int i = 0;
  for (auto it = a->evictable.begin(); it != a->evictable.end() && i < capacity; ++it) out[i++] = *it;
  return PA_OK;
}

extern "C" pa_status pa_seq_add_cached(pa_allocator* a, int64_t seq_id, const int32_t* token_ids,
                                       int num_tokens, int* num_cached) {
  const char* fn = "pa_seq_add_cached";
  if (!a || !num_cached || num_tokens < 0 || (num_tokens > 0 && !token_ids))
    return pa::fail(PA_ERR_INVALID, "%s: bad argument", fn);
  if (a->seqs.count(seq_id))
    return pa::fail(PA_ERR_INVALID, "%s: sequence %lld exists", fn, (long long)seq_id);
  pa_allocator::Seq s;
  if (a->prefix && num_tokens > 0) {
    const int bs = a->block_size;
    const int full = (num_tokens - 1) / bs;  // leave at least one token to compute
    int64_t parent = -1;
    for (int k = 0; k < full; ++k) {
      const int64_t node = a->find_node(parent, token_ids + static_cast<int64_t>(k) * bs);
      if (node < 0 || a->node_block[node] < 0) break;
      const int32_t b = a->node_block[node];
      a->ref_cached(b);
      s.blocks.push_back(b);
      parent = node;
    }
    s.tokens = static_cast<int64_t>(s.blocks.size()) * bs;
  }
  *num_cached = static_cast<int>(s.tokens);
  a->seqs.emplace(seq_id, std::move(s));
  return PA_OK;
}

extern "C" pa_status pa_seq_commit(pa_allocator* a, int64_t seq_id, const int32_t* token_ids,
                                   int num_tokens) {
  const char* fn = "pa_seq_commit";
  if (!a || num_tokens < 0 || (num_tokens > 0 && !token_ids))
    return pa::fail(PA_ERR_INVALID, "%s: bad argument", fn);
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end())
    return pa::fail(PA_ERR_INVALID, "%s: unknown sequence %lld", fn, (long long)seq_id);
  if (num_tokens > it->second.tokens)
    return pa::fail(PA_ERR_INVALID, "%s: %d tokens given, the sequence holds %lld", fn,
                    num_tokens, (long long)it->second.tokens);
  if (!a->prefix) return PA_OK;
  const int bs = a->block_size;
  int64_t parent = -1;
  for (int k = 0; k < num_tokens / bs; ++k) {
    const int64_t node = a->intern(parent, token_ids + static_cast<int64_t>(k) * bs);
    const int32_t b = it->second.blocks[k];
    // first writer wins: a key keeps its block, a block keeps its key
    if (a->node_block[node] < 0 && a->block_node[b] < 0) {
      a->node_block[node] = b;
      a->block_node[b] = node;
    }
    parent = node;
  }
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
  if (need > static_cast<int64_t>(a->available()))
    return pa::fail(PA_ERR_OOM, "pa_seq_append: need %lld blocks, %zu free", (long long)need,
                    a->available());
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
  for (int32_t b : it->second.blocks) a->unref(b);
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
  if (distinct > static_cast<int64_t>(dst->available()))
    return pa::fail(PA_ERR_OOM, "%s: need %lld blocks, %zu free", fn, (long long)distinct,
                    dst->available());
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

extern "C" pa_status pa_build_groups(const int32_t* block_tables, int num_seqs,
                                     int max_blocks_per_seq, const int32_t* context_lens,
                                     int block_size, int32_t* group_start_out,
                                     int32_t* shared_lens_out, int* num_groups_out,
                                     int* max_group_size_out, int* max_shared_len_out) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || !group_start_out ||
      !num_groups_out || !max_group_size_out || !max_shared_len_out ||
      (num_seqs > 0 && (!block_tables || !context_lens || !shared_lens_out)))
    return pa::fail(PA_ERR_INVALID, "pa_build_groups: bad argument");
  for (int b = 0; b < num_seqs; ++b)
    if (context_lens[b] < 0 ||
        static_cast<int64_t>(context_lens[b]) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
      return pa::fail(PA_ERR_INVALID, "pa_build_groups: context length %d of sequence %d out of range",
                      context_lens[b], b);
  auto row = [&](int b) { return block_tables + static_cast<int64_t>(b) * max_blocks_per_seq; };
  // whole blocks of sequence b that hold only its tokens' slots it uses
  auto full_blocks = [&](int b) { return context_lens[b] / block_size; };
  int ng = 0, max_size = 0, max_shared = 0;
  int b0 = 0;
  while (b0 < num_seqs) {
    // members: the following sequences whose first block is b0's first block
    int b1 = b0 + 1;
    if (full_blocks(b0) > 0)
      while (b1 < num_seqs && full_blocks(b1) > 0 && row(b1)[0] == row(b0)[0]) ++b1;
    // the leading entries every member has in common, within every member's
    // whole blocks
    int k = full_blocks(b0);
    for (int m = b0 + 1; m < b1; ++m) {
      int c = 0;
      const int lim = k < full_blocks(m) ? k : full_blocks(m);
      while (c < lim && row(m)[c] == row(b0)[c]) ++c;
      k = c;
    }
    const int shared = b1 - b0 > 1 ? k * block_size : 0;
    group_start_out[ng++] = b0;
    for (int m = b0; m < b1; ++m) shared_lens_out[m] = shared;
    max_size = max_size > b1 - b0 ? max_size : b1 - b0;
    max_shared = max_shared > shared ? max_shared : shared;
    b0 = b1;
  }
  group_start_out[ng] = num_seqs;
  *num_groups_out = ng;
  *max_group_size_out = max_size;
  *max_shared_len_out = max_shared;
  return PA_OK;
}
