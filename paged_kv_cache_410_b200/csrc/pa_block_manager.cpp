// Host-side KV block manager (include/pa_block_manager.h): a free list of
// physical blocks, per-block reference counts, on-demand allocation,
// copy-on-write after forks, and a block-granular radix tree of token ids
// for prefix reuse with least-recently-used eviction.
#include "pa_block_manager.h"

#include <cstdint>
#include <cstring>
#include <memory>
#include <new>
#include <set>
#include <algorithm>
#include <unordered_map>
#include <utility>
#include <vector>

namespace {

// One cached full block: an edge of the radix tree labelled by the block's
// block_size token ids, under the node of the block before it.
struct Node {
  int64_t block = -1;
  std::vector<int32_t> tokens;
  Node* parent = nullptr;
  std::unordered_multimap<uint64_t, Node*> children;  // keyed by a hash of the tokens
  uint64_t last_use = 0;
};

struct Seq {
  std::vector<int64_t> blocks;   // physical block of each logical block
  std::vector<int32_t> tokens;   // token ids, for caching full blocks
  int32_t length = 0;
  int32_t released = 0;          // leading blocks already released (sliding window)
  Node* tail = nullptr;          // tree node of the last leading block known to the cache
  int32_t tail_blocks = 0;       // leading blocks covered by the path ending at `tail`
  uint64_t version = 0;          // stamp of the last change to `blocks` (never 0)
  uint64_t batch = 0;            // last batched call that listed this sequence
};

uint64_t hash_tokens(const int32_t* t, int32_t n) {
  uint64_t h = 1469598103934665603ull;  // FNV-1a
  for (int32_t i = 0; i < n; ++i) {
    uint32_t v = static_cast<uint32_t>(t[i]);
    for (int k = 0; k < 4; ++k) {
      h ^= (v >> (8 * k)) & 0xffu;
      h *= 1099511628211ull;
    }
  }
  return h;
}

}  // namespace

struct pa_block_manager {
  int64_t num_blocks = 0;
  int32_t bs = 0;
  bool prefix_cache = false;
  std::vector<int32_t> refcount;
  std::vector<int64_t> free_list;
  std::unordered_map<int64_t, Seq> seqs;
  Node root;
  std::unordered_map<int64_t, std::unique_ptr<Node>> nodes;  // cached block -> node
  std::set<std::pair<uint64_t, int64_t>> evictable;           // (last_use, block)
  uint64_t tick = 0;
  uint64_t versions = 0;  // last stamp handed out; stamps are unique across sequences
  uint64_t batches = 0;   // batched calls so far (duplicate ids within one are refused)

  void changed(Seq& s) { s.version = ++versions; }

  bool is_evictable(const Node* n) const {
    return n->block >= 0 && refcount[n->block] == 1 && n->children.empty();
  }
  void track(Node* n) {  // keep `evictable` in step with a node's state
    if (n == &root || !n) return;
    const auto key = std::make_pair(n->last_use, n->block);
    if (is_evictable(n))
      evictable.insert(key);
    else
      evictable.erase(key);
  }
  void touch(Node* n) {
    if (n == &root || !n) return;
    evictable.erase(std::make_pair(n->last_use, n->block));
    n->last_use = ++tick;
    track(n);
  }

  // Drop the least recently used cached block that nobody else holds.
  bool evict_one() {
    if (evictable.empty()) return false;
    const int64_t blk = evictable.begin()->second;
    evictable.erase(evictable.begin());
    auto it = nodes.find(blk);
    Node* n = it->second.get();
    Node* parent = n->parent;
    auto range = parent->children.equal_range(hash_tokens(n->tokens.data(), bs));
    for (auto c = range.first; c != range.second; ++c)
      if (c->second == n) {
        parent->children.erase(c);
        break;
      }
    // sequences whose cached path ends at this node stop extending it
    for (auto& kv : seqs)
      if (kv.second.tail == n) kv.second.tail = nullptr;
    nodes.erase(it);
    refcount[blk] = 0;
    free_list.push_back(blk);
    track(parent);
    return true;
  }

  // Whether `need` blocks can be had from the free list plus evictions,
  // without evicting anything: a cached block is reclaimable when it and every
  // block below it in the tree is held by the cache alone (eviction takes
  // leaves first, so exactly those subtrees can go).
  bool can_reclaim(int64_t need) const {
    int64_t have = static_cast<int64_t>(free_list.size());
    if (have >= need) return true;
    std::vector<const Node*> order;  // pre-order: parents before children
    std::vector<const Node*> stack{&root};
    while (!stack.empty()) {
      const Node* n = stack.back();
      stack.pop_back();
      order.push_back(n);
      for (const auto& c : n->children) stack.push_back(c.second);
    }
    std::unordered_map<const Node*, bool> clean;
    for (auto it = order.rbegin(); it != order.rend(); ++it) {
      const Node* n = *it;
      if (n == &root) break;
      bool ok = refcount[n->block] == 1;
      for (const auto& c : n->children) ok = ok && clean[c.second];
      clean[n] = ok;
      if (ok && ++have >= need) return true;
    }
    return false;
  }

  int64_t alloc() {
    if (free_list.empty() && !evict_one()) return -1;
    const int64_t b = free_list.back();
    free_list.pop_back();
    refcount[b] = 1;
    return b;
  }

  void unref(int64_t b) {
    if (--refcount[b] == 0) {
      free_list.push_back(b);
      return;
    }
    auto it = nodes.find(b);
    if (it != nodes.end()) track(it->second.get());
  }

  void ref(int64_t b) {
    ++refcount[b];
    auto it = nodes.find(b);
    if (it != nodes.end()) track(it->second.get());
  }

  // The block the next token of `s` goes to: a new block at a block
  // boundary, a private copy of a shared partial last block (copy on write:
  // *cow_src / *cow_dst receive the pair), else the last block as it is.
  // Fails (changing nothing) only if a block is needed and none can be had.
  int32_t take_block(Seq& s, int32_t* cow_src, int32_t* cow_dst) {
    *cow_src = *cow_dst = -1;
    if (s.length % bs == 0) {
      const int64_t b = alloc();
      if (b < 0) return PA_BM_ERR_NO_BLOCKS;
      s.blocks.push_back(b);
      changed(s);
    } else {
      const int64_t last = s.blocks.back();
      if (refcount[last] > 1) {  // shared partial block: copy on write
        const int64_t b = alloc();
        if (b < 0) return PA_BM_ERR_NO_BLOCKS;
        *cow_src = static_cast<int32_t>(last);
        *cow_dst = static_cast<int32_t>(b);
        unref(last);
        s.blocks.back() = b;
        changed(s);
      }
    }
    return PA_BM_OK;
  }

  // Records the token taken by take_block: its slot, its id, and the block
  // it fills joins the prefix cache.
  void commit_token(Seq& s, int32_t token, int64_t* slot) {
    const int32_t pos = s.length;
    *slot = s.blocks[pos / bs] * bs + pos % bs;
    s.tokens.push_back(token);
    s.length = pos + 1;
    if (s.length % bs == 0) cache_full_block(s, s.length / bs - 1);
  }

  // Blocks that one append to each of `rows` (distinct sequences, in this
  // order) takes: one at each block boundary, one for each copy on write.
  // A sequence that copies drops its share of the old block, so a later row
  // that shared it with only that sequence writes in place.
  int64_t blocks_for_appends(const std::vector<Seq*>& rows) const {
    std::unordered_map<int64_t, int32_t> dropped;
    int64_t need = 0;
    for (const Seq* r : rows) {
      if (r->length % bs == 0) {
        ++need;
        continue;
      }
      const int64_t last = r->blocks.back();
      if (refcount[last] == 1) continue;  // private: written in place
      int32_t& d = dropped[last];
      if (refcount[last] - d > 1) {
        ++need;
        ++d;
      }
    }
    return need;
  }

  // Block `index` of `s` is full: extend the cached path with it.
  void cache_full_block(Seq& s, int32_t index) {
    if (!prefix_cache || s.tail_blocks != index) return;
    Node* parent = s.tail ? s.tail : &root;
    if (index > 0 && !s.tail) return;  // the path was cut by an eviction
    const int32_t* tok = s.tokens.data() + static_cast<size_t>(index) * bs;
    const uint64_t h = hash_tokens(tok, bs);
    auto range = parent->children.equal_range(h);
    for (auto c = range.first; c != range.second; ++c)
      if (std::memcmp(c->second->tokens.data(), tok, sizeof(int32_t) * bs) == 0) {
        s.tail = c->second;  // same content already cached (in another block)
        s.tail_blocks = index + 1;
        touch(c->second);
        return;
      }
    const int64_t blk = s.blocks[index];
    if (nodes.count(blk)) return;  // this block already labels another path
    auto node = std::make_unique<Node>();
    node->block = blk;
    node->tokens.assign(tok, tok + bs);
    node->parent = parent;
    node->last_use = ++tick;
    Node* raw = node.get();
    parent->children.emplace(h, raw);
    nodes.emplace(blk, std::move(node));
    ++refcount[blk];  // the cache's own reference
    track(parent);
    track(raw);
    s.tail = raw;
    s.tail_blocks = index + 1;
  }
};

extern "C" {

pa_block_manager* pa_bm_create(int64_t num_blocks, int32_t block_size, int32_t prefix_cache) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  auto* bm = new (std::nothrow) pa_block_manager();
  if (!bm) return nullptr;
  try {
    bm->num_blocks = num_blocks;
    bm->bs = block_size;
    bm->prefix_cache = prefix_cache != 0;
    bm->refcount.assign(static_cast<size_t>(num_blocks), 0);
    bm->free_list.reserve(static_cast<size_t>(num_blocks));
    for (int64_t b = num_blocks - 1; b >= 0; --b) bm->free_list.push_back(b);  // pop 0 first
  } catch (...) {
    delete bm;
    return nullptr;
  }
  return bm;
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

int64_t pa_bm_num_free_blocks(const pa_block_manager* bm) {
  return bm ? static_cast<int64_t>(bm->free_list.size()) : -1;
}

int64_t pa_bm_num_cached_blocks(const pa_block_manager* bm) {
  if (!bm) return -1;
  int64_t n = 0;  // cached blocks no sequence uses (leaves are evicted first)
  for (const auto& kv : bm->nodes) n += bm->refcount[kv.first] == 1;
  return n;
}

int32_t pa_bm_block_refcount(const pa_block_manager* bm, int64_t block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->refcount[block];
}

int32_t pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* tokens,
                           int32_t n_tokens, int32_t* cached_tokens) {
  if (!bm || n_tokens < 0 || (n_tokens > 0 && !tokens) || bm->seqs.count(seq_id))
    return PA_BM_ERR_INVALID;
  const int32_t bs = bm->bs;
  Seq s;
  s.tokens.assign(tokens, tokens + n_tokens);
  // 1. reuse the longest cached run of leading full blocks
  Node* node = &bm->root;
  std::vector<Node*> matched;
  if (bm->prefix_cache) {
    for (int32_t i = 0; (i + 1) * bs <= n_tokens; ++i) {
      const int32_t* tok = tokens + static_cast<size_t>(i) * bs;
      Node* next = nullptr;
      auto range = node->children.equal_range(hash_tokens(tok, bs));
      for (auto c = range.first; c != range.second; ++c)
        if (std::memcmp(c->second->tokens.data(), tok, sizeof(int32_t) * bs) == 0) {
          next = c->second;
          break;
        }
      if (!next) break;
      matched.push_back(next);
      node = next;
    }
  }
  for (Node* m : matched) bm->ref(m->block);
  // 2. fail before anything changes if the rest cannot be allocated (a
  // reference taken and dropped leaves a node exactly as it was)
  const int32_t need = (n_tokens + bs - 1) / bs;
  if (!bm->can_reclaim(need - static_cast<int64_t>(matched.size()))) {
    for (Node* m : matched) bm->unref(m->block);
    return PA_BM_ERR_NO_BLOCKS;
  }
  for (Node* m : matched) {
    s.blocks.push_back(m->block);
    bm->touch(m);
  }
  s.tail = matched.empty() ? nullptr : matched.back();
  s.tail_blocks = static_cast<int32_t>(matched.size());
  // 3. private blocks for the rest
  for (int32_t i = static_cast<int32_t>(matched.size()); i < need; ++i) {
    const int64_t b = bm->alloc();
    if (b < 0) {  // roll back (not reached after the check above)
      for (size_t k = 0; k < s.blocks.size(); ++k) bm->unref(s.blocks[k]);
      return PA_BM_ERR_NO_BLOCKS;
    }
    s.blocks.push_back(b);
  }
  s.length = n_tokens;
  bm->changed(s);
  if (cached_tokens) *cached_tokens = static_cast<int32_t>(matched.size()) * bs;
  auto& ins = bm->seqs.emplace(seq_id, std::move(s)).first->second;
  // 4. the prompt's full blocks join the cache as soon as they exist
  for (int32_t i = ins.tail_blocks; (i + 1) * bs <= n_tokens; ++i) bm->cache_full_block(ins, i);
  return PA_BM_OK;
}

int32_t pa_bm_append_token(pa_block_manager* bm, int64_t seq_id, int32_t token, int64_t* slot,
                           int32_t* cow_src, int32_t* cow_dst) {
  if (!bm || !slot) return PA_BM_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_BM_ERR_INVALID;
  int32_t src = -1, dst = -1;
  const int32_t rc = bm->take_block(it->second, &src, &dst);
  if (rc != PA_BM_OK) return rc;
  bm->commit_token(it->second, token, slot);
  if (cow_src) *cow_src = src;
  if (cow_dst) *cow_dst = dst;
  return PA_BM_OK;
}

int32_t pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seq_ids, const int32_t* tokens,
                            int32_t n, int64_t* slots, int32_t* cow_pairs, int32_t* num_pairs) {
  if (!bm || n < 0 || !num_pairs || (n > 0 && (!seq_ids || !tokens || !slots || !cow_pairs)))
    return PA_BM_ERR_INVALID;
  // every id known and distinct, and every block the batch needs obtainable,
  // before anything changes
  std::vector<Seq*> rows(static_cast<size_t>(n));
  const uint64_t mark = ++bm->batches;
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || it->second.batch == mark) return PA_BM_ERR_INVALID;
    it->second.batch = mark;
    rows[static_cast<size_t>(i)] = &it->second;
  }
  if (!bm->can_reclaim(bm->blocks_for_appends(rows))) return PA_BM_ERR_NO_BLOCKS;
  // First every row's block, then the tokens: caching a block a row fills
  // can pin a released block that only the cache held (it becomes a parent),
  // which the count above took as reclaimable, so no row may fill the cache
  // before every block of the batch is taken.
  int32_t pairs = 0;
  for (int32_t i = 0; i < n; ++i) {
    int32_t src = -1, dst = -1;
    if (bm->take_block(*rows[static_cast<size_t>(i)], &src, &dst) != PA_BM_OK)
      return PA_BM_ERR_NO_BLOCKS;  // not reached: the blocks were counted above
    if (src >= 0) {
      cow_pairs[2 * pairs] = src;
      cow_pairs[2 * pairs + 1] = dst;
      ++pairs;
    }
  }
  for (int32_t i = 0; i < n; ++i)
    bm->commit_token(*rows[static_cast<size_t>(i)], tokens[i], &slots[i]);
  *num_pairs = pairs;
  return PA_BM_OK;
}

int32_t pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id) {
  if (!bm || bm->seqs.count(child_id)) return PA_BM_ERR_INVALID;
  auto it = bm->seqs.find(parent_id);
  if (it == bm->seqs.end()) return PA_BM_ERR_INVALID;
  Seq child = it->second;
  bm->changed(child);  // same blocks, but a row that held another table must be rewritten
  for (size_t k = static_cast<size_t>(child.released); k < child.blocks.size(); ++k)
    bm->ref(child.blocks[k]);
  bm->seqs.emplace(child_id, std::move(child));
  return PA_BM_OK;
}

int32_t pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id) {
  if (!bm) return PA_BM_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_BM_ERR_INVALID;
  Seq& s = it->second;
  for (size_t k = static_cast<size_t>(s.released); k < s.blocks.size(); ++k)
    bm->unref(s.blocks[k]);
  bm->seqs.erase(it);
  return PA_BM_OK;
}

int32_t pa_bm_release_before(pa_block_manager* bm, int64_t seq_id, int32_t position) {
  if (!bm || position < 0) return PA_BM_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end() || position > it->second.length) return PA_BM_ERR_INVALID;
  Seq& s = it->second;
  const int32_t upto = position / bm->bs;
  for (int32_t k = s.released; k < upto; ++k) bm->unref(s.blocks[k]);
  if (upto > s.released) s.released = upto;
  return PA_BM_OK;
}

int32_t pa_bm_release_window(pa_block_manager* bm, const int64_t* seq_ids, int32_t n,
                             int32_t window) {
  if (!bm || n < 0 || window < 1 || (n > 0 && !seq_ids)) return PA_BM_ERR_INVALID;
  std::vector<Seq*> rows(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PA_BM_ERR_INVALID;
    rows[static_cast<size_t>(i)] = &it->second;
  }
  for (Seq* s : rows) {
    // blocks holding only tokens before length - window
    const int32_t upto = std::max(s->length - window, 0) / bm->bs;
    for (int32_t k = s->released; k < upto; ++k) bm->unref(s->blocks[k]);
    if (upto > s->released) s->released = upto;
  }
  return PA_BM_OK;
}

int32_t pa_bm_sequence_length(const pa_block_manager* bm, int64_t seq_id) {
  if (!bm) return PA_BM_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  return it == bm->seqs.end() ? PA_BM_ERR_INVALID : it->second.length;
}

int32_t pa_bm_slots(const pa_block_manager* bm, int64_t seq_id, int32_t first, int32_t count,
                    int64_t* slots) {
  if (!bm || first < 0 || count < 0 || (count > 0 && !slots)) return PA_BM_ERR_INVALID;
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return PA_BM_ERR_INVALID;
  const Seq& s = it->second;
  if (static_cast<int64_t>(first) + count > s.length) return PA_BM_ERR_INVALID;
  if (count > 0 && first / bm->bs < s.released) return PA_BM_ERR_INVALID;
  for (int32_t i = 0; i < count; ++i) {
    const int32_t pos = first + i;
    slots[i] = s.blocks[pos / bm->bs] * bm->bs + pos % bm->bs;
  }
  return PA_BM_OK;
}

}  // extern "C"

namespace {

// Looks up every sequence of a batch and checks that its table fits, before
// anything is written.
int32_t lookup_rows(const pa_block_manager* bm, const int64_t* seq_ids, int32_t n_seqs,
                    int32_t max_blocks_per_seq, std::vector<const Seq*>& rows) {
  rows.resize(static_cast<size_t>(n_seqs));
  for (int32_t i = 0; i < n_seqs; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end()) return PA_BM_ERR_INVALID;
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks_per_seq)
      return PA_BM_ERR_CAPACITY;
    rows[static_cast<size_t>(i)] = &it->second;
  }
  return PA_BM_OK;
}

void write_row(const Seq& s, int32_t max_blocks_per_seq, int32_t* row) {
  const int32_t n = static_cast<int32_t>(s.blocks.size());
  const int64_t* src = s.blocks.data();
  for (int32_t k = 0; k < n; ++k) row[k] = static_cast<int32_t>(src[k]);
  std::fill(row + n, row + max_blocks_per_seq, 0);
}

}  // namespace

extern "C" {

int32_t pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int32_t n_seqs,
                           int32_t max_blocks_per_seq, int32_t* block_tables,
                           int32_t* context_lens) {
  if (!bm || n_seqs < 0 || max_blocks_per_seq <= 0 ||
      (n_seqs > 0 && (!seq_ids || !block_tables || !context_lens)))
    return PA_BM_ERR_INVALID;
  std::vector<const Seq*> rows;
  const int32_t rc = lookup_rows(bm, seq_ids, n_seqs, max_blocks_per_seq, rows);
  if (rc != PA_BM_OK) return rc;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq& s = *rows[static_cast<size_t>(i)];
    write_row(s, max_blocks_per_seq, block_tables + static_cast<int64_t>(i) * max_blocks_per_seq);
    context_lens[i] = s.length;
  }
  return PA_BM_OK;
}

int32_t pa_bm_block_tables_update(const pa_block_manager* bm, const int64_t* seq_ids,
                                  int32_t n_seqs, int32_t max_blocks_per_seq,
                                  int32_t* block_tables, int32_t* context_lens,
                                  uint64_t* row_versions, int32_t* rows_written) {
  if (!bm || n_seqs < 0 || max_blocks_per_seq <= 0 ||
      (n_seqs > 0 && (!seq_ids || !block_tables || !context_lens || !row_versions)))
    return PA_BM_ERR_INVALID;
  std::vector<const Seq*> rows;
  const int32_t rc = lookup_rows(bm, seq_ids, n_seqs, max_blocks_per_seq, rows);
  if (rc != PA_BM_OK) return rc;
  int32_t written = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Seq& s = *rows[static_cast<size_t>(i)];
    if (row_versions[i] != s.version) {
      write_row(s, max_blocks_per_seq, block_tables + static_cast<int64_t>(i) * max_blocks_per_seq);
      row_versions[i] = s.version;
      ++written;
    }
    context_lens[i] = s.length;
  }
  if (rows_written) *rows_written = written;
  return PA_BM_OK;
}

}  // extern "C"
