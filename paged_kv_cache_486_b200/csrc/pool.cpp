// Host block pool: free stack, per-block holder counts, per-sequence block lists.
//
// "PagedAttention for professionals..." / "The scientific explanation": the KV
// cache is split into fixed-size blocks stored anywhere in GPU memory, and a
// block table per request maps logical blocks to physical ones.  Same page,
// "Beginner example: library shelves": a request takes a block only when it
// needs one and a finished request's blocks are reused at once.  "KV Cache and
// PagedAttention: Why Your LLM Server Slows Down" / "How PagedAttention solves
// this": on-demand pages; shared prefix pages with copy-on-write.
//
// Data layout: flat arrays indexed by block id (holder counts, prefix-cache
// flags and the links of the evictable list), a vector used as the free stack
// (back = top), and a hash map from sequence id to the sequence's block vector.
// Every operation checks all preconditions before it mutates anything, so a
// failed call leaves the pool unchanged.
//
// Prefix caching ("The KV cache and PagedAttention: why the LLM server chokes
// at 10 users" / the serving example with --enable-prefix-caching, and "The
// trade-offs": blocks are reused when several requests share the same
// beginning, such as one system prompt; the cached blocks occupy the pool) is
// opt-in per pool and described with pa_pool_set_prefix_caching in pa.h.
#include <algorithm>
#include <cstdint>
#include <unordered_map>
#include <vector>

#include "host_common.h"

struct pa_pool {
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t len = 0;
    // Prefix-cache state: token ids are known for every token (pa_alloc_tokens
    // only); `hashed` full blocks have been keyed, `chain` is the key of the
    // last of them, `tail` holds the ids of the tokens after them.
    bool ids_known = true;
    int64_t hashed = 0;
    uint64_t chain = kRootKey;
    std::vector<int32_t> tail;
  };
  static constexpr uint64_t kRootKey = 0x9e3779b97f4a7c15ull;

  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // back() = next block handed out
  std::vector<int32_t> refs;        // holders per block (sequences)
  std::unordered_map<int64_t, Seq> seqs;

  // Prefix cache: full blocks keyed by their token prefix.  A key is a 64-bit
  // chain over (parent key, the block's token ids); each entry keeps its parent
  // key and token ids, and a lookup compares them, so two different blocks
  // only collide if their parents' 64-bit keys do.  A cached block with no
  // holder waits in an LRU list (lru_*, oldest at the head) and is still found
  // by lookups; fresh allocation takes the free stack first, then evicts the
  // head of that list.
  bool prefix = false;
  struct Entry {
    int32_t block;
    uint64_t parent;
    std::vector<int32_t> tokens;
  };
  std::unordered_map<uint64_t, Entry> entries;
  std::vector<uint64_t> key_of;     // key of a cached block
  std::vector<uint8_t> cached;      // block has an entry
  std::vector<int32_t> lru_prev, lru_next;
  int32_t lru_head = -1, lru_tail = -1, n_evictable = 0;

  size_t available() const { return free_stack.size() + static_cast<size_t>(n_evictable); }

  void lru_push_back(int32_t b) {
    lru_prev[b] = lru_tail;
    lru_next[b] = -1;
    if (lru_tail >= 0) lru_next[lru_tail] = b; else lru_head = b;
    lru_tail = b;
    ++n_evictable;
  }
  void lru_remove(int32_t b) {
    if (lru_prev[b] >= 0) lru_next[lru_prev[b]] = lru_next[b]; else lru_head = lru_next[b];
    if (lru_next[b] >= 0) lru_prev[lru_next[b]] = lru_prev[b]; else lru_tail = lru_prev[b];
    lru_prev[b] = lru_next[b] = -1;
    --n_evictable;
  }
  void uncache(int32_t b) {
    entries.erase(key_of[b]);
    cached[b] = 0;
  }
  // A block for new tokens: the top of the free stack, else the least recently
  // released cached block (its entry is dropped).
  int32_t pop() {
    int32_t b;
    if (!free_stack.empty()) {
      b = free_stack.back();
      free_stack.pop_back();
    } else {
      b = lru_head;
      lru_remove(b);
      uncache(b);
    }
    refs[b] = 1;
    return b;
  }
  // One more holder for a cached block found by a lookup.
  void hold(int32_t b) {
    if (refs[b]++ == 0) lru_remove(b);
  }
  // Drop one holder of each block of a list.  Blocks left without a holder
  // return to the free stack in list order, or, if cached, join the LRU list
  // in reverse list order (a sequence's later blocks are evicted first).
  void release(const std::vector<int32_t>& bl) {
    for (int32_t b : bl)
      if (--refs[b] == 0 && !cached[b]) free_stack.push_back(b);
    for (auto r = bl.rbegin(); r != bl.rend(); ++r)
      if (refs[*r] == 0 && cached[*r]) lru_push_back(*r);
  }
  void unref(int32_t b) { release(std::vector<int32_t>{b}); }

  static uint64_t mix(uint64_t x) {
    x ^= x >> 31;
    x *= 0x7fb5d329728ea185ull;
    x ^= x >> 27;
    x *= 0x81dadef4bc2dd44dull;
    x ^= x >> 33;
    return x;
  }
  static uint64_t block_key(uint64_t parent, const int32_t* ids, int n) {
    uint64_t h = mix(parent ^ 0x5851f42d4c957f2dull);
    for (int i = 0; i < n; ++i) h = mix(h + static_cast<uint32_t>(ids[i]) + 0x632be59bd9b4e019ull);
    return h;
  }
  // The cached block holding (parent, ids), or -1.
  int32_t lookup(uint64_t key, uint64_t parent, const int32_t* ids) const {
    auto e = entries.find(key);
    if (e == entries.end() || e->second.parent != parent ||
        !std::equal(e->second.tokens.begin(), e->second.tokens.end(), ids))
      return -1;
    return e->second.block;
  }
  // Key every full block of `s` not keyed yet (its ids are known); register
  // those whose key has no entry (while caching is on).
  void key_full_blocks(Seq& s) {
    const int64_t bs = block_size;
    while (s.ids_known && (s.hashed + 1) * bs <= s.len) {
      const uint64_t key = block_key(s.chain, s.tail.data(), block_size);
      if (prefix && lookup(key, s.chain, s.tail.data()) < 0 && !entries.count(key)) {
        const int32_t b = s.blocks[s.hashed];
        entries.emplace(key, Entry{b, s.chain, std::vector<int32_t>(s.tail.begin(),
                                                                    s.tail.begin() + bs)});
        key_of[b] = key;
        cached[b] = 1;
      }
      s.chain = key;
      ++s.hashed;
      s.tail.erase(s.tail.begin(), s.tail.begin() + bs);
    }
  }
  void forget_ids(Seq& s) {
    s.ids_known = false;
    s.tail.clear();
    s.tail.shrink_to_fit();
  }
};

extern "C" {

pa_status pa_pool_create(int32_t num_blocks, int32_t block_size, pa_pool** pool_out) {
  if (!pool_out) return pa::fail(PA_ERR_INVALID, "pa_pool_create: pool_out is NULL");
  if (num_blocks < 0 || block_size < 1)
    return pa::fail(PA_ERR_INVALID, "pa_pool_create: num_blocks=%d block_size=%d", num_blocks,
                    block_size);
  pa_pool* p = new pa_pool;
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  p->refs.assign(num_blocks, 0);
  p->key_of.assign(num_blocks, 0);
  p->cached.assign(num_blocks, 0);
  p->lru_prev.assign(num_blocks, -1);
  p->lru_next.assign(num_blocks, -1);
  p->free_stack.resize(num_blocks);
  for (int32_t i = 0; i < num_blocks; ++i) p->free_stack[i] = num_blocks - 1 - i;
  *pool_out = p;
  return PA_OK;
}

void pa_pool_destroy(pa_pool* pool) { delete pool; }

pa_status pa_alloc(pa_pool* pool, int64_t seq_id, int32_t n_new, int64_t* slot_mapping_out_host,
                   int32_t* cow_pairs_out_host, int32_t max_cow, int32_t* n_cow_out) {
  if (!pool || n_new < 0 || (n_new > 0 && !slot_mapping_out_host) || !n_cow_out)
    return pa::fail(PA_ERR_INVALID, "pa_alloc: bad arguments (n_new=%d)", n_new);
  const int64_t bs = pool->block_size;
  auto it = pool->seqs.find(seq_id);
  const bool known = it != pool->seqs.end();
  const int64_t len = known ? it->second.len : 0;
  const int64_t tail = len % bs;
  const int64_t fill = tail ? std::min<int64_t>(bs - tail, n_new) : 0;
  const bool copy = fill > 0 && pool->refs[it->second.blocks.back()] > 1;
  const int64_t fresh = (n_new - fill + bs - 1) / bs;
  if (copy && (max_cow < 1 || !cow_pairs_out_host))
    return pa::fail(PA_ERR_INVALID, "pa_alloc: a copy-on-write pair is needed but max_cow=%d",
                    max_cow);
  if ((copy ? 1 : 0) + fresh > static_cast<int64_t>(pool->available()))
    return pa::fail(PA_ERR_OOM, "pa_alloc: need %lld blocks, %zu free",
                    static_cast<long long>((copy ? 1 : 0) + fresh), pool->available());
  if (len + n_new > (int64_t(1) << 40))
    return pa::fail(PA_ERR_INVALID, "pa_alloc: sequence too long");

  pa_pool::Seq& s = known ? it->second : pool->seqs[seq_id];
  if (n_new > 0) pool->forget_ids(s);  // tokens without ids: no more prefix keys
  *n_cow_out = 0;
  if (copy) {
    const int32_t src = s.blocks.back();
    const int32_t dst = pool->pop();
    pool->unref(src);
    s.blocks.back() = dst;
    cow_pairs_out_host[0] = src;
    cow_pairs_out_host[1] = dst;
    *n_cow_out = 1;
  }
  s.blocks.reserve(s.blocks.size() + fresh);
  for (int64_t k = 0; k < fresh; ++k) s.blocks.push_back(pool->pop());
  for (int64_t i = 0; i < n_new; ++i) {
    const int64_t pos = len + i;
    slot_mapping_out_host[i] = static_cast<int64_t>(s.blocks[pos / bs]) * bs + pos % bs;
  }
  s.len = len + n_new;
  return PA_OK;
}

// Batched growth: the same effect as n_seqs calls of pa_alloc in order, but one
// call, and all or nothing.  A first pass replays the batch on the lengths,
// last blocks and holder counts it touches (a copy-on-write of a shared last
// block drops that block's holder count, which can spare a later sequence its
// copy) and checks the block demand and the copy pairs; the second pass then
// cannot fail, so it never has to undo (an undo could not restore a cached
// block that an allocation evicted).
pa_status pa_alloc_batch(pa_pool* pool, const int64_t* seq_ids_host, int32_t n_seqs,
                         int32_t n_new_each, int64_t* slot_mapping_out_host,
                         int32_t* cow_pairs_out_host, int32_t max_cow, int32_t* n_cow_out) {
  if (!pool || n_seqs < 0 || n_new_each < 0 || !n_cow_out || max_cow < 0 ||
      (n_seqs > 0 && !seq_ids_host) ||
      (n_seqs > 0 && n_new_each > 0 && !slot_mapping_out_host) || (max_cow > 0 && !cow_pairs_out_host))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_batch: bad arguments");
  const int64_t bs = pool->block_size;
  {
    std::unordered_map<int64_t, std::pair<int64_t, int32_t>> sim;  // id -> (len, last block)
    std::unordered_map<int32_t, int32_t> drop;                      // block -> holders lost
    int64_t need = 0;
    int32_t cows = 0;
    for (int32_t i = 0; i < n_seqs; ++i) {
      const int64_t id = seq_ids_host[i];
      auto si = sim.find(id);
      int64_t len;
      int32_t last;  // -1: none, -2: a block this batch gave the sequence
      if (si != sim.end()) {
        len = si->second.first;
        last = si->second.second;
      } else {
        auto it = pool->seqs.find(id);
        len = it == pool->seqs.end() ? 0 : it->second.len;
        last = it == pool->seqs.end() || it->second.blocks.empty() ? -1 : it->second.blocks.back();
      }
      const int64_t tail = len % bs;
      const int64_t fill = tail ? std::min<int64_t>(bs - tail, n_new_each) : 0;
      const bool copy = fill > 0 && last >= 0 && pool->refs[last] - drop[last] > 1;
      const int64_t fresh = (n_new_each - fill + bs - 1) / bs;
      if (copy) {
        ++cows;
        ++drop[last];
        last = -2;
      }
      if (fresh > 0) last = -2;
      need += (copy ? 1 : 0) + fresh;
      sim[id] = {len + n_new_each, last};
      if (len + n_new_each > (int64_t(1) << 40))
        return pa::fail(PA_ERR_INVALID, "pa_alloc_batch: sequence too long");
    }
    if (cows > max_cow)
      return pa::fail(PA_ERR_INVALID, "pa_alloc_batch: %d copy pairs needed, room for %d", cows,
                      max_cow);
    if (need > static_cast<int64_t>(pool->available()))
      return pa::fail(PA_ERR_OOM, "pa_alloc_batch: need %lld blocks, %zu free",
                      static_cast<long long>(need), pool->available());
  }
  int32_t n_cow = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int64_t id = seq_ids_host[i];
    auto it = pool->seqs.find(id);
    const bool known = it != pool->seqs.end();
    const int64_t len = known ? it->second.len : 0;
    const int64_t tail = len % bs;
    const int64_t fill = tail ? std::min<int64_t>(bs - tail, n_new_each) : 0;
    const bool copy = fill > 0 && pool->refs[it->second.blocks.back()] > 1;
    const int64_t fresh = (n_new_each - fill + bs - 1) / bs;
    pa_pool::Seq& s = known ? it->second : pool->seqs[id];
    if (n_new_each > 0) pool->forget_ids(s);
    if (copy) {
      const int32_t src = s.blocks.back();
      const int32_t dst = pool->pop();
      pool->unref(src);
      s.blocks.back() = dst;
      cow_pairs_out_host[2 * n_cow] = src;
      cow_pairs_out_host[2 * n_cow + 1] = dst;
      ++n_cow;
    }
    for (int64_t k = 0; k < fresh; ++k) s.blocks.push_back(pool->pop());
    int64_t* slots = slot_mapping_out_host + static_cast<int64_t>(i) * n_new_each;
    for (int64_t k = 0; k < n_new_each; ++k) {
      const int64_t pos = len + k;
      slots[k] = static_cast<int64_t>(s.blocks[pos / bs]) * bs + pos % bs;
    }
    s.len = len + n_new_each;
  }
  *n_cow_out = n_cow;
  return PA_OK;
}

// Growth with token ids, and prefix-cache lookups for a new sequence (see
// pa.h).  All or nothing: the blocks it must take (those the cache does not
// supply, plus a copy-on-write block) are checked against the free stack plus
// the evictable cached blocks that are not among its own hits, before anything
// changes.
pa_status pa_alloc_tokens(pa_pool* pool, int64_t seq_id, const int32_t* token_ids_host,
                          int32_t n_new, int64_t* slot_mapping_out_host,
                          int32_t* cow_pairs_out_host, int32_t max_cow, int32_t* n_cow_out,
                          int32_t* n_cached_out) {
  if (!pool || n_new < 0 || (n_new > 0 && (!slot_mapping_out_host || !token_ids_host)) ||
      !n_cow_out || !n_cached_out)
    return pa::fail(PA_ERR_INVALID, "pa_alloc_tokens: bad arguments (n_new=%d)", n_new);
  const int64_t bs = pool->block_size;
  auto it = pool->seqs.find(seq_id);
  const bool known = it != pool->seqs.end();
  const int64_t len = known ? it->second.len : 0;
  // cache lookups: a sequence that holds no token yet, whole blocks that end
  // before its last new token (that token is always computed)
  std::vector<int32_t> hits;
  uint64_t chain = pa_pool::kRootKey;
  int32_t hits_evictable = 0;
  if (pool->prefix && len == 0 && (!known || it->second.ids_known)) {
    for (int64_t j = 0; (j + 1) * bs <= static_cast<int64_t>(n_new) - 1; ++j) {
      const int32_t* ids = token_ids_host + j * bs;
      const uint64_t key = pa_pool::block_key(chain, ids, pool->block_size);
      const int32_t b = pool->lookup(key, chain, ids);
      if (b < 0) break;
      hits.push_back(b);
      hits_evictable += pool->refs[b] == 0 ? 1 : 0;
      chain = key;
    }
  }
  const int64_t hit_tokens = static_cast<int64_t>(hits.size()) * bs;
  const int64_t tail = len % bs;
  const int64_t fill = tail ? std::min<int64_t>(bs - tail, n_new) : 0;
  const bool copy = fill > 0 && pool->refs[it->second.blocks.back()] > 1;
  const int64_t fresh = (n_new - hit_tokens - fill + bs - 1) / bs;
  if (copy && (max_cow < 1 || !cow_pairs_out_host))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_tokens: a copy-on-write pair is needed but "
                    "max_cow=%d", max_cow);
  const int64_t avail = static_cast<int64_t>(pool->available()) - hits_evictable;
  if ((copy ? 1 : 0) + fresh > avail)
    return pa::fail(PA_ERR_OOM, "pa_alloc_tokens: need %lld blocks, %lld free",
                    static_cast<long long>((copy ? 1 : 0) + fresh), static_cast<long long>(avail));
  if (len + n_new > (int64_t(1) << 40))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_tokens: sequence too long");

  pa_pool::Seq& s = known ? it->second : pool->seqs[seq_id];
  for (int32_t b : hits) {
    pool->hold(b);
    s.blocks.push_back(b);
  }
  *n_cow_out = 0;
  if (copy) {
    const int32_t src = s.blocks.back();
    const int32_t dst = pool->pop();
    pool->unref(src);
    s.blocks.back() = dst;
    cow_pairs_out_host[0] = src;
    cow_pairs_out_host[1] = dst;
    *n_cow_out = 1;
  }
  for (int64_t k = 0; k < fresh; ++k) s.blocks.push_back(pool->pop());
  for (int64_t i = 0; i < n_new; ++i) {
    const int64_t pos = len + i;
    slot_mapping_out_host[i] =
        i < hit_tokens ? -1 : static_cast<int64_t>(s.blocks[pos / bs]) * bs + pos % bs;
  }
  s.len = len + n_new;
  if (s.ids_known) {
    if (!hits.empty()) {
      s.hashed = static_cast<int64_t>(hits.size());
      s.chain = chain;
    }
    s.tail.insert(s.tail.end(), token_ids_host + hit_tokens, token_ids_host + n_new);
    pool->key_full_blocks(s);
  }
  *n_cached_out = static_cast<int32_t>(hit_tokens);
  return PA_OK;
}

pa_status pa_pool_set_prefix_caching(pa_pool* pool, int32_t enable) {
  if (!pool) return pa::fail(PA_ERR_INVALID, "pa_pool_set_prefix_caching: NULL pool");
  if (enable) {
    pool->prefix = true;
    return PA_OK;
  }
  pool->prefix = false;
  // evictable cached blocks become plain free blocks (oldest pushed first)
  while (pool->lru_head >= 0) {
    const int32_t b = pool->lru_head;
    pool->lru_remove(b);
    pool->free_stack.push_back(b);
  }
  pool->entries.clear();
  std::fill(pool->cached.begin(), pool->cached.end(), 0);
  return PA_OK;
}

int32_t pa_num_cached_blocks(const pa_pool* pool) {
  return pool ? static_cast<int32_t>(pool->entries.size()) : -1;
}

int32_t pa_num_evictable_blocks(const pa_pool* pool) { return pool ? pool->n_evictable : -1; }

// "KV Cache and PagedAttention: Why Your LLM Server Slows Down" / "How
// PagedAttention solves this": under memory pressure small pages move to the
// CPU.  The sequence moves to `to` with one new block per old block (logical
// order) and the same length; its old blocks each lose one holder.  Nothing
// changes unless `to` has room for every block.
pa_status pa_swap(pa_pool* from, pa_pool* to, int64_t seq_id, int32_t* pairs_out_host,
                  int32_t max_pairs, int32_t* n_pairs_out) {
  if (!from || !to || from == to || !n_pairs_out || max_pairs < 0 ||
      (max_pairs > 0 && !pairs_out_host))
    return pa::fail(PA_ERR_INVALID, "pa_swap: bad arguments");
  if (from->block_size != to->block_size)
    return pa::fail(PA_ERR_INVALID, "pa_swap: block sizes differ (%d vs %d)", from->block_size,
                    to->block_size);
  auto it = from->seqs.find(seq_id);
  if (it == from->seqs.end())
    return pa::fail(PA_ERR_NOT_FOUND, "pa_swap: unknown sequence %lld",
                    static_cast<long long>(seq_id));
  if (to->seqs.count(seq_id))
    return pa::fail(PA_ERR_INVALID, "pa_swap: sequence %lld is already in the destination pool",
                    static_cast<long long>(seq_id));
  const std::vector<int32_t>& src = it->second.blocks;
  const int32_t n = static_cast<int32_t>(src.size());
  if (n > max_pairs)
    return pa::fail(PA_ERR_INVALID, "pa_swap: %d pairs needed, room for %d", n, max_pairs);
  if (n > static_cast<int32_t>(to->available()))
    return pa::fail(PA_ERR_OOM, "pa_swap: %d blocks needed, %zu free in the destination", n,
                    to->available());
  pa_pool::Seq moved;
  moved.len = it->second.len;
  moved.ids_known = it->second.ids_known;  // keys continue; the moved blocks are not cached
  moved.hashed = it->second.hashed;
  moved.chain = it->second.chain;
  moved.tail = it->second.tail;
  moved.blocks.reserve(n);
  for (int32_t k = 0; k < n; ++k) {
    const int32_t b = to->pop();
    moved.blocks.push_back(b);
    pairs_out_host[2 * k] = src[k];
    pairs_out_host[2 * k + 1] = b;
  }
  from->release(src);
  from->seqs.erase(it);
  to->seqs.emplace(seq_id, std::move(moved));
  *n_pairs_out = n;
  return PA_OK;
}

pa_status pa_free(pa_pool* pool, int64_t seq_id) {
  if (!pool) return pa::fail(PA_ERR_INVALID, "pa_free: NULL pool");
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_NOT_FOUND, "pa_free: unknown sequence %lld",
                    static_cast<long long>(seq_id));
  pool->release(it->second.blocks);
  pool->seqs.erase(it);
  return PA_OK;
}

pa_status pa_fork(pa_pool* pool, int64_t parent_id, int64_t child_id) {
  if (!pool) return pa::fail(PA_ERR_INVALID, "pa_fork: NULL pool");
  auto it = pool->seqs.find(parent_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_NOT_FOUND, "pa_fork: unknown parent %lld",
                    static_cast<long long>(parent_id));
  if (pool->seqs.count(child_id))
    return pa::fail(PA_ERR_INVALID, "pa_fork: child %lld exists", static_cast<long long>(child_id));
  pa_pool::Seq child = it->second;  // copy before inserting (rehash may move `it`)
  for (int32_t b : child.blocks) pool->refs[b] += 1;
  pool->seqs.emplace(child_id, std::move(child));
  return PA_OK;
}

pa_status pa_block_table(const pa_pool* pool, const int64_t* seq_ids_host, int32_t n_seqs,
                         int32_t max_blocks, int32_t* table_out_host, int32_t* ctx_lens_out_host) {
  if (!pool || n_seqs < 0 || max_blocks < 0 ||
      (n_seqs > 0 && (!seq_ids_host || !table_out_host || !ctx_lens_out_host)))
    return pa::fail(PA_ERR_INVALID, "pa_block_table: bad arguments");
  for (int32_t i = 0; i < n_seqs; ++i) {
    auto it = pool->seqs.find(seq_ids_host[i]);
    if (it == pool->seqs.end())
      return pa::fail(PA_ERR_NOT_FOUND, "pa_block_table: unknown sequence %lld",
                      static_cast<long long>(seq_ids_host[i]));
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks)
      return pa::fail(PA_ERR_INVALID, "pa_block_table: sequence %lld holds %zu blocks > %d",
                      static_cast<long long>(seq_ids_host[i]), it->second.blocks.size(),
                      max_blocks);
    if (it->second.len > INT32_MAX)
      return pa::fail(PA_ERR_INVALID, "pa_block_table: context length exceeds int32");
  }
  for (int32_t i = 0; i < n_seqs; ++i) {
    const pa_pool::Seq& s = pool->seqs.find(seq_ids_host[i])->second;
    int32_t* row = table_out_host + static_cast<int64_t>(i) * max_blocks;
    const int32_t n = static_cast<int32_t>(s.blocks.size());
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    std::fill(row + n, row + max_blocks, -1);
    ctx_lens_out_host[i] = static_cast<int32_t>(s.len);
  }
  return PA_OK;
}

int32_t pa_num_free_blocks(const pa_pool* pool) {
  return pool ? static_cast<int32_t>(pool->available()) : -1;
}

int32_t pa_refcount(const pa_pool* pool, int32_t block) {
  if (!pool || block < 0 || block >= pool->num_blocks) return -1;
  return pool->refs[block];
}

int64_t pa_seq_len(const pa_pool* pool, int64_t seq_id) {
  if (!pool) return -1;
  auto it = pool->seqs.find(seq_id);
  return it == pool->seqs.end() ? -1 : it->second.len;
}

uint64_t pa_kv_bytes(int32_t num_layers, int64_t num_tokens, int32_t num_kv_heads,
                     int32_t head_dim, int32_t dtype_bytes) {
  if (num_layers < 0 || num_tokens < 0 || num_kv_heads < 0 || head_dim < 0 || dtype_bytes < 0)
    return 0;
  // "KV Cache for intermediates..." / "The precise scientific definition".
  return uint64_t(2) * uint64_t(num_layers) * uint64_t(num_tokens) * uint64_t(num_kv_heads) *
         uint64_t(head_dim) * uint64_t(dtype_bytes);
}

// ------------------------------- validators --------------------------------
pa_status pa_validate_slot_mapping(const int64_t* slot_mapping_host, int32_t n_tokens,
                                   int32_t block_size, int32_t num_blocks) {
  if (n_tokens < 0 || (n_tokens > 0 && !slot_mapping_host) || block_size < 1 || num_blocks < 0)
    return pa::fail(PA_ERR_INVALID, "pa_validate_slot_mapping: bad arguments");
  const int64_t limit = static_cast<int64_t>(num_blocks) * block_size;
  std::vector<int64_t> seen;
  seen.reserve(n_tokens);
  for (int32_t t = 0; t < n_tokens; ++t) {
    const int64_t s = slot_mapping_host[t];
    if (s == -1) continue;
    if (s < 0 || s >= limit)
      return pa::fail(PA_ERR_INVALID, "slot_mapping[%d] = %lld outside [0, %lld)", t,
                      static_cast<long long>(s), static_cast<long long>(limit));
    seen.push_back(s);
  }
  std::sort(seen.begin(), seen.end());
  if (std::adjacent_find(seen.begin(), seen.end()) != seen.end())
    return pa::fail(PA_ERR_INVALID, "slot_mapping repeats a slot");
  return PA_OK;
}

pa_status pa_validate_block_table(const int32_t* block_tables_host,
                                  const int32_t* context_lens_host, int32_t batch,
                                  int32_t max_blocks, int32_t block_size, int32_t num_blocks) {
  if (batch < 0 || max_blocks < 0 || block_size < 1 ||
      (batch > 0 && (!block_tables_host || !context_lens_host)))
    return pa::fail(PA_ERR_INVALID, "pa_validate_block_table: bad arguments");
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t ctx = context_lens_host[b];
    if (ctx < 0 || ctx > static_cast<int64_t>(max_blocks) * block_size)
      return pa::fail(PA_ERR_INVALID, "context_lens[%d] = %lld outside [0, %lld]", b,
                      static_cast<long long>(ctx),
                      static_cast<long long>(max_blocks) * block_size);
    const int64_t nblk = (ctx + block_size - 1) / block_size;
    for (int64_t j = 0; j < nblk; ++j) {
      const int32_t id = block_tables_host[static_cast<int64_t>(b) * max_blocks + j];
      if (id < 0 || id >= num_blocks)
        return pa::fail(PA_ERR_INVALID, "block_tables[%d][%lld] = %d outside [0, %d)", b,
                        static_cast<long long>(j), id, num_blocks);
    }
  }
  return PA_OK;
}

pa_status pa_validate_copy_pairs(const int32_t* pairs_host, int32_t n_pairs, int32_t num_blocks) {
  if (n_pairs < 0 || (n_pairs > 0 && !pairs_host))
    return pa::fail(PA_ERR_INVALID, "pa_validate_copy_pairs: bad arguments");
  std::vector<int32_t> srcs, dsts;
  for (int32_t i = 0; i < n_pairs; ++i) {
    const int32_t s = pairs_host[2 * i], d = pairs_host[2 * i + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks)
      return pa::fail(PA_ERR_INVALID, "pair %d = (%d, %d) outside [0, %d)", i, s, d, num_blocks);
    srcs.push_back(s);
    dsts.push_back(d);
  }
  std::sort(srcs.begin(), srcs.end());
  std::sort(dsts.begin(), dsts.end());
  if (std::adjacent_find(dsts.begin(), dsts.end()) != dsts.end())
    return pa::fail(PA_ERR_INVALID, "a destination block repeats");
  for (int32_t d : dsts)
    if (std::binary_search(srcs.begin(), srcs.end(), d))
      return pa::fail(PA_ERR_INVALID, "block %d is both a source and a destination", d);
  return PA_OK;
}

}  // extern "C"
