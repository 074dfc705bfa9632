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
// Data layout: flat arrays indexed by block id (holder counts), a vector used
// as the free stack (back = top), and a hash map from sequence id to the
// sequence's block vector.  Every operation checks all preconditions before it
// mutates anything, so a failed call leaves the pool unchanged.
#include <algorithm>
#include <cstdint>
#include <unordered_map>
#include <vector>

#include "host_common.h"

struct pa_pool {
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t len = 0;
  };
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // back() = next block handed out
  std::vector<int32_t> refs;        // holders per block
  std::unordered_map<int64_t, Seq> seqs;

  int32_t pop() {
    const int32_t b = free_stack.back();
    free_stack.pop_back();
    refs[b] = 1;
    return b;
  }
  void unref(int32_t b) {
    if (--refs[b] == 0) free_stack.push_back(b);
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
  if ((copy ? 1 : 0) + fresh > static_cast<int64_t>(pool->free_stack.size()))
    return pa::fail(PA_ERR_OOM, "pa_alloc: need %lld blocks, %zu free",
                    static_cast<long long>((copy ? 1 : 0) + fresh), pool->free_stack.size());
  if (len + n_new > (int64_t(1) << 40))
    return pa::fail(PA_ERR_INVALID, "pa_alloc: sequence too long");

  pa_pool::Seq& s = known ? it->second : pool->seqs[seq_id];
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
// call, and all or nothing -- on failure every sequence already grown in this
// batch is restored exactly (blocks go back on the free stack in the order
// they left it), so the pool is unchanged.
pa_status pa_alloc_batch(pa_pool* pool, const int64_t* seq_ids_host, int32_t n_seqs,
                         int32_t n_new_each, int64_t* slot_mapping_out_host,
                         int32_t* cow_pairs_out_host, int32_t max_cow, int32_t* n_cow_out) {
  if (!pool || n_seqs < 0 || n_new_each < 0 || !n_cow_out || max_cow < 0 ||
      (n_seqs > 0 && !seq_ids_host) ||
      (n_seqs > 0 && n_new_each > 0 && !slot_mapping_out_host) || (max_cow > 0 && !cow_pairs_out_host))
    return pa::fail(PA_ERR_INVALID, "pa_alloc_batch: bad arguments");
  struct Undo {
    int64_t seq;
    bool created;
    int64_t old_len;
    int32_t cow_src, cow_dst;
    int64_t fresh;
  };
  std::vector<Undo> log;
  log.reserve(n_seqs);
  int32_t n_cow = 0;
  pa_status st = PA_OK;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int64_t id = seq_ids_host[i];
    auto it = pool->seqs.find(id);
    const bool known = it != pool->seqs.end();
    const int64_t bs = pool->block_size;
    const int64_t len = known ? it->second.len : 0;
    const int64_t tail = len % bs;
    const int64_t fill = tail ? std::min<int64_t>(bs - tail, n_new_each) : 0;
    const bool copy = fill > 0 && pool->refs[it->second.blocks.back()] > 1;
    const int64_t fresh = (n_new_each - fill + bs - 1) / bs;
    if (copy && n_cow >= max_cow) {
      st = pa::fail(PA_ERR_INVALID, "pa_alloc_batch: more than max_cow=%d copy pairs", max_cow);
      break;
    }
    if ((copy ? 1 : 0) + fresh > static_cast<int64_t>(pool->free_stack.size())) {
      st = pa::fail(PA_ERR_OOM, "pa_alloc_batch: sequence %d of %d needs %lld blocks, %zu free",
                    i, n_seqs, static_cast<long long>((copy ? 1 : 0) + fresh),
                    pool->free_stack.size());
      break;
    }
    pa_pool::Seq& s = known ? it->second : pool->seqs[id];
    Undo u{id, !known, len, -1, -1, fresh};
    if (copy) {
      u.cow_src = s.blocks.back();
      u.cow_dst = pool->pop();
      pool->unref(u.cow_src);
      s.blocks.back() = u.cow_dst;
      cow_pairs_out_host[2 * n_cow] = u.cow_src;
      cow_pairs_out_host[2 * n_cow + 1] = u.cow_dst;
      ++n_cow;
    }
    for (int64_t k = 0; k < fresh; ++k) s.blocks.push_back(pool->pop());
    int64_t* slots = slot_mapping_out_host + static_cast<int64_t>(i) * n_new_each;
    for (int64_t k = 0; k < n_new_each; ++k) {
      const int64_t pos = len + k;
      slots[k] = static_cast<int64_t>(s.blocks[pos / bs]) * bs + pos % bs;
    }
    s.len = len + n_new_each;
    log.push_back(u);
  }
  if (st != PA_OK) {
    for (auto r = log.rbegin(); r != log.rend(); ++r) {
      pa_pool::Seq& s = pool->seqs[r->seq];
      for (int64_t k = 0; k < r->fresh; ++k) {
        const int32_t b = s.blocks.back();
        s.blocks.pop_back();
        pool->refs[b] = 0;
        pool->free_stack.push_back(b);
      }
      if (r->cow_dst >= 0) {
        s.blocks.back() = r->cow_src;
        pool->refs[r->cow_src] += 1;
        pool->refs[r->cow_dst] = 0;
        pool->free_stack.push_back(r->cow_dst);
      }
      s.len = r->old_len;
      if (r->created) pool->seqs.erase(r->seq);
    }
    return st;
  }
  *n_cow_out = n_cow;
  return PA_OK;
}

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
  if (n > static_cast<int32_t>(to->free_stack.size()))
    return pa::fail(PA_ERR_OOM, "pa_swap: %d blocks needed, %zu free in the destination", n,
                    to->free_stack.size());
  pa_pool::Seq moved;
  moved.len = it->second.len;
  moved.blocks.reserve(n);
  for (int32_t k = 0; k < n; ++k) {
    const int32_t b = to->pop();
    moved.blocks.push_back(b);
    pairs_out_host[2 * k] = src[k];
    pairs_out_host[2 * k + 1] = b;
  }
  for (int32_t b : src) from->unref(b);
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
  for (int32_t b : it->second.blocks) pool->unref(b);
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
  return pool ? static_cast<int32_t>(pool->free_stack.size()) : -1;
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
