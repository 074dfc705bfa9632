// Oracle for the paged decode hot path.  TEST INFRASTRUCTURE, NOT PRODUCT CODE.
//
// Only the test suite, the package smoke check and the benchmark's CPU-baseline
// leg may load this library.  It shares no code, header or table with the CUDA
// library: it is a plain, slow, literal restatement of what the pages describe,
// in fp64 for the floating-point parts, so that a reader can check it by eye.
//
// Sources (web pages, cited by title and section):
//  [P1] "PagedAttention for professionals: how vLLM serves more requests on the
//       same H100" -- "The problem in brief", "Beginner example: library shelves",
//       "The scientific explanation: why PagedAttention is a breakthrough" and the
//       results list under it.
//  [P2] "KV Cache and PagedAttention: Why Your LLM Server Slows Down" -- "What is
//       the KV cache?", "How PagedAttention solves this", "How does PagedAttention
//       work?", "Key benefits".
//  [P5] "KV Cache for intermediates: why long context eats the GPU and how to cut
//       it 4x" -- "The precise scientific definition" (the KV-size formula) and
//       "The four solutions" (MQA, GQA, PagedAttention).
//
// Where the pages are silent the reading taken is stated next to the code and
// listed in the design notes.
//
// Parity status: every function here is pinned by a "not gpu" test (closed
// forms, invariants, brute force, or library routines on special cases); none
// is "parity unpinned".

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <deque>
#include <map>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Number formats.  Written from the IEEE 754 binary16 definition and from the
// bfloat16 definition (the upper 16 bits of an IEEE binary32).
// ---------------------------------------------------------------------------

double f16_bits_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int expo = (h >> 10) & 0x1f;
  const int mant = h & 0x3ff;
  double mag;
  if (expo == 0) {
    mag = std::ldexp(static_cast<double>(mant), -24);          // subnormal
  } else if (expo == 31) {
    mag = mant ? NAN : INFINITY;
  } else {
    mag = std::ldexp(static_cast<double>(1024 + mant), expo - 25);
  }
  return sign ? -mag : mag;
}

double bf16_bits_to_double(uint16_t b) {
  const uint32_t w = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &w, sizeof f);
  return static_cast<double>(f);
}

// Round |x| to the grid of a binary format with `sig` significant bits,
// smallest normal exponent `emin` (value 2^emin), ties to even.  Returns the
// rounded magnitude as a double (exact, since every such value fits a double).
double round_to_format(double a, int sig, int emin) {
  if (a == 0.0) return 0.0;
  int e2;
  std::frexp(a, &e2);            // a = f * 2^e2, f in [0.5, 1)
  int e = e2 - 1;                // a in [2^e, 2^(e+1))
  if (e < emin) e = emin;        // subnormal range shares the quantum of 2^emin
  const double quantum = std::ldexp(1.0, e - (sig - 1));
  const double n = a / quantum;  // exact: dividing by a power of two
  const double r = std::nearbyint(n);  // default rounding mode: nearest, ties to even
  return r * quantum;
}

uint16_t double_to_f16_bits(double x) {
  if (std::isnan(x)) return 0x7e00;
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double r = round_to_format(std::fabs(x), 11, -14);
  if (r >= 65536.0) return sign | 0x7c00;  // rounded past the largest finite value
  if (r == 0.0) return sign;
  if (r < std::ldexp(1.0, -14)) {
    return sign | static_cast<uint16_t>(r / std::ldexp(1.0, -24));  // subnormal
  }
  int e2;
  std::frexp(r, &e2);
  const int e = e2 - 1;
  const uint16_t mant = static_cast<uint16_t>(r / std::ldexp(1.0, e - 10) - 1024.0);
  return sign | static_cast<uint16_t>((e + 15) << 10) | mant;
}

uint16_t double_to_bf16_bits(double x) {
  if (std::isnan(x)) return 0x7fc0;
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double r = round_to_format(std::fabs(x), 8, -126);
  if (r >= std::ldexp(1.0, 128)) return sign | 0x7f80;
  if (r == 0.0) return sign;
  if (r < std::ldexp(1.0, -126)) {
    return sign | static_cast<uint16_t>(r / std::ldexp(1.0, -133));
  }
  int e2;
  std::frexp(r, &e2);
  const int e = e2 - 1;
  const uint16_t mant = static_cast<uint16_t>(r / std::ldexp(1.0, e - 7) - 128.0);
  return sign | static_cast<uint16_t>((e + 127) << 7) | mant;
}

// dtype codes: 0 = fp32, 1 = fp16, 2 = bf16 (element of the cache, q and output)
double load_elem(const void* base, int64_t idx, int dtype) {
  if (dtype == 0) return static_cast<double>(static_cast<const float*>(base)[idx]);
  const uint16_t bits = static_cast<const uint16_t*>(base)[idx];
  return dtype == 1 ? f16_bits_to_double(bits) : bf16_bits_to_double(bits);
}

// ---------------------------------------------------------------------------
// Block pool model.
//
// [P1] "The scientific explanation": the KV cache is split into fixed-size
// blocks (default 16 tokens), each stored anywhere in GPU memory, and a block
// table per request maps logical blocks to physical ones.  [P1] "Beginner
// example: library shelves": a request takes a new block only when its 17th
// token arrives, and a finished request's blocks return to the pool where the
// next request takes them at once.  [P2] "How PagedAttention solves this":
// pages are taken on demand as a sequence grows; sequences share the physical
// pages of a common prefix, with copy-on-write.  [P1] results list: parallel
// sampling with n=4 takes about the memory of n=1.
//
// Readings where the pages are silent:
//  * The free list is a stack (last freed, first reused).  Initially block 0 is
//    on top, so a fresh pool hands out 0, 1, 2, ...
//  * A sequence that grows into a partially filled last block that other
//    sequences also hold copies that block first (one copy pair per call); a
//    full shared block stays shared; the last holder writes in place.
//  * An allocation either succeeds completely or changes nothing.
//
// Prefix caching ([P3] the serving example with --enable-prefix-caching: a
// request reuses the blocks of another request that began the same way, such
// as one system prompt; [P3] "The trade-offs": those cached blocks take space
// in the pool).  Readings where the pages are silent:
//  * Only full blocks are cached, each under the exact list of token ids from
//    the sequence's start to the block's end.  A full block is entered once its
//    sequence's ids are all known (given with the tokens), unless that list
//    already has a block.
//  * A sequence receiving its first tokens reuses cached blocks for its
//    leading full blocks while they match, but never one holding the last of
//    the tokens given (that token is always computed).
//  * A cached block whose last holder lets go stays findable, in a queue of
//    releasable blocks (a sequence's blocks in reverse logical order).  New
//    blocks come from the free stack first, then from the front of that queue
//    (the block leaves the cache).
//  * Growth without ids ends the sequence's entries; turning caching off
//    returns the queue to the free stack (front first) and empties the cache.
// ---------------------------------------------------------------------------

struct Sequence {
  std::deque<int32_t> blocks;  // logical block j -> physical block id
  int64_t len = 0;             // tokens held
  bool ids_known = true;       // every token came with its id
  std::vector<int32_t> ids;    // the token ids (while ids_known)
  int64_t considered = 0;      // full blocks already offered to the cache
};

struct Pool {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::deque<int32_t> free_stack;      // back() is the top of the stack
  std::map<int32_t, int32_t> holders;  // physical block -> number of sequences holding it
  std::map<int64_t, Sequence> seqs;
  bool prefix = false;                               // prefix caching on
  std::map<std::vector<int32_t>, int32_t> cache;     // token ids from the start -> block
  std::map<int32_t, std::vector<int32_t>> entry_of;  // cached block -> its list of ids
  std::deque<int32_t> releasable;                    // cached, no holder; front leaves first
};

enum { ORC_OK = 0, ORC_INVALID = 1, ORC_OOM = 2, ORC_NOT_FOUND = 3 };

int64_t available(const Pool* p) {
  return static_cast<int64_t>(p->free_stack.size() + p->releasable.size());
}

int32_t take_block(Pool* p) {
  int32_t b;
  if (!p->free_stack.empty()) {
    b = p->free_stack.back();
    p->free_stack.pop_back();
  } else {
    b = p->releasable.front();
    p->releasable.pop_front();
    p->cache.erase(p->entry_of[b]);
    p->entry_of.erase(b);
  }
  p->holders[b] = 1;
  return b;
}

// A cached block found for a new sequence gains a holder (leaving the queue).
void hold_block(Pool* p, int32_t b) {
  if (p->holders[b] == 0) {
    p->releasable.erase(std::find(p->releasable.begin(), p->releasable.end(), b));
  }
  p->holders[b] += 1;
}

// Each block of `list` loses one holder; those left without one go to the
// free stack in list order, or, if cached, to the back of the queue in
// reverse list order.
template <typename List>
void release_blocks(Pool* p, const List& list) {
  std::vector<int32_t> emptied;
  for (int32_t b : list) {
    auto it = p->holders.find(b);
    it->second -= 1;
    if (it->second == 0) {
      p->holders.erase(it);
      if (p->entry_of.count(b)) {
        emptied.push_back(b);
      } else {
        p->free_stack.push_back(b);
      }
    }
  }
  for (auto r = emptied.rbegin(); r != emptied.rend(); ++r) p->releasable.push_back(*r);
}

void drop_block(Pool* p, int32_t b) { release_blocks(p, std::vector<int32_t>{b}); }

// Offer every full block of `s` not offered yet to the cache.
void offer_full_blocks(Pool* p, Sequence& s) {
  const int64_t bs = p->block_size;
  while (s.ids_known && (s.considered + 1) * bs <= s.len) {
    std::vector<int32_t> key(s.ids.begin(), s.ids.begin() + (s.considered + 1) * bs);
    if (p->prefix && !p->cache.count(key)) {
      const int32_t b = s.blocks[s.considered];
      p->cache[key] = b;
      p->entry_of[b] = key;
    }
    ++s.considered;
  }
}

int32_t holders_of(const Pool* p, int32_t b) {
  auto it = p->holders.find(b);
  return it == p->holders.end() ? 0 : it->second;
}

}  // namespace

extern "C" {

// ----------------------------- number formats ------------------------------
double orc_f16_to_f64(uint16_t h) { return f16_bits_to_double(h); }
double orc_bf16_to_f64(uint16_t b) { return bf16_bits_to_double(b); }
uint16_t orc_f64_to_f16(double x) { return double_to_f16_bits(x); }
uint16_t orc_f64_to_bf16(double x) { return double_to_bf16_bits(x); }

// Round an array of doubles to the storage dtype (1 = fp16, 2 = bf16, 0 = fp32).
void orc_round_array(const double* x, int64_t n, int dtype, void* out) {
  for (int64_t i = 0; i < n; ++i) {
    if (dtype == 0) {
      static_cast<float*>(out)[i] = static_cast<float>(x[i]);
    } else if (dtype == 1) {
      static_cast<uint16_t*>(out)[i] = double_to_f16_bits(x[i]);
    } else {
      static_cast<uint16_t*>(out)[i] = double_to_bf16_bits(x[i]);
    }
  }
}

// ------------------------------ KV size ------------------------------------
// [P5] "The precise scientific definition": the cache holds a key and a value
// (the factor 2) for every layer, token, KV head and head dimension, each of
// precision_bytes bytes.
uint64_t orc_kv_bytes(int32_t num_layers, int64_t seq_length, int32_t num_kv_heads,
                      int32_t head_dim, int32_t precision_bytes) {
  return 2ull * static_cast<uint64_t>(num_layers) * static_cast<uint64_t>(seq_length) *
         static_cast<uint64_t>(num_kv_heads) * static_cast<uint64_t>(head_dim) *
         static_cast<uint64_t>(precision_bytes);
}

// ------------------------------- pool model --------------------------------
void* orc_pool_new(int32_t num_blocks, int32_t block_size) {
  if (num_blocks < 0 || block_size <= 0) return nullptr;
  Pool* p = new Pool;
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  for (int32_t b = num_blocks - 1; b >= 0; --b) p->free_stack.push_back(b);  // 0 on top
  return p;
}

void orc_pool_delete(void* pool) { delete static_cast<Pool*>(pool); }

int32_t orc_num_free(const void* pool) {
  return static_cast<int32_t>(available(static_cast<const Pool*>(pool)));
}

int32_t orc_num_cached(const void* pool) {
  return static_cast<int32_t>(static_cast<const Pool*>(pool)->cache.size());
}

int32_t orc_num_releasable(const void* pool) {
  return static_cast<int32_t>(static_cast<const Pool*>(pool)->releasable.size());
}

void orc_set_prefix_caching(void* pool, int32_t enable) {
  Pool* p = static_cast<Pool*>(pool);
  p->prefix = enable != 0;
  if (p->prefix) return;
  while (!p->releasable.empty()) {
    p->free_stack.push_back(p->releasable.front());
    p->releasable.pop_front();
  }
  p->cache.clear();
  p->entry_of.clear();
}

int32_t orc_holders(const void* pool, int32_t block) {
  return holders_of(static_cast<const Pool*>(pool), block);
}

// Grow sequence `seq` by n tokens (creating it if absent).  Writes the slot of
// each new token (physical block * block_size + offset in block) and, when the
// shared partial last block had to be copied first, one (source, destination)
// pair.  All or nothing: on failure nothing changes.
int orc_alloc(void* pool, int64_t seq, int32_t n, int64_t* slots_out, int32_t* cow_pair_out,
              int32_t* n_cow_out) {
  Pool* p = static_cast<Pool*>(pool);
  if (n < 0) return ORC_INVALID;
  const int32_t bs = p->block_size;
  Sequence fresh_seq;
  auto it = p->seqs.find(seq);
  Sequence& s = (it == p->seqs.end()) ? fresh_seq : it->second;

  const int64_t used_in_last = s.len % bs;
  const int64_t room = used_in_last == 0 ? 0 : bs - used_in_last;
  const int64_t into_last = std::min<int64_t>(room, n);
  const bool must_copy = into_last > 0 && holders_of(p, s.blocks.back()) > 1;
  const int64_t new_blocks = (n - into_last + bs - 1) / bs;
  const int64_t needed = (must_copy ? 1 : 0) + new_blocks;
  if (needed > available(p)) return ORC_OOM;

  *n_cow_out = 0;
  if (n > 0) {
    s.ids_known = false;  // tokens without ids
    s.ids.clear();
  }
  if (must_copy) {
    const int32_t old_block = s.blocks.back();
    const int32_t new_block = take_block(p);
    drop_block(p, old_block);
    s.blocks.back() = new_block;
    cow_pair_out[0] = old_block;
    cow_pair_out[1] = new_block;
    *n_cow_out = 1;
  }
  for (int64_t k = 0; k < new_blocks; ++k) s.blocks.push_back(take_block(p));
  for (int32_t i = 0; i < n; ++i) {
    const int64_t pos = s.len + i;
    slots_out[i] = static_cast<int64_t>(s.blocks[pos / bs]) * bs + pos % bs;
  }
  s.len += n;
  if (it == p->seqs.end()) p->seqs.emplace(seq, s);
  return ORC_OK;
}

// Release every block of `seq` (in logical order) and forget the sequence.
int orc_free(void* pool, int64_t seq) {
  Pool* p = static_cast<Pool*>(pool);
  auto it = p->seqs.find(seq);
  if (it == p->seqs.end()) return ORC_NOT_FOUND;
  release_blocks(p, it->second.blocks);
  p->seqs.erase(it);
  return ORC_OK;
}

// orc_alloc with the new tokens' ids, and prefix-cache reuse for a sequence
// that holds no token yet.  Tokens served from the cache get slot -1; their
// count goes to *n_cached_out.  All or nothing.
int orc_alloc_tokens(void* pool, int64_t seq, const int32_t* ids, int32_t n, int64_t* slots_out,
                     int32_t* cow_pair_out, int32_t* n_cow_out, int32_t* n_cached_out) {
  Pool* p = static_cast<Pool*>(pool);
  if (n < 0) return ORC_INVALID;
  const int32_t bs = p->block_size;
  Sequence fresh_seq;
  auto it = p->seqs.find(seq);
  Sequence& s = (it == p->seqs.end()) ? fresh_seq : it->second;

  std::vector<int32_t> found;
  if (p->prefix && s.len == 0 && s.ids_known) {
    for (int64_t j = 0; (j + 1) * bs <= static_cast<int64_t>(n) - 1; ++j) {
      const std::vector<int32_t> key(ids, ids + (j + 1) * bs);
      auto c = p->cache.find(key);
      if (c == p->cache.end()) break;
      found.push_back(c->second);
    }
  }
  int64_t found_unheld = 0;
  for (int32_t b : found) found_unheld += holders_of(p, b) == 0 ? 1 : 0;
  const int64_t cached_tokens = static_cast<int64_t>(found.size()) * bs;
  const int64_t used_in_last = s.len % bs;
  const int64_t room = used_in_last == 0 ? 0 : bs - used_in_last;
  const int64_t into_last = std::min<int64_t>(room, n);
  const bool must_copy = into_last > 0 && holders_of(p, s.blocks.back()) > 1;
  const int64_t new_blocks = (n - cached_tokens - into_last + bs - 1) / bs;
  if ((must_copy ? 1 : 0) + new_blocks > available(p) - found_unheld) return ORC_OOM;

  for (int32_t b : found) {
    hold_block(p, b);
    s.blocks.push_back(b);
  }
  *n_cow_out = 0;
  if (must_copy) {
    const int32_t old_block = s.blocks.back();
    const int32_t new_block = take_block(p);
    drop_block(p, old_block);
    s.blocks.back() = new_block;
    cow_pair_out[0] = old_block;
    cow_pair_out[1] = new_block;
    *n_cow_out = 1;
  }
  for (int64_t k = 0; k < new_blocks; ++k) s.blocks.push_back(take_block(p));
  for (int32_t i = 0; i < n; ++i) {
    const int64_t pos = s.len + i;
    slots_out[i] = i < cached_tokens ? -1 : static_cast<int64_t>(s.blocks[pos / bs]) * bs + pos % bs;
  }
  s.len += n;
  if (s.ids_known) s.ids.insert(s.ids.end(), ids, ids + n);
  offer_full_blocks(p, s);
  *n_cached_out = static_cast<int32_t>(cached_tokens);
  if (it == p->seqs.end()) p->seqs.emplace(seq, s);
  return ORC_OK;
}

// `child` becomes a copy of `parent` that shares all of its physical blocks.
int orc_fork(void* pool, int64_t parent, int64_t child) {
  Pool* p = static_cast<Pool*>(pool);
  auto it = p->seqs.find(parent);
  if (it == p->seqs.end()) return ORC_NOT_FOUND;
  if (p->seqs.count(child)) return ORC_INVALID;
  Sequence copy = it->second;
  for (int32_t b : copy.blocks) p->holders[b] += 1;
  p->seqs.emplace(child, copy);
  return ORC_OK;
}

int64_t orc_seq_len(const void* pool, int64_t seq) {
  const Pool* p = static_cast<const Pool*>(pool);
  auto it = p->seqs.find(seq);
  return it == p->seqs.end() ? -1 : it->second.len;
}

// Block table rows (pad -1) and context lengths for a list of sequences.
int orc_block_table(const void* pool, const int64_t* seqs, int32_t n_seqs, int32_t max_blocks,
                    int32_t* table_out, int32_t* ctx_out) {
  const Pool* p = static_cast<const Pool*>(pool);
  for (int32_t i = 0; i < n_seqs; ++i) {
    auto it = p->seqs.find(seqs[i]);
    if (it == p->seqs.end()) return ORC_NOT_FOUND;
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks) return ORC_INVALID;
  }
  for (int32_t i = 0; i < n_seqs; ++i) {
    const Sequence& s = p->seqs.find(seqs[i])->second;
    for (int32_t j = 0; j < max_blocks; ++j) {
      table_out[static_cast<int64_t>(i) * max_blocks + j] =
          j < static_cast<int32_t>(s.blocks.size()) ? s.blocks[j] : -1;
    }
    ctx_out[i] = static_cast<int32_t>(s.len);
  }
  return ORC_OK;
}

// ------------------------------- swapping ----------------------------------
// [P2] "How PagedAttention solves this", fine-grained eviction: under memory
// pressure small pages move to the CPU instead of whole sequences staying or
// going.  Reading: a sequence is moved between a device pool and a host pool
// block by block: every block of the sequence gets a block in the other pool
// (in logical order), the sequence then lives in the other pool with the same
// length, and its old blocks lose one holder (a block shared with other
// sequences stays where it is for them).  All or nothing.  The (from, to)
// block pairs are what the caller copies.
int orc_swap(void* from_pool, void* to_pool, int64_t seq, int32_t* pairs_out, int32_t* n_out) {
  Pool* from = static_cast<Pool*>(from_pool);
  Pool* to = static_cast<Pool*>(to_pool);
  auto it = from->seqs.find(seq);
  if (it == from->seqs.end()) return ORC_NOT_FOUND;
  if (to->seqs.count(seq) || from->block_size != to->block_size) return ORC_INVALID;
  const Sequence old = it->second;
  if (static_cast<int64_t>(old.blocks.size()) > available(to)) return ORC_OOM;
  Sequence moved = old;  // length and ids move along; the new blocks are not cached
  moved.blocks.clear();
  int32_t k = 0;
  for (int32_t b : old.blocks) {
    const int32_t nb = take_block(to);
    moved.blocks.push_back(nb);
    pairs_out[2 * k] = b;
    pairs_out[2 * k + 1] = nb;
    ++k;
  }
  release_blocks(from, old.blocks);
  from->seqs.erase(seq);
  to->seqs.emplace(seq, moved);
  *n_out = k;
  return ORC_OK;
}

// Block copy between two pools (e.g. device -> host): for each pair, in order,
// block `to` of the destination caches becomes a byte copy of block `from` of
// the source caches, for every layer.
int orc_copy_between(void* const* dst_k, void* const* dst_v, void* const* src_k,
                     void* const* src_v, int32_t num_layers, const int32_t* pairs,
                     int32_t n_pairs, int64_t block_bytes) {
  for (int32_t i = 0; i < n_pairs; ++i) {
    const int64_t src = pairs[2 * i];
    const int64_t dst = pairs[2 * i + 1];
    for (int32_t l = 0; l < num_layers; ++l) {
      std::memcpy(static_cast<char*>(dst_k[l]) + dst * block_bytes,
                  static_cast<const char*>(src_k[l]) + src * block_bytes, block_bytes);
      std::memcpy(static_cast<char*>(dst_v[l]) + dst * block_bytes,
                  static_cast<const char*>(src_v[l]) + src * block_bytes, block_bytes);
    }
  }
  return ORC_OK;
}

// ----------------------------- cache write ---------------------------------
// Store each new token's key and value rows in the cache at its slot; slot -1
// means "no token" and is skipped.  Cache layout: [num_blocks, kv_heads,
// block_size, head_dim]; key/value layout: [n_tokens, kv_heads, head_dim].
// The copy is byte for byte.
int orc_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                          const int64_t* slots, int64_t n_tokens, int32_t kv_heads,
                          int32_t head_dim, int32_t block_size, int32_t num_blocks,
                          int32_t elem_bytes) {
  const int64_t row = static_cast<int64_t>(head_dim) * elem_bytes;
  for (int64_t t = 0; t < n_tokens; ++t) {
    const int64_t slot = slots[t];
    if (slot < 0) continue;
    if (slot >= static_cast<int64_t>(num_blocks) * block_size) return ORC_INVALID;
    const int64_t block = slot / block_size;
    const int64_t offset = slot % block_size;
    for (int32_t h = 0; h < kv_heads; ++h) {
      const int64_t dst = ((block * kv_heads + h) * block_size + offset) * row;
      const int64_t src = (t * kv_heads + h) * row;
      std::memcpy(static_cast<char*>(k_cache) + dst, static_cast<const char*>(key) + src, row);
      std::memcpy(static_cast<char*>(v_cache) + dst, static_cast<const char*>(value) + src, row);
    }
  }
  return ORC_OK;
}

// ----------------------------- block copy ----------------------------------
// Copy-on-write ([P2] "How PagedAttention solves this"): for each (src, dst)
// pair, in order, copy the whole key block and value block of every layer.
int orc_copy_blocks(void* const* k_caches, void* const* v_caches, int32_t num_layers,
                    const int32_t* pairs, int32_t n_pairs, int64_t block_bytes) {
  for (int32_t i = 0; i < n_pairs; ++i) {
    const int64_t src = pairs[2 * i];
    const int64_t dst = pairs[2 * i + 1];
    for (int32_t l = 0; l < num_layers; ++l) {
      std::memmove(static_cast<char*>(k_caches[l]) + dst * block_bytes,
                   static_cast<const char*>(k_caches[l]) + src * block_bytes, block_bytes);
      std::memmove(static_cast<char*>(v_caches[l]) + dst * block_bytes,
                   static_cast<const char*>(v_caches[l]) + src * block_bytes, block_bytes);
    }
  }
  return ORC_OK;
}

// ------------------------------ INT8 cache ---------------------------------
// "KV Cache for intermediates..." / "The four solutions", KV-cache quantisation:
// keys and values stored in 8 bits (about half the memory of fp16).  The pages
// fix no scheme; the reading taken here: per (token, kv head), symmetric over
// head_dim, with every step in IEEE fp32 so that the integer decisions are
// reproducible:  amax = max_d |x_d|,  scale = amax / 127,  code_d = round to
// nearest even of (x_d / scale), clamped to [-127, 127]; a zero row has scale 0
// and zero codes.  A value is read back as code * scale.
static void quantize_row(const void* src, int64_t base, int32_t D, int dtype, int8_t* codes,
                         float* scale_out) {
  float amax = 0.f;
  for (int32_t d = 0; d < D; ++d)
    amax = std::max(amax, std::fabs(static_cast<float>(load_elem(src, base + d, dtype))));
  const float scale = amax / 127.0f;
  for (int32_t d = 0; d < D; ++d) {
    int32_t c = 0;
    if (scale > 0.f) {
      const float x = static_cast<float>(load_elem(src, base + d, dtype));
      c = static_cast<int32_t>(std::nearbyint(x / scale));
      c = std::min(127, std::max(-127, c));
    }
    codes[d] = static_cast<int8_t>(c);
  }
  *scale_out = scale;
}

// Write new tokens into an INT8 cache, kept here in its logical layout: key
// codes and value codes [NB, Hkv, bs, D], scales [NB, Hkv, bs] (fp32) for each.
int orc_reshape_and_cache_int8(const void* key, const void* value, int8_t* k_codes,
                               int8_t* v_codes, float* k_scales, float* v_scales,
                               const int64_t* slots, int64_t n_tokens, int32_t kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t num_blocks,
                               int dtype) {
  const int32_t D = head_dim;
  std::vector<int8_t> row(D);
  for (int64_t t = 0; t < n_tokens; ++t) {
    const int64_t slot = slots[t];
    if (slot < 0) continue;
    if (slot >= static_cast<int64_t>(num_blocks) * block_size) return ORC_INVALID;
    const int64_t blk = slot / block_size, off = slot % block_size;
    for (int32_t h = 0; h < kv_heads; ++h) {
      const int64_t src = (t * kv_heads + h) * D;
      const int64_t tile = blk * kv_heads + h;
      float sc;
      quantize_row(key, src, D, dtype, row.data(), &sc);
      for (int32_t d = 0; d < D; ++d) k_codes[(tile * block_size + off) * D + d] = row[d];
      k_scales[tile * block_size + off] = sc;
      quantize_row(value, src, D, dtype, row.data(), &sc);
      for (int32_t d = 0; d < D; ++d) v_codes[(tile * block_size + off) * D + d] = row[d];
      v_scales[tile * block_size + off] = sc;
    }
  }
  return ORC_OK;
}

// Quantise rows [n, D] (tests): codes [n, D], scales [n].
void orc_quantize_rows(const void* x, int64_t n, int32_t D, int dtype, int8_t* codes,
                       float* scales) {
  for (int64_t i = 0; i < n; ++i) quantize_row(x, i * D, D, dtype, codes + i * D, scales + i);
}

// ------------------------------ attention ----------------------------------
// One new query per sequence attends to the cached keys and values of all of
// the sequence's tokens ([P5] "The precise scientific definition": a new token
// computes its Q while K and V of every earlier token must already be in
// memory).  The pages do not print the attention formula; the reading taken is
//   o = sum_j softmax_j(scale * q . k_j) v_j,   j < context length,
// with query head h reading KV head h / G, G = q_heads / kv_heads ([P5] "The
// four solutions", GQA: a group of query heads shares one K/V head; MQA and full
// multi-head attention are the cases kv_heads = 1 and G = 1).
//
// The core takes one query row and contiguous key/value rows of one KV head:
// it is the plain definition, with the maximum subtracted before exp.
static void attend_one(const double* q, const double* k, const double* v, int64_t n,
                       int32_t head_dim, double scale, double* out) {
  for (int32_t d = 0; d < head_dim; ++d) out[d] = 0.0;
  if (n == 0) return;  // reading: an empty context gives a zero output
  std::vector<double> s(n);
  for (int64_t j = 0; j < n; ++j) {
    double dot = 0.0;
    for (int32_t d = 0; d < head_dim; ++d) dot += q[d] * k[j * head_dim + d];
    s[j] = scale * dot;
  }
  double m = s[0];
  for (int64_t j = 1; j < n; ++j) m = std::max(m, s[j]);
  double den = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    s[j] = std::exp(s[j] - m);
    den += s[j];
  }
  for (int64_t j = 0; j < n; ++j) {
    for (int32_t d = 0; d < head_dim; ++d) out[d] += s[j] * v[j * head_dim + d];
  }
  for (int32_t d = 0; d < head_dim; ++d) out[d] /= den;
}

// Paged form: gather each sequence's keys and values through its block table
// into contiguous rows ([P1] "The scientific explanation": the block table maps
// the sequence's logical blocks to physical ones; token j lives in logical block
// j / block_size at offset j % block_size), then apply the definition above.
//
//   q          [batch, q_heads, head_dim]            dtype
//   k/v_cache  [num_blocks, kv_heads, block_size, head_dim]  dtype
//   tables     [batch, max_blocks] int32,  ctx [batch] int32
//   out        [batch, q_heads, head_dim] fp64
//   rows       optional list of n_rows flat (b * q_heads + h) indices to compute
//              (NULL = all); other outputs are left untouched.
struct PagedArgs {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* tables;
  const int32_t* ctx;
  int32_t batch, q_heads, kv_heads, head_dim, block_size, max_blocks;
  double scale;
  int dtype;
  double* out;
};

static void paged_row(const PagedArgs& a, int64_t row) {
  const int64_t b = row / a.q_heads;
  const int32_t h = static_cast<int32_t>(row % a.q_heads);
  const int32_t group = a.q_heads / a.kv_heads;
  const int32_t g = h / group;
  const int64_t n = a.ctx[b];
  const int32_t D = a.head_dim;
  std::vector<double> q(D), k(n * D), v(n * D);
  for (int32_t d = 0; d < D; ++d) q[d] = load_elem(a.q, (b * a.q_heads + h) * D + d, a.dtype);
  for (int64_t j = 0; j < n; ++j) {
    const int64_t phys = a.tables[b * a.max_blocks + j / a.block_size];
    const int64_t base = ((phys * a.kv_heads + g) * a.block_size + j % a.block_size) * D;
    for (int32_t d = 0; d < D; ++d) {
      k[j * D + d] = load_elem(a.k_cache, base + d, a.dtype);
      v[j * D + d] = load_elem(a.v_cache, base + d, a.dtype);
    }
  }
  attend_one(q.data(), k.data(), v.data(), n, D, a.scale, a.out + row * D);
}

int orc_paged_decode_attention(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* tables, const int32_t* ctx, int32_t batch,
                               int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                               int32_t block_size, int32_t max_blocks, double scale, int dtype,
                               double* out, const int64_t* rows, int64_t n_rows,
                               int32_t n_threads) {
  if (kv_heads <= 0 || q_heads % kv_heads != 0) return ORC_INVALID;
  PagedArgs a{q, k_cache, v_cache, tables, ctx, batch, q_heads, kv_heads,
              head_dim, block_size, max_blocks, scale, dtype, out};
  const int64_t total = rows ? n_rows : static_cast<int64_t>(batch) * q_heads;
  if (n_threads < 1) n_threads = 1;
  std::vector<std::thread> pool;
  for (int32_t t = 0; t < n_threads; ++t) {
    pool.emplace_back([&, t]() {
      for (int64_t i = t; i < total; i += n_threads) paged_row(a, rows ? rows[i] : i);
    });
  }
  for (auto& th : pool) th.join();
  return ORC_OK;
}

// Paged prefill (and chunked prefill) attention.  [P4] mentions serving the
// prompt phase over the same paged cache; the pages print no formula.
// Reading: sequence b has n_b = query_start[b + 1] - query_start[b] new tokens,
// the last n_b of its ctx[b] tokens (their keys and values already written);
// new token i sits at position p = ctx[b] - n_b + i and attends causally, to
// every token j <= p of the sequence:
//   out[query_start[b] + i, h] = sum_{j <= p} softmax_j(scale q . K_b[j, g]) V_b[j, g]
// with g = h / (q_heads / kv_heads).  A single new token (n_b = 1) is decode.
//   q, out  [total_q, q_heads, head_dim]   (out fp64)
//   query_start [batch + 1] int32 (non-decreasing, starts at 0)
// Only the listed rows (flat (token, head) indices) are computed when rows != NULL.
int orc_paged_prefill_attention(const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* tables, const int32_t* ctx,
                                const int32_t* query_start, int32_t batch, int32_t q_heads,
                                int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                int32_t max_blocks, double scale, int dtype, double* out,
                                const int64_t* rows, int64_t n_rows, int32_t n_threads) {
  if (kv_heads <= 0 || q_heads % kv_heads != 0) return ORC_INVALID;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t n_new = query_start[b + 1] - query_start[b];
    if (n_new < 0 || n_new > ctx[b]) return ORC_INVALID;
  }
  const int32_t group = q_heads / kv_heads, D = head_dim, bs = block_size;
  const int64_t total_q = query_start[batch];
  const int64_t total = rows ? n_rows : total_q * q_heads;
  auto one = [&](int64_t row) {
    const int64_t t = row / q_heads;
    const int32_t h = static_cast<int32_t>(row % q_heads);
    int32_t b = 0;
    while (query_start[b + 1] <= t) ++b;  // the sequence that owns token t
    const int64_t i = t - query_start[b];
    const int64_t n_new = query_start[b + 1] - query_start[b];
    const int64_t p = ctx[b] - n_new + i;  // position of the token
    const int32_t g = h / group;
    const int64_t n = p + 1;  // keys 0 .. p
    std::vector<double> qq(D), kk(n * D), vv(n * D);
    for (int32_t d = 0; d < D; ++d) qq[d] = load_elem(q, (t * q_heads + h) * D + d, dtype);
    for (int64_t j = 0; j < n; ++j) {
      const int64_t blk = tables[static_cast<int64_t>(b) * max_blocks + j / bs];
      const int64_t base = ((blk * kv_heads + g) * bs + j % bs) * D;
      for (int32_t d = 0; d < D; ++d) {
        kk[j * D + d] = load_elem(k_cache, base + d, dtype);
        vv[j * D + d] = load_elem(v_cache, base + d, dtype);
      }
    }
    attend_one(qq.data(), kk.data(), vv.data(), n, D, scale, out + row * D);
  };
  if (n_threads < 1) n_threads = 1;
  std::vector<std::thread> pool;
  for (int32_t th = 0; th < n_threads; ++th) {
    pool.emplace_back([&, th]() {
      for (int64_t k = th; k < total; k += n_threads) one(rows ? rows[k] : k);
    });
  }
  for (auto& x : pool) x.join();
  return ORC_OK;
}

// Paged attention over an INT8 cache: the gather reads code * scale (exact in
// fp64), then the same definition as above.  q / out as in the paged form.
int orc_paged_decode_attention_int8(const void* q, const int8_t* k_codes, const int8_t* v_codes,
                                    const float* k_scales, const float* v_scales,
                                    const int32_t* tables, const int32_t* ctx, int32_t batch,
                                    int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                                    int32_t block_size, int32_t max_blocks, double scale,
                                    int dtype, double* out, const int64_t* rows, int64_t n_rows,
                                    int32_t n_threads) {
  if (kv_heads <= 0 || q_heads % kv_heads != 0) return ORC_INVALID;
  const int32_t group = q_heads / kv_heads, D = head_dim, bs = block_size;
  const int64_t total = rows ? n_rows : static_cast<int64_t>(batch) * q_heads;
  auto one = [&](int64_t row) {
    const int64_t b = row / q_heads;
    const int32_t h = static_cast<int32_t>(row % q_heads);
    const int32_t g = h / group;
    const int64_t n = ctx[b];
    std::vector<double> qq(D), kk(n * D), vv(n * D);
    for (int32_t d = 0; d < D; ++d) qq[d] = load_elem(q, (b * q_heads + h) * D + d, dtype);
    for (int64_t j = 0; j < n; ++j) {
      const int64_t tile = static_cast<int64_t>(tables[b * max_blocks + j / bs]) * kv_heads + g;
      const int64_t off = j % bs;
      const double ks = k_scales[tile * bs + off], vs = v_scales[tile * bs + off];
      for (int32_t d = 0; d < D; ++d) {
        kk[j * D + d] = ks * k_codes[(tile * bs + off) * D + d];
        vv[j * D + d] = vs * v_codes[(tile * bs + off) * D + d];
      }
    }
    attend_one(qq.data(), kk.data(), vv.data(), n, D, scale, out + row * D);
  };
  if (n_threads < 1) n_threads = 1;
  std::vector<std::thread> pool;
  for (int32_t t = 0; t < n_threads; ++t)
    pool.emplace_back([&, t]() {
      for (int64_t i = t; i < total; i += n_threads) one(rows ? rows[i] : i);
    });
  for (auto& th : pool) th.join();
  return ORC_OK;
}

// Contiguous form, used where a sequence's keys and values are already laid
// out in logical order: q [q_heads, head_dim], k/v [n, kv_heads, head_dim]
// (dtype), out [q_heads, head_dim] fp64.  Only the listed query heads are
// computed (heads = NULL: all).
int orc_contiguous_attention(const void* q, const void* k, const void* v, int64_t n,
                             int32_t q_heads, int32_t kv_heads, int32_t head_dim, double scale,
                             int dtype, double* out, const int32_t* heads, int32_t n_heads) {
  if (kv_heads <= 0 || q_heads % kv_heads != 0) return ORC_INVALID;
  const int32_t group = q_heads / kv_heads;
  const int32_t D = head_dim;
  const int32_t count = heads ? n_heads : q_heads;
  std::vector<double> qq(D), kk(n * D), vv(n * D);
  for (int32_t i = 0; i < count; ++i) {
    const int32_t h = heads ? heads[i] : i;
    const int32_t g = h / group;
    for (int32_t d = 0; d < D; ++d) qq[d] = load_elem(q, static_cast<int64_t>(h) * D + d, dtype);
    for (int64_t j = 0; j < n; ++j) {
      for (int32_t d = 0; d < D; ++d) {
        kk[j * D + d] = load_elem(k, (j * kv_heads + g) * D + d, dtype);
        vv[j * D + d] = load_elem(v, (j * kv_heads + g) * D + d, dtype);
      }
    }
    attend_one(qq.data(), kk.data(), vv.data(), n, D, scale, out + static_cast<int64_t>(h) * D);
  }
  return ORC_OK;
}

// Host threads the C++ runtime reports (std::thread::hardware_concurrency; 0 if
// unknown): the core count printed beside the oracle's timings.
int32_t orc_hardware_concurrency(void) {
  return static_cast<int32_t>(std::thread::hardware_concurrency());
}

}  // extern "C"
