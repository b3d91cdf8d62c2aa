// Host block allocator: the memory-management layer of paged attention.
//
// Fixed 16-token blocks, one block table per sequence, a new block only when
// the last one is full, release when a request finishes ("vLLM explained",
// "PagedAttention：用分頁管理 KV cache" items 1-4 and "兩層實作"); sharing by
// reference count with copy-on-write of a block a branch is about to write
// ("LLM inference optimization: KV cache & PagedAttention", §三.2); a block
// whose count is above zero is never handed out ("vLLM explained",
// "KV cache 什麼時候可以被覆蓋").
//
// Prefix caching ("vLLM explained", "Prefix Caching：相同前綴只算一次"), off
// unless switched on: a block is in use (count > 0), free and empty, or free
// but holding cached content (count 0, content kept).  A full block whose
// token ids are known is registered under a hash of its whole prefix (the
// chain of the previous block's hash and its own 16 tokens; a hit is also
// checked against the stored tokens and parent hash).  pa_alloc_admit reuses
// the longest run of leading full blocks held by a block in use or cached,
// so their prefill can be skipped.  New blocks come from the empty blocks
// first and only then from the cached ones, least recently released first;
// blocks in use are never taken.  A finished request's registered blocks
// whose count reaches zero become cached, released from the sequence's last
// block to its first (of blocks released together the prefix's tail goes
// first).  A second block with an already registered prefix stays
// unregistered; a partial last block is never registered.
//
// Free blocks are handed out first-in first-out, so the state after a call
// sequence is a deterministic function of the calls.  Each call either does
// all of its work or leaves the state as it was.
#include <cstdint>
#include <cstring>
#include <deque>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pa.h"

namespace {

constexpr int kB = 16;  // tokens per block

struct Seq {
  std::vector<int32_t> blocks;  // physical ids, logical order
  int64_t n_tokens = 0;
  bool known = true;             // every token id of the sequence is known
  std::vector<int32_t> tokens;   // the ids, while known
  std::vector<uint64_t> hchain;  // prefix hash of each full block, while known
};

// 64-bit mix (the splitmix64 finaliser)
uint64_t mix(uint64_t x) {
  x ^= x >> 30;
  x *= 0xbf58476d1ce4e5b9ull;
  x ^= x >> 27;
  x *= 0x94d049bb133111ebull;
  return x ^ (x >> 31);
}

// hash of a block's whole prefix: the previous block's prefix hash chained
// with this block's 16 token ids
uint64_t block_hash(uint64_t parent, const int32_t* toks) {
  uint64_t h = mix(parent ^ 0x9e3779b97f4a7c15ull);
  for (int i = 0; i < kB; i++) h = mix(h ^ (uint64_t)(uint32_t)toks[i] ^ ((uint64_t)i << 32));
  return h;
}

}  // namespace

struct pa_alloc {
  int num_blocks = 0;
  int block_size = kB;
  std::deque<int32_t> free_q;  // empty free blocks, FIFO
  std::vector<int32_t> rc;
  std::unordered_map<int64_t, Seq> seqs;
  // prefix caching
  bool pc = false;
  std::vector<char> reg;                      // block registered
  std::vector<uint64_t> bhash, bparent;       // its prefix hash, its parent's
  std::vector<int32_t> btok;                  // its 16 token ids
  std::unordered_map<uint64_t, int32_t> holder;  // prefix hash -> registered block
  std::list<int32_t> lru;                     // cached free blocks, least recent first
  std::vector<std::list<int32_t>::iterator> lru_pos;

  size_t allocatable() const { return free_q.size() + lru.size(); }

  void unregister(int32_t b) {
    auto it = holder.find(bhash[b]);
    if (it != holder.end() && it->second == b) holder.erase(it);
    reg[b] = 0;
  }

  // an empty block if there is one, else the least recently released cached
  // block (its content forgotten); the caller checked allocatable() first
  int32_t take() {
    int32_t b;
    if (!free_q.empty()) {
      b = free_q.front();
      free_q.pop_front();
    } else {
      b = lru.front();
      lru.pop_front();
      unregister(b);
    }
    rc[b] = 1;
    return b;
  }

  // the registered block holding this prefix, or -1
  int32_t lookup(uint64_t h, uint64_t parent, const int32_t* toks) const {
    auto it = holder.find(h);
    if (it == holder.end()) return -1;
    const int32_t b = it->second;
    if (bparent[b] != parent || std::memcmp(&btok[(size_t)b * kB], toks, kB * sizeof(int32_t)))
      return -1;
    return b;
  }

  // extend the sequence's hash chain over its full blocks and register the
  // ones from index `from` on (known tokens, prefix caching on)
  void register_full(Seq& s, size_t from) {
    if (!s.known) return;
    const size_t full = (size_t)(s.n_tokens / kB);
    while (s.hchain.size() < full) {
      const size_t i = s.hchain.size();
      s.hchain.push_back(block_hash(i ? s.hchain[i - 1] : 0, &s.tokens[i * kB]));
    }
    if (!pc) return;
    for (size_t i = from; i < full; i++) {
      const int32_t b = s.blocks[i];
      const uint64_t h = s.hchain[i];
      if (reg[b] || holder.count(h)) continue;  // registered already, or a duplicate
      reg[b] = 1;
      bhash[b] = h;
      bparent[b] = i ? s.hchain[i - 1] : 0;
      std::memcpy(&btok[(size_t)b * kB], &s.tokens[i * kB], kB * sizeof(int32_t));
      holder[h] = b;
    }
  }

  // reserve slots for n new tokens of seq (creating it), all-or-nothing
  pa_status append(int64_t seq, int n_tokens, int64_t* slots_out) {
    const int64_t B = block_size;
    auto it = seqs.find(seq);
    const int64_t n = (it == seqs.end()) ? 0 : it->second.n_tokens;
    if (it != seqs.end() && n_tokens > 0 && n % B != 0 && rc[it->second.blocks.back()] > 1)
      return PA_ERR_INVALID_ARG;  // shared partial block: copy-on-write first
    const int64_t have = (n + B - 1) / B;
    const int64_t need = (n + n_tokens + B - 1) / B - have;
    if (need > (int64_t)allocatable()) return PA_ERR_OOM;
    Seq& s = seqs[seq];  // creates the sequence on first use
    for (int64_t i = 0; i < need; i++) s.blocks.push_back(take());
    for (int64_t p = n; p < n + n_tokens; p++)
      slots_out[p - n] = (int64_t)s.blocks[p / B] * B + p % B;
    s.n_tokens = n + n_tokens;
    return PA_OK;
  }
};

extern "C" {

pa_alloc* pa_alloc_create(int num_blocks, int block_size, const int32_t* order) {
  if (num_blocks < 1 || block_size != kB) return nullptr;
  pa_alloc* a = new (std::nothrow) pa_alloc;
  if (!a) return nullptr;
  try {
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->rc.assign(num_blocks, 0);
    a->reg.assign(num_blocks, 0);
    a->bhash.assign(num_blocks, 0);
    a->bparent.assign(num_blocks, 0);
    a->btok.assign((size_t)num_blocks * kB, 0);
    a->lru_pos.resize(num_blocks);
  } catch (...) {
    delete a;
    return nullptr;
  }
  if (order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; i++) {
      int32_t b = order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete a;
        return nullptr;
      }
      seen[b] = 1;
      a->free_q.push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; i++) a->free_q.push_back(i);
  }
  return a;
}

void pa_alloc_destroy(pa_alloc* a) { delete a; }

pa_status pa_alloc_set_prefix_caching(pa_alloc* a, int on) {
  if (!a || !a->seqs.empty()) return PA_ERR_INVALID_ARG;
  a->pc = on != 0;
  return PA_OK;
}

pa_status pa_alloc_append(pa_alloc* a, int64_t seq, int n_tokens, int64_t* slots_out) {
  if (!a || n_tokens < 0 || (n_tokens > 0 && !slots_out)) return PA_ERR_INVALID_ARG;
  const bool is_new = !a->seqs.count(seq);
  pa_status st = a->append(seq, n_tokens, slots_out);
  if (st != PA_OK) return st;
  Seq& s = a->seqs[seq];
  if (n_tokens > 0 || is_new) {  // tokens without ids: no longer known
    s.known = false;
    s.tokens.clear();
    s.hchain.clear();
  }
  return PA_OK;
}

pa_status pa_alloc_append_tokens(pa_alloc* a, int64_t seq, const int32_t* tokens, int n_tokens,
                                 int64_t* slots_out) {
  if (!a || n_tokens < 0 || (n_tokens > 0 && (!slots_out || !tokens)))
    return PA_ERR_INVALID_ARG;
  const int64_t n0 = a->seqs.count(seq) ? a->seqs[seq].n_tokens : 0;
  pa_status st = a->append(seq, n_tokens, slots_out);
  if (st != PA_OK) return st;
  Seq& s = a->seqs[seq];
  if (s.known) {
    s.tokens.insert(s.tokens.end(), tokens, tokens + n_tokens);
    a->register_full(s, (size_t)(n0 / kB));
  }
  return PA_OK;
}

pa_status pa_alloc_admit(pa_alloc* a, int64_t seq, const int32_t* tokens, int n_tokens,
                         int64_t* slots_out, int* n_cached_out) {
  if (!a || n_tokens < 0 || !n_cached_out || (n_tokens > 0 && (!slots_out || !tokens)))
    return PA_ERR_INVALID_ARG;
  if (a->seqs.count(seq)) return PA_ERR_INVALID_ARG;
  std::vector<int32_t> hits;
  std::vector<uint64_t> hashes;
  if (a->pc) {
    uint64_t parent = 0;
    for (int i = 0; (i + 1) * kB <= n_tokens; i++) {
      const uint64_t h = block_hash(parent, tokens + (size_t)i * kB);
      const int32_t b = a->lookup(h, parent, tokens + (size_t)i * kB);
      if (b < 0) break;
      hits.push_back(b);
      hashes.push_back(h);
      parent = h;
    }
  }
  size_t revived = 0;
  for (int32_t b : hits) revived += a->rc[b] == 0;
  const int64_t need = ((int64_t)n_tokens + kB - 1) / kB - (int64_t)hits.size();
  if (need > (int64_t)(a->allocatable() - revived)) return PA_ERR_OOM;
  Seq s;
  for (int32_t b : hits) {
    if (a->rc[b] == 0) a->lru.erase(a->lru_pos[b]);
    a->rc[b] += 1;
    s.blocks.push_back(b);
  }
  for (int64_t i = 0; i < need; i++) s.blocks.push_back(a->take());
  s.n_tokens = n_tokens;
  s.tokens.assign(tokens, tokens + n_tokens);
  s.hchain = hashes;
  Seq& ins = a->seqs.emplace(seq, std::move(s)).first->second;
  a->register_full(ins, hits.size());
  for (int p = 0; p < n_tokens; p++)
    slots_out[p] = (int64_t)ins.blocks[p / kB] * kB + p % kB;
  *n_cached_out = (int)hits.size() * kB;
  return PA_OK;
}

pa_status pa_alloc_fork(pa_alloc* a, int64_t parent, int64_t child) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->seqs.count(child)) return PA_ERR_INVALID_ARG;
  Seq c = it->second;
  for (int32_t b : c.blocks) a->rc[b] += 1;
  a->seqs.emplace(child, std::move(c));
  return PA_OK;
}

pa_status pa_alloc_prepare_write(pa_alloc* a, int64_t seq, int64_t* pairs, int* n_pairs) {
  if (!a || !n_pairs) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
  Seq& s = it->second;
  *n_pairs = 0;
  if (s.n_tokens % a->block_size == 0 || a->rc[s.blocks.back()] <= 1) return PA_OK;
  if (!pairs) return PA_ERR_INVALID_ARG;
  if (a->allocatable() == 0) return PA_ERR_OOM;
  int32_t old_b = s.blocks.back();
  int32_t new_b = a->take();
  a->rc[old_b] -= 1;
  s.blocks.back() = new_b;
  pairs[0] = old_b;
  pairs[1] = new_b;
  *n_pairs = 1;
  return PA_OK;
}

pa_status pa_alloc_free_seq(pa_alloc* a, int64_t seq) {
  if (!a) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
  const auto& bl = it->second.blocks;
  for (size_t k = bl.size(); k-- > 0;) {  // last block first
    const int32_t b = bl[k];
    if (--a->rc[b] == 0) {
      if (a->reg[b]) {
        a->lru.push_back(b);
        a->lru_pos[b] = std::prev(a->lru.end());
      } else {
        a->free_q.push_back(b);
      }
    }
  }
  a->seqs.erase(it);
  return PA_OK;
}

pa_status pa_alloc_block_table(const pa_alloc* a, int64_t seq, int32_t* out, int cap,
                               int* n_out) {
  if (!a || !n_out) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq);
  if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
  const auto& bl = it->second.blocks;
  *n_out = (int)bl.size();
  if ((int)bl.size() > cap || (!out && !bl.empty())) return PA_ERR_INVALID_ARG;
  for (size_t i = 0; i < bl.size(); i++) out[i] = bl[i];
  return PA_OK;
}

pa_status pa_alloc_free_list(const pa_alloc* a, int32_t* out, int cap, int* n_out) {
  if (!a || !n_out) return PA_ERR_INVALID_ARG;
  *n_out = (int)a->free_q.size();
  if ((int)a->free_q.size() > cap || (!out && !a->free_q.empty())) return PA_ERR_INVALID_ARG;
  int i = 0;
  for (int32_t b : a->free_q) out[i++] = b;
  return PA_OK;
}

pa_status pa_alloc_cached_list(const pa_alloc* a, int32_t* out, int cap, int* n_out) {
  if (!a || !n_out) return PA_ERR_INVALID_ARG;
  *n_out = (int)a->lru.size();
  if ((int)a->lru.size() > cap || (!out && !a->lru.empty())) return PA_ERR_INVALID_ARG;
  int i = 0;
  for (int32_t b : a->lru) out[i++] = b;
  return PA_OK;
}

int pa_alloc_num_tokens(const pa_alloc* a, int64_t seq) {
  if (!a) return -1;
  auto it = a->seqs.find(seq);
  return it == a->seqs.end() ? -1 : (int)it->second.n_tokens;
}

int pa_alloc_refcount(const pa_alloc* a, int32_t block) {
  if (!a || block < 0 || block >= a->num_blocks) return -1;
  return a->rc[block];
}

int pa_alloc_num_free(const pa_alloc* a) { return a ? (int)a->free_q.size() : -1; }

int pa_alloc_num_cached(const pa_alloc* a) { return a ? (int)a->lru.size() : -1; }

int pa_alloc_num_seqs(const pa_alloc* a) { return a ? (int)a->seqs.size() : -1; }

}  // extern "C"
