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
// Free blocks are handed out first-in first-out, so the state after a call
// sequence is a deterministic function of the calls.  Each call either does
// all of its work or leaves the state as it was.
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pa.h"

namespace {

struct Seq {
  std::vector<int32_t> blocks;  // physical ids, logical order
  int64_t n_tokens = 0;
};

}  // namespace

struct pa_alloc {
  int num_blocks = 0;
  int block_size = 16;
  std::deque<int32_t> free_q;
  std::vector<int32_t> rc;
  std::unordered_map<int64_t, Seq> seqs;
};

extern "C" {

pa_alloc* pa_alloc_create(int num_blocks, int block_size, const int32_t* order) {
  if (num_blocks < 1 || block_size != 16) return nullptr;
  pa_alloc* a = new (std::nothrow) pa_alloc;
  if (!a) return nullptr;
  a->num_blocks = num_blocks;
  a->block_size = block_size;
  a->rc.assign(num_blocks, 0);
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

pa_status pa_alloc_append(pa_alloc* a, int64_t seq, int n_tokens, int64_t* slots_out) {
  if (!a || n_tokens < 0 || (n_tokens > 0 && !slots_out)) return PA_ERR_INVALID_ARG;
  const int64_t B = a->block_size;
  auto it = a->seqs.find(seq);
  const int64_t n = (it == a->seqs.end()) ? 0 : it->second.n_tokens;
  if (it != a->seqs.end() && n_tokens > 0 && n % B != 0 &&
      a->rc[it->second.blocks.back()] > 1)
    return PA_ERR_INVALID_ARG;  // shared partial block: copy-on-write first
  const int64_t have = (n + B - 1) / B;
  const int64_t need = (n + n_tokens + B - 1) / B - have;
  if (need > (int64_t)a->free_q.size()) return PA_ERR_OOM;
  Seq& s = a->seqs[seq];  // creates the sequence on first use
  for (int64_t i = 0; i < need; i++) {
    int32_t b = a->free_q.front();
    a->free_q.pop_front();
    a->rc[b] = 1;
    s.blocks.push_back(b);
  }
  for (int64_t p = n; p < n + n_tokens; p++)
    slots_out[p - n] = (int64_t)s.blocks[p / B] * B + p % B;
  s.n_tokens = n + n_tokens;
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
  if (a->free_q.empty()) return PA_ERR_OOM;
  int32_t old_b = s.blocks.back();
  int32_t new_b = a->free_q.front();
  a->free_q.pop_front();
  a->rc[new_b] = 1;
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
  for (int32_t b : it->second.blocks) {
    if (--a->rc[b] == 0) a->free_q.push_back(b);
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

int pa_alloc_num_seqs(const pa_alloc* a) { return a ? (int)a->seqs.size() : -1; }

}  // extern "C"
