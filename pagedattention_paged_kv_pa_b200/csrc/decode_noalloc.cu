// pa_decode_noalloc: decode attention for callers that cannot allocate device
// memory.
//
// pa_decode needs a workspace for its per-partition results and leaves it to
// the caller to provide one.  Some callers cannot: a host program whose
// device memory is owned by someone else (a framework plugin that may not
// call cudaMalloc after start-up), or a loop that must not pay for
// cudaMalloc's implicit device synchronisation and has no buffer of its own
// to lend.  This entry point runs the same two kernels as pa_decode, but on
// a scratch area that is part of the library itself: a file-scope
// __device__ array of kNoAllocScratchBytes.  Every GPU that loads the library
// holds that array until the process exits.
//
// The array's name in host code is only a host-side stand-in, not a device
// address, so the address the kernels get comes from cudaGetSymbolAddress.
// The address belongs to the CUDA context the lookup ran in (the device's
// primary context for ordinary runtime users, or a driver-API context a
// plugin made current), so it is looked up on the first call made with a
// given context current and cached under that context's id
// (cuCtxGetCurrent / cuCtxGetId).  A context created later -- after a
// cudaDeviceReset, say -- has a new id and gets a fresh lookup.  Calls share
// the one array: two calls whose work overlaps on the GPU (different streams,
// or different host threads) race on it and must be ordered by the caller.
// Nothing in the scratch has to start at zero -- every value the merge kernel
// reads is written earlier in the same call -- so it is never cleared.
#include <mutex>
#include <utility>
#include <vector>

#include "pa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

// Id of the context current on this thread; 0 when there is none (or the
// driver cannot say).
unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  return get_id(c, &id) == CUDA_SUCCESS ? id : 0;
}

std::mutex g_mu;
std::vector<std::pair<unsigned long long, void*>> g_scratch_by_context;  // (context id, address)

// Device address of the scratch array in the context current on this thread.
pa_status scratch_for_current_context(void** out) {
  unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (id != 0)
    for (const auto& e : g_scratch_by_context)
      if (e.first == id) {
        *out = e.second;
        return PA_OK;
      }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
  // the lookup makes the device's primary context current if none was
  if (id == 0) id = current_context_id();
  if (id != 0) {
    if (g_scratch_by_context.size() >= 64) g_scratch_by_context.erase(g_scratch_by_context.begin());
    g_scratch_by_context.emplace_back(id, p);
  }
  *out = p;
  return PA_OK;
}

}  // namespace

extern "C" {

size_t pa_decode_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

pa_status pa_decode_noalloc(void* out, const void* q, const void* k_pool, const void* v_pool,
                            const int32_t* block_tables, const int32_t* context_lens,
                            float scale, int block_size, int n_q_heads, int n_kv_heads,
                            int head_dim, int num_seqs, int max_blocks_per_seq, int num_blocks,
                            pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
                            int32_t* dev_err, void* stream) {
  const size_t need =
      pa_decode_workspace_size(num_seqs, n_q_heads, head_dim, max_blocks_per_seq);
  if (need > kNoAllocScratchBytes) return PA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0) {
    pa_status st = scratch_for_current_context(&scratch);
    if (st != PA_OK) return st;
  }
  return pa_decode(out, q, k_pool, v_pool, block_tables, context_lens, scale, block_size,
                   n_q_heads, n_kv_heads, head_dim, num_seqs, max_blocks_per_seq, num_blocks,
                   q_dtype, kv_dtype, k_scale, v_scale, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                   dev_err, stream);
}

}  // extern "C"
