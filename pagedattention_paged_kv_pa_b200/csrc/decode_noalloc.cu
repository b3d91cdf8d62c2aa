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
// address, so the address the kernels get comes from cudaGetSymbolAddress,
// looked up once per device (on the first call made with that device
// current) and cached.  Calls share the one array: two calls whose work
// overlaps on the GPU (different streams, or different host threads) race on
// it and must be ordered by the caller.  Nothing in the scratch has to start
// at zero -- every value the merge kernel reads is written earlier in the same
// call -- so it is never cleared.
#include <mutex>

#include "pa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
pa_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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
    pa_status st = scratch_for_current_device(&scratch);
    if (st != PA_OK) return st;
  }
  return pa_decode(out, q, k_pool, v_pool, block_tables, context_lens, scale, block_size,
                   n_q_heads, n_kv_heads, head_dim, num_seqs, max_blocks_per_seq, num_blocks,
                   q_dtype, kv_dtype, k_scale, v_scale, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                   dev_err, stream);
}

}  // extern "C"
