// Slot write (reshape_and_cache) and copy-on-write block copy (copy_blocks).
//
// Both are pure data movement bound by HBM bandwidth and, at one decode step's
// sizes, by launch latency.  Threads move 16-byte chunks, consecutive threads
// take consecutive chunks of a row, so loads and stores are coalesced.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

// One thread per 16-byte chunk of a source row.  Index order, fastest first:
// chunk, kv head, token, K-or-V.  A token's slot names block slot/16 and row
// slot%16 of that block's tile for every kv head ("vLLM explained",
// "PagedAttention" items 1-4).
template <typename SrcT, bool TO_FP8>
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const ScatterParams p) {
  // the attention kernel that follows may start its set-up now; it waits for
  // this grid before it reads the cache
  pdl_launch_dependents();
  constexpr int EPC = 16 / sizeof(SrcT);  // source elements per chunk
  const int cpr = p.head_dim / EPC;       // chunks per row
  const int64_t per_kv = (int64_t)p.num_tokens * p.n_kv * cpr;
  const int64_t total = 2 * per_kv;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const bool is_v = i >= per_kv;
    const int64_t r = is_v ? i - per_kv : i;
    const int c = (int)(r % cpr);
    const int h = (int)((r / cpr) % p.n_kv);
    const int64_t t = r / ((int64_t)cpr * p.n_kv);
    const int64_t slot = p.slot_mapping[t];
    if (slot < 0) continue;
    const int64_t blk = slot >> 4, off = slot & 15;
    if (blk >= p.num_blocks) {
      if (c == 0 && h == 0 && !is_v) flag_error(p.dev_err, PA_DEVERR_SLOT);
      continue;
    }
    const SrcT* src = reinterpret_cast<const SrcT*>(is_v ? p.value : p.key) +
                      (t * p.n_kv + h) * p.head_dim + c * EPC;
    const int64_t dst_elem = ((blk * p.n_kv + h) * 16 + off) * p.head_dim + (int64_t)c * EPC;
    const uint4 raw = *reinterpret_cast<const uint4*>(src);
    if constexpr (!TO_FP8) {
      SrcT* dst = reinterpret_cast<SrcT*>(is_v ? p.v_pool : p.k_pool) + dst_elem;
      *reinterpret_cast<uint4*>(dst) = raw;
    } else {
      const float sc = is_v ? p.v_scale : p.k_scale;
      const SrcT* e = reinterpret_cast<const SrcT*>(&raw);
      uint8_t* dst = reinterpret_cast<uint8_t*>(is_v ? p.v_pool : p.k_pool) + dst_elem;
      uint16_t pk[EPC / 2];
#pragma unroll
      for (int k = 0; k < EPC / 2; ++k) {
        float a, b;
        if constexpr (sizeof(SrcT) == 4) {
          a = e[2 * k];
          b = e[2 * k + 1];
        } else if constexpr (std::is_same<SrcT, __nv_bfloat16>::value) {
          a = __bfloat162float(e[2 * k]);
          b = __bfloat162float(e[2 * k + 1]);
        } else {
          a = __half2float(e[2 * k]);
          b = __half2float(e[2 * k + 1]);
        }
        // quotient in binary32 (IEEE division), then E4M3 nearest-even, saturating
        pk[k] = __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(a, sc), __fdiv_rn(b, sc)),
                                         __NV_SATFINITE, __NV_E4M3);
      }
      if constexpr (EPC == 8) {
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(pk[0] | ((uint32_t)pk[1] << 16), pk[2] | ((uint32_t)pk[3] << 16));
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pk[0] | ((uint32_t)pk[1] << 16);
      }
    }
  }
}

// grid = (pairs, K-or-V, 16 KiB piece of the block); 256 threads x 4 x 16 B,
// the x dimension striding over the pairs.  Either pool may be pinned host
// memory mapped into the device address space (swapping); its bytes then
// cross the host link in 512-byte warp-wide requests.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyParams p) {
  const uint8_t* spool = reinterpret_cast<const uint8_t*>(blockIdx.y ? p.src_v : p.src_k);
  uint8_t* dpool = reinterpret_cast<uint8_t*>(blockIdx.y ? p.dst_v : p.dst_k);
  const int64_t n16 = p.block_bytes / 16;
  const int64_t lo = (int64_t)blockIdx.z * 1024;
  const int64_t hi = lo + 1024 < n16 ? lo + 1024 : n16;
  for (int pair = blockIdx.x; pair < p.n_pairs; pair += gridDim.x) {
    const int64_t s = p.pairs[2 * pair], d = p.pairs[2 * pair + 1];
    if (s < 0 || s >= p.src_num_blocks || d < 0 || d >= p.dst_num_blocks) {
      if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
        flag_error(p.dev_err, PA_DEVERR_SLOT);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(spool + s * p.block_bytes);
    uint4* dst = reinterpret_cast<uint4*>(dpool + d * p.block_bytes);
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t idx = lo + threadIdx.x + 256 * k;
      if (idx < hi) v[k] = src[idx];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t idx = lo + threadIdx.x + 256 * k;
      if (idx < hi) dst[idx] = v[k];
    }
  }
}

template <typename SrcT, bool FP8>
cudaError_t launch_rc(const ScatterParams& p, cudaStream_t st) {
  const int64_t total = 2ll * p.num_tokens * p.n_kv * (p.head_dim * (int)sizeof(SrcT) / 16);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks == 0) return cudaSuccess;
  reshape_and_cache_kernel<SrcT, FP8><<<(unsigned)blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_reshape_and_cache(const ScatterParams& p, pa_dtype src_dt, pa_dtype cache_dt,
                                     cudaStream_t st) {
  const bool fp8 = cache_dt == PA_FP8_E4M3;
  switch (src_dt) {
    case PA_F32: return fp8 ? launch_rc<float, true>(p, st) : launch_rc<float, false>(p, st);
    case PA_F16: return fp8 ? launch_rc<__half, true>(p, st) : launch_rc<__half, false>(p, st);
    case PA_BF16:
      return fp8 ? launch_rc<__nv_bfloat16, true>(p, st) : launch_rc<__nv_bfloat16, false>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_copy_blocks(const CopyParams& p, cudaStream_t st) {
  if (p.n_pairs == 0) return cudaSuccess;
  const int64_t n16 = p.block_bytes / 16;
  dim3 grid(p.n_pairs < 65535 ? p.n_pairs : 65535, 2, (unsigned)((n16 + 1023) / 1024));
  copy_blocks_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace pa
