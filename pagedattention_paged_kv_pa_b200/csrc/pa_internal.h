// Internal interfaces between the C ABI shim (capi.cu) and the kernel
// launchers.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/pa.h"

namespace pa {

// Tokens per decode context partition (32 blocks of 16).
constexpr int kPart = 512;

struct DecodeParams {
  void* out;
  const void* q;
  const void* k_pool;
  const void* v_pool;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;    // [num_seqs][n_q][n_parts_max][D] unnormalised partition outputs
  float2* ws_ml;  // [num_seqs][n_q][n_parts_max] (log2-domain max, sum)
  int32_t* dev_err;
  float scale_log2;  // scale * log2(e) (* k_scale for fp8 caches)
  float out_mul;     // fp8 caches: v_scale x 256 (V is widened as code x 2^-8); else 1
  int n_q, n_kv, group, num_seqs, max_blocks, num_blocks, n_parts_max;
};

struct ReduceParams {
  void* out;
  const int32_t* context_lens;
  const float* ws_o;
  const float2* ws_ml;
  float out_mul;
  int n_q, num_seqs, max_blocks, n_parts_max;
};

int decode_num_parts(int max_blocks_per_seq);
bool decode_uses_tma(pa_dtype q_dt, pa_dtype kv_dt);
cudaError_t launch_decode_partitions(const DecodeParams& p, int D, pa_dtype q_dt,
                                     pa_dtype kv_dt, const CUtensorMap* tmk,
                                     const CUtensorMap* tmv, cudaStream_t st);
cudaError_t launch_decode_reduce(const ReduceParams& r, int D, pa_dtype out_dt,
                                 cudaStream_t st);

struct ScatterParams {
  void* k_pool;
  void* v_pool;
  const void* key;
  const void* value;
  const int64_t* slot_mapping;
  int32_t* dev_err;
  float k_scale, v_scale;
  int num_tokens, n_kv, head_dim, num_blocks;
};
cudaError_t launch_reshape_and_cache(const ScatterParams& p, pa_dtype src_dt,
                                     pa_dtype cache_dt, cudaStream_t st);

struct CopyParams {
  void* k_pool;
  void* v_pool;
  const int64_t* pairs;
  int32_t* dev_err;
  int n_pairs, num_blocks;
  int64_t block_bytes;  // bytes of one block (all heads) in one pool
};
cudaError_t launch_copy_blocks(const CopyParams& p, cudaStream_t st);

struct PrefillParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* query_start_loc;
  const int32_t* context_lens;
  int32_t* dev_err;
  float scale_log2;
  float out_mul;
  int n_q, n_kv, group, n_chunks, max_blocks, num_blocks, max_chunk_len;
};
cudaError_t launch_prefill(const PrefillParams& p, pa_dtype kv_dt, const void* k_pool,
                           const void* v_pool, cudaStream_t st);

}  // namespace pa
