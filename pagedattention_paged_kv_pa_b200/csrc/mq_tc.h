// Multi-query decode on tcgen05 tensor cores: the launcher the C ABI shim
// calls for 16-bit queries over a cache of the same type with head_dim 128.
// Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace pa {

struct MQParams {
  void* out;                   // [num_seqs][q_len][n_q][128], the query type
  const int32_t* block_tables;  // [num_seqs][max_blocks]
  const int32_t* context_lens;  // [num_seqs], the q_len new tokens included
  float* ws_o;    // [num_seqs][q_len][n_q][n_parts_max][128] unnormalised segment outputs
  float2* ws_ml;  // [num_seqs][q_len][n_q][n_parts_max] (log2-domain max, sum)
  int32_t* dev_err;
  float scale_log2;  // scale x log2(e)
  int n_q, n_kv, group, q_len, num_seqs, max_blocks, num_blocks;
  int n_parts_max;  // workspace slots per row: 1024-token partitions of max_blocks
};

// tmq: 3-D map over q viewed as [num_seqs x q_len][n_q][128] (16-bit), box
// {64, group, q_len}, 128-byte swizzle; tmk / tmv: 2-D maps over the pools
// viewed as [num_blocks x n_kv x 16][128], box {64, 16}, 128-byte swizzle.
// `merge`: the workspace is present (some sequence may span more than one
// 1024-token partition) and the merge kernel runs after the attention kernel.
cudaError_t launch_mq_tc(const MQParams& p, bool bf16, const void* k_pool, const void* v_pool,
                         const CUtensorMap* tmq, const CUtensorMap* tmk, const CUtensorMap* tmv,
                         bool merge, cudaStream_t st);

}  // namespace pa
