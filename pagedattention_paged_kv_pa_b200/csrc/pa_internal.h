// Internal interfaces between the C ABI shim (capi.cu) and the kernel
// launchers.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/pa.h"

namespace pa {

// A bounded wait inside a kernel gives up after this long (the kernels'
// normal waits last microseconds) and flags PA_DEVERR_TIMEOUT.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

// Tokens per decode context partition: 1024 (64 blocks of 16) with 16-bit
// and fp32 caches, 2048 with fp8 caches (about the same K/V bytes per CTA).
// Longer partitions spread each CTA's fixed costs (block-table read, first
// load latency, query setup, merge) over more blocks; measured on B200 with
// the benchmark workloads, 1024 beats 512/768/2048 for 16-bit caches and
// 2048 beats 1024 for fp8.  The workspace is laid out for the shorter one.
constexpr int kPart16 = 1024;
constexpr int kPartFp8 = 2048;
inline int decode_part_tokens(pa_dtype kv_dt) {
  return kv_dt == PA_FP8_E4M3 ? kPartFp8 : kPart16;
}

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
  int n_q, n_kv, group, num_seqs, max_blocks, num_blocks;
  int n_parts_max;   // workspace stride: partitions of max_blocks at kPart16
  int n_parts_grid;  // partitions of max_blocks at this cache type's length
  int q_len;         // queries per sequence (1: decode; >1: multi-query decode)
  int n_cg;          // groups of 8 (query, head) columns per kv head
  // shared-prefix decode: groups of sequences whose tables start with the
  // same blocks.  grp_members [n_groups][grp_width] (-1: unused),
  // grp_shared_blocks [n_groups], seq_group [num_seqs] (-1: none).  A group
  // launch (grp_members set) computes the partitions wholly inside a group's
  // shared blocks for all members; a per-sequence launch with seq_group set
  // skips them.
  const int32_t* grp_members;
  const int32_t* grp_shared_blocks;
  const int32_t* seq_group;
  int grp_width;
  int n_groups;     // for range checks of seq_group
  int n_seqs_all;   // for range checks of grp_members (num_seqs is the grid)
  // bounded waits give up after wait_ns; skip_tile >= 0 (pa_test_decode_timeout
  // only) makes each CTA's producer leave the stage of that tile unfilled
  unsigned long long wait_ns;
  int skip_tile;
};

struct ReduceParams {
  void* out;
  const int32_t* context_lens;
  const float* ws_o;
  const float2* ws_ml;
  float out_mul;
  int n_q, num_seqs, max_blocks, n_parts_max;
  int part_tokens;  // partition length the partition kernel used
};

int decode_num_parts(int max_blocks_per_seq, int part_tokens);
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

// Block copy from (src_k, src_v) to (dst_k, dst_v): the same pools for
// copy-on-write, a device and a pinned host pool for swapping.
struct CopyParams {
  void* dst_k;
  void* dst_v;
  const void* src_k;
  const void* src_v;
  const int64_t* pairs;
  int32_t* dev_err;
  int n_pairs, src_num_blocks, dst_num_blocks;
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
  int stage_rows;  // workspace rows per (chunk, kv head): max_blocks * 16 rounded up to 128
  // 0: chunk c's queries are query_start_loc[c] .. query_start_loc[c+1]-1.
  // q_len > 0 (multi-query decode): chunk c is sequence c's q_len queries,
  // rows c q_len .. c q_len + q_len - 1, at the last q_len positions of its
  // context; query_start_loc is not read, and queries before the context's
  // start get all-zero rows.
  int fixed_q_len;
};
// Without a workspace the attention kernel widens K/V itself (tmk / tmv: TMA
// maps over the fp8 pools, the decode kernel's; unused for bf16).  With one,
// a first pass widens every chunk's history into it (K rows, then V rows, f16
// [n_chunks][n_kv][stage_rows][128]) and tmk / tmv map its two halves.
cudaError_t launch_prefill(const PrefillParams& p, pa_dtype kv_dt, const void* k_pool,
                           const void* v_pool, const CUtensorMap* tmk, const CUtensorMap* tmv,
                           void* workspace, cudaStream_t st);
size_t prefill_stage_rows(int max_blocks);

}  // namespace pa
