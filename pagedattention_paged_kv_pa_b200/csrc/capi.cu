// C ABI shim: validates arguments on the host, sizes the decode workspace,
// builds (and caches) TMA tensor maps over the KV pools, and queues the
// kernels on the caller's stream.  No device memory is allocated here and no
// call synchronises with the device.
#include <algorithm>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "mq_tc.h"
#include "pa_internal.h"

namespace {

using pa::DecodeParams;
using pa::ReduceParams;

constexpr float kLog2e = 1.4426950408889634f;
// The decode and prefill kernels widen fp8 V codes to f16 as code x 2^-8; the
// output scale undoes it (exact: a power of two).
constexpr float kFp8VUnscale = 256.f;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(pa_dtype d) {
  switch (d) {
    case PA_F32: return 4;
    case PA_F16: return 2;
    case PA_BF16: return 2;
    case PA_FP8_E4M3: return 1;
  }
  return 0;
}

bool valid_dtype(int d) { return d >= PA_F32 && d <= PA_FP8_E4M3; }

// ---------------------------------------------------------------- tensor maps

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeFn>(nullptr);
    return reinterpret_cast<EncodeFn>(p);
  }();
  return fn;
}

struct MapKey {
  const void* ptr;
  uint64_t rows;
  uint32_t cols, esize, box_x, box_y, swz;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && rows == o.rows && cols == o.cols && esize == o.esize &&
           box_x == o.box_x && box_y == o.box_y && swz == o.swz;
  }
};

struct MapCache {
  std::mutex mu;
  std::vector<std::pair<MapKey, CUtensorMap>> entries;  // most recent last
};

MapCache& map_cache() {
  static MapCache c;
  return c;
}

// A 2-D map over a row-major [rows][cols] array of `esize`-byte elements with a
// (box_x cols) x (box_y rows) box and the given swizzle.  Returns false if the
// driver refuses it.
bool get_map(const void* ptr, uint64_t rows, uint32_t cols, uint32_t esize, uint32_t box_x,
             uint32_t box_y, CUtensorMapSwizzle swz, CUtensorMap* out) {
  MapKey key{ptr, rows, cols, esize, box_x, box_y, static_cast<uint32_t>(swz)};
  MapCache& c = map_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  for (size_t i = 0; i < c.entries.size(); ++i)
    if (c.entries[i].first == key) {
      *out = c.entries[i].second;
      return true;
    }
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMap m;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esize};
  const cuuint32_t box[2] = {box_x, box_y};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      esize == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  if (fn(&m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  if (c.entries.size() >= 64) c.entries.erase(c.entries.begin());
  c.entries.emplace_back(key, m);
  *out = m;
  return true;
}

// Map over a KV pool viewed as [num_blocks * n_kv * 16][head_dim]: one box is a
// 16-token tile (or its first/second 64-column half for 16-bit head_dim 128),
// written to shared memory with the swizzle the decode kernel reads with.
bool kv_pool_map(const void* pool, int num_blocks, int n_kv, int d, pa_dtype dt, CUtensorMap* m) {
  const uint32_t es = elem_bytes(dt);
  const uint32_t row_bytes = d * es;
  const uint32_t box_x = row_bytes > 128 ? 128 / es : d;
  const CUtensorMapSwizzle swz =
      (box_x * es == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return get_map(pool, (uint64_t)num_blocks * n_kv * 16, d, es, box_x, 16, swz, m);
}

// Map over 16-bit queries [num_seqs x q_len][n_q][128] for the multi-query
// tensor-core kernel: one box is the q_len x G rows of one kv head's query
// heads, 64 columns wide (128-byte swizzle), landing as rows query x G + head.
// Not cached: the query tensor usually changes from call to call.
bool q_rows_map(const void* q, int rows, int n_q, int group, int q_len, CUtensorMap* m) {
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(n_q), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(n_q) * 256};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(q_len)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------ decode checks

struct DecodeShape {
  int n_q, n_kv, d, num_seqs, max_blocks, num_blocks, n_parts;
};

pa_status check_decode(const DecodeShape& s, int block_size, pa_dtype q_dt, pa_dtype kv_dt) {
  if (block_size != 16) return PA_ERR_UNSUPPORTED;
  if (s.d != 64 && s.d != 128) return PA_ERR_UNSUPPORTED;
  if (s.n_q < 1 || s.n_kv < 1 || s.n_q % s.n_kv != 0) return PA_ERR_INVALID_ARG;
  if (s.n_q / s.n_kv > 8) return PA_ERR_UNSUPPORTED;
  if (s.num_seqs < 0 || s.max_blocks < 1 || s.num_blocks < 1) return PA_ERR_INVALID_ARG;
  if (s.num_seqs > 65535 || s.n_kv > 65535) return PA_ERR_UNSUPPORTED;
  if ((int64_t)s.num_blocks * s.n_kv * 16 >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  if ((int64_t)s.max_blocks * 16 >= (int64_t(1) << 30)) return PA_ERR_UNSUPPORTED;
  if (!valid_dtype(q_dt) || !valid_dtype(kv_dt)) return PA_ERR_INVALID_ARG;
  const bool ok = (q_dt == PA_F32 && kv_dt == PA_F32) || (q_dt == PA_F16 && kv_dt == PA_F16) ||
                  (q_dt == PA_BF16 && kv_dt == PA_BF16) ||
                  ((q_dt == PA_F16 || q_dt == PA_BF16) && kv_dt == PA_FP8_E4M3);
  return ok ? PA_OK : PA_ERR_UNSUPPORTED;
}

size_t ws_o_bytes(const DecodeShape& s) {
  return (size_t)s.num_seqs * s.n_q * s.n_parts * s.d * sizeof(float);
}
size_t ws_total_bytes(const DecodeShape& s) {
  const size_t o = (ws_o_bytes(s) + 255) & ~size_t(255);
  return o + (size_t)s.num_seqs * s.n_q * s.n_parts * sizeof(float2);
}

pa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

}  // namespace

extern "C" {

int pa_abi_version(void) { return PA_ABI_VERSION; }

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PA_ERR_OOM: return "out of blocks";
    case PA_ERR_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

size_t pa_decode_workspace_size(int num_seqs, int n_q_heads, int head_dim, int max_blocks_per_seq) {
  if (num_seqs < 0 || n_q_heads < 1 || head_dim < 1 || max_blocks_per_seq < 1) return 0;
  DecodeShape s{n_q_heads, 1, head_dim, num_seqs, max_blocks_per_seq, 1,
                pa::decode_num_parts(max_blocks_per_seq, pa::kPart16)};
  if (s.n_parts <= 1) return 0;
  return ws_total_bytes(s);
}

// pa_decode_multi's step is the causal chunk of a sequence's q_len newest
// queries over its cache.  With head_dim 128 and group 1, 2, 4 or 8 it runs on
// tensor cores, each K/V tile read once for all q_len x G (query, head) rows of
// a kv head: 16-bit queries over a cache of the same type on the multi-query
// kernel (64-row tiles, persistent CTAs with equal shares of the key tiles),
// bf16 queries over an fp8 cache on the chunked-prefill kernel (one 128-row
// tile per (sequence, kv head)).
static bool multi_on_tensor_cores(int q_len, int head_dim, int group, pa_dtype q_dt,
                                  pa_dtype kv_dt) {
  const bool same16 = (q_dt == PA_BF16 || q_dt == PA_F16) && kv_dt == q_dt;
  return q_len > 1 && head_dim == 128 && (same16 || (q_dt == PA_BF16 && kv_dt == PA_FP8_E4M3)) &&
         (group == 1 || group == 2 || group == 4 || group == 8);
}

static pa_status decode_parts_impl(void* out, const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, const int32_t* context_lens,
                               float scale, int block_size, int n_q_heads, int n_kv_heads,
                               int head_dim, int num_seqs, int q_len, int max_blocks_per_seq,
                               int num_blocks, pa_dtype q_dtype, pa_dtype kv_dtype,
                               float k_scale, float v_scale, void* workspace,
                               size_t workspace_bytes, int32_t* dev_err, void* stream,
                               const int32_t* grp_members = nullptr,
                               const int32_t* grp_shared_blocks = nullptr,
                               const int32_t* seq_group = nullptr, int n_groups = 0,
                               int grp_width = 0, bool tensor_core_multi = false,
                               unsigned long long wait_ns = pa::kWaitLimitNs,
                               int skip_tile = -1) {
  DecodeShape s{n_q_heads, n_kv_heads, head_dim, num_seqs, max_blocks_per_seq, num_blocks,
                pa::decode_num_parts(max_blocks_per_seq, pa::kPart16)};
  pa_status st = check_decode(s, block_size, q_dtype, kv_dtype);
  if (st != PA_OK) return st;
  if (q_len < 1 || q_len > 8) return PA_ERR_INVALID_ARG;
  if (q_len > 1 && q_dtype == PA_F32) return PA_ERR_UNSUPPORTED;
  const int n_cg = (n_q_heads / n_kv_heads * q_len + 7) / 8;  // column groups per kv head
  if ((int64_t)n_kv_heads * n_cg > 65535) return PA_ERR_UNSUPPORTED;
  DecodeShape ws = s;  // workspace rows: every (query, q head) of a sequence
  ws.n_q = n_q_heads * q_len;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool))
    return PA_ERR_INVALID_ARG;
  if (!(scale == scale) || (kv_dtype == PA_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)))
    return PA_ERR_INVALID_ARG;
  // partitions this cache type uses; the workspace stride is s.n_parts
  const int n_grid = pa::decode_num_parts(max_blocks_per_seq, pa::decode_part_tokens(kv_dtype));
  if (n_grid > 1) {
    if (!workspace || !aligned16(workspace) || workspace_bytes < ws_total_bytes(ws))
      return PA_ERR_INVALID_ARG;
  }
  const bool fp8 = kv_dtype == PA_FP8_E4M3;
  DecodeParams p;
  p.out = out;
  p.q = q;
  p.k_pool = k_pool;
  p.v_pool = v_pool;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_ml = workspace ? reinterpret_cast<float2*>(static_cast<char*>(workspace) +
                                                  ((ws_o_bytes(ws) + 255) & ~size_t(255)))
                      : nullptr;
  p.dev_err = dev_err;
  p.scale_log2 = scale * kLog2e * (fp8 ? k_scale : 1.f);
  p.out_mul = fp8 ? v_scale * kFp8VUnscale : 1.f;
  p.n_q = n_q_heads;
  p.n_kv = n_kv_heads;
  p.group = n_q_heads / n_kv_heads;
  p.num_seqs = num_seqs;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.n_parts_max = s.n_parts;
  p.n_parts_grid = n_grid;
  p.q_len = q_len;
  p.n_cg = n_cg;
  p.grp_members = nullptr;
  p.grp_shared_blocks = nullptr;
  p.seq_group = nullptr;
  p.grp_width = 0;
  p.n_groups = n_groups;
  p.n_seqs_all = num_seqs;
  p.wait_ns = wait_ns;
  p.skip_tile = skip_tile;
  CUtensorMap tmk, tmv;
  if (pa::decode_uses_tma(q_dtype, kv_dtype)) {
    if (!kv_pool_map(k_pool, num_blocks, n_kv_heads, head_dim, kv_dtype, &tmk) ||
        !kv_pool_map(v_pool, num_blocks, n_kv_heads, head_dim, kv_dtype, &tmv))
      return PA_ERR_CUDA;
  }
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (tensor_core_multi && kv_dtype == q_dtype) {
    pa::MQParams mp;
    mp.out = out;
    mp.block_tables = block_tables;
    mp.context_lens = context_lens;
    mp.ws_o = p.ws_o;
    mp.ws_ml = p.ws_ml;
    mp.dev_err = dev_err;
    mp.scale_log2 = p.scale_log2;
    mp.n_q = n_q_heads;
    mp.n_kv = n_kv_heads;
    mp.group = p.group;
    mp.q_len = q_len;
    mp.num_seqs = num_seqs;
    mp.max_blocks = max_blocks_per_seq;
    mp.num_blocks = num_blocks;
    mp.n_parts_max = s.n_parts;
    CUtensorMap tmq;
    if (!q_rows_map(q, num_seqs * q_len, n_q_heads, p.group, q_len, &tmq)) return PA_ERR_CUDA;
    return cuda_status(pa::launch_mq_tc(mp, q_dtype == PA_BF16, k_pool, v_pool, &tmq, &tmk, &tmv,
                                        n_grid > 1, cs));
  }
  if (tensor_core_multi) {
    pa::PrefillParams pp;
    pp.out = out;
    pp.q = q;
    pp.block_tables = block_tables;
    pp.query_start_loc = nullptr;
    pp.context_lens = context_lens;
    pp.dev_err = dev_err;
    pp.scale_log2 = p.scale_log2;
    pp.out_mul = p.out_mul;  // the in-kernel widening takes fp8 V as code x 2^-8 too
    pp.n_q = n_q_heads;
    pp.n_kv = n_kv_heads;
    pp.group = p.group;
    pp.n_chunks = num_seqs;
    pp.max_blocks = max_blocks_per_seq;
    pp.num_blocks = num_blocks;
    pp.max_chunk_len = q_len;
    pp.stage_rows = static_cast<int>(pa::prefill_stage_rows(max_blocks_per_seq));
    pp.fixed_q_len = q_len;
    return cuda_status(pa::launch_prefill(pp, kv_dtype, k_pool, v_pool, &tmk, &tmv, nullptr, cs));
  }
  if (n_groups > 0) {
    // one launch: the groups' shared partitions, every member at once (one
    // column per (member, head)), next to every sequence's other partitions
    if ((int64_t)n_groups + num_seqs > 65535) return PA_ERR_UNSUPPORTED;
    p.grp_members = grp_members;
    p.grp_shared_blocks = grp_shared_blocks;
    p.seq_group = seq_group;
    p.grp_width = grp_width;
    p.num_seqs = n_groups + num_seqs;  // grid z: groups, then sequences
  }
  return cuda_status(pa::launch_decode_partitions(p, head_dim, q_dtype, kv_dtype, &tmk, &tmv, cs));
}

pa_status pa_decode_partitions(void* out, const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, const int32_t* context_lens,
                               float scale, int block_size, int n_q_heads, int n_kv_heads,
                               int head_dim, int num_seqs, int max_blocks_per_seq,
                               int num_blocks, pa_dtype q_dtype, pa_dtype kv_dtype,
                               float k_scale, float v_scale, void* workspace,
                               size_t workspace_bytes, int32_t* dev_err, void* stream) {
  return decode_parts_impl(out, q, k_pool, v_pool, block_tables, context_lens, scale, block_size,
                           n_q_heads, n_kv_heads, head_dim, num_seqs, 1, max_blocks_per_seq,
                           num_blocks, q_dtype, kv_dtype, k_scale, v_scale, workspace,
                           workspace_bytes, dev_err, stream);
}

static pa_status decode_reduce_impl(void* out, const int32_t* context_lens, int n_rows, int head_dim,
                           int num_seqs, int max_blocks_per_seq, pa_dtype q_dtype,
                           pa_dtype kv_dtype, float v_scale, const void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_seqs < 0 || n_rows < 1 || max_blocks_per_seq < 1) return PA_ERR_INVALID_ARG;
  if (!valid_dtype(q_dtype) || !valid_dtype(kv_dtype) || q_dtype == PA_FP8_E4M3)
    return PA_ERR_INVALID_ARG;
  DecodeShape s{n_rows, 1, head_dim, num_seqs, max_blocks_per_seq, 1,
                pa::decode_num_parts(max_blocks_per_seq, pa::kPart16)};
  const int part_tokens = pa::decode_part_tokens(kv_dtype);
  if (num_seqs == 0 || pa::decode_num_parts(max_blocks_per_seq, part_tokens) <= 1) return PA_OK;
  if (!out || !context_lens || !workspace || !aligned16(out) || !aligned16(workspace) ||
      workspace_bytes < ws_total_bytes(s))
    return PA_ERR_INVALID_ARG;
  ReduceParams r;
  r.out = out;
  r.context_lens = context_lens;
  r.ws_o = static_cast<const float*>(workspace);
  r.ws_ml = reinterpret_cast<const float2*>(static_cast<const char*>(workspace) +
                                            ((ws_o_bytes(s) + 255) & ~size_t(255)));
  r.out_mul = kv_dtype == PA_FP8_E4M3 ? v_scale * kFp8VUnscale : 1.f;
  r.n_q = n_rows;
  r.num_seqs = num_seqs;
  r.max_blocks = max_blocks_per_seq;
  r.n_parts_max = s.n_parts;
  r.part_tokens = part_tokens;
  return cuda_status(pa::launch_decode_reduce(r, head_dim, q_dtype,
                                              static_cast<cudaStream_t>(stream)));
}

pa_status pa_decode_reduce(void* out, const int32_t* context_lens, int n_q_heads, int head_dim,
                           int num_seqs, int max_blocks_per_seq, pa_dtype q_dtype,
                           pa_dtype kv_dtype, float v_scale, const void* workspace,
                           size_t workspace_bytes, void* stream) {
  return decode_reduce_impl(out, context_lens, n_q_heads, head_dim, num_seqs, max_blocks_per_seq,
                            q_dtype, kv_dtype, v_scale, workspace, workspace_bytes, stream);
}

pa_status pa_decode(void* out, const void* q, const void* k_pool, const void* v_pool,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    int block_size, int n_q_heads, int n_kv_heads, int head_dim, int num_seqs,
                    int max_blocks_per_seq, int num_blocks, pa_dtype q_dtype, pa_dtype kv_dtype,
                    float k_scale, float v_scale, void* workspace, size_t workspace_bytes,
                    int32_t* dev_err, void* stream) {
  pa_status st = pa_decode_partitions(out, q, k_pool, v_pool, block_tables, context_lens, scale,
                                      block_size, n_q_heads, n_kv_heads, head_dim, num_seqs,
                                      max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                                      v_scale, workspace, workspace_bytes, dev_err, stream);
  if (st != PA_OK) return st;
  return pa_decode_reduce(out, context_lens, n_q_heads, head_dim, num_seqs, max_blocks_per_seq,
                          q_dtype, kv_dtype, v_scale, workspace, workspace_bytes, stream);
}

pa_status pa_test_decode_timeout(void* out, const void* q, const void* k_pool,
                                 const void* v_pool, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, int block_size,
                                 int n_q_heads, int n_kv_heads, int head_dim, int num_seqs,
                                 int max_blocks_per_seq, int num_blocks, pa_dtype q_dtype,
                                 pa_dtype kv_dtype, float k_scale, float v_scale, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_err, void* stream,
                                 int skip_tile, uint32_t wait_limit_us) {
  if (skip_tile < 0 || wait_limit_us < 1 || wait_limit_us > 1000000) return PA_ERR_INVALID_ARG;
  if (q_dtype == PA_F32) return PA_ERR_UNSUPPORTED;  // the TMA kernels only
  pa_status st = decode_parts_impl(out, q, k_pool, v_pool, block_tables, context_lens, scale,
                                   block_size, n_q_heads, n_kv_heads, head_dim, num_seqs, 1,
                                   max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                                   v_scale, workspace, workspace_bytes, dev_err, stream, nullptr,
                                   nullptr, nullptr, 0, 0, false,
                                   (unsigned long long)wait_limit_us * 1000ull, skip_tile);
  if (st != PA_OK) return st;
  return decode_reduce_impl(out, context_lens, n_q_heads, head_dim, num_seqs, max_blocks_per_seq,
                            q_dtype, kv_dtype, v_scale, workspace, workspace_bytes, stream);
}

pa_status pa_decode_multi(void* out, const void* q, const void* k_pool, const void* v_pool,
                          const int32_t* block_tables, const int32_t* context_lens, float scale,
                          int block_size, int n_q_heads, int n_kv_heads, int head_dim,
                          int num_seqs, int q_len, int max_blocks_per_seq, int num_blocks,
                          pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
                          void* workspace, size_t workspace_bytes, int32_t* dev_err,
                          void* stream) {
  const bool tc = n_kv_heads > 0 && n_q_heads % n_kv_heads == 0 &&
                  multi_on_tensor_cores(q_len, head_dim, n_q_heads / n_kv_heads, q_dtype,
                                        kv_dtype);
  pa_status st = decode_parts_impl(out, q, k_pool, v_pool, block_tables, context_lens, scale,
                                   block_size, n_q_heads, n_kv_heads, head_dim, num_seqs, q_len,
                                   max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                                   v_scale, workspace, workspace_bytes, dev_err, stream, nullptr,
                                   nullptr, nullptr, 0, 0, tc);
  if (st != PA_OK || tc) return st;  // the tensor-core route has no partitions to merge
  return decode_reduce_impl(out, context_lens, n_q_heads * q_len, head_dim, num_seqs,
                            max_blocks_per_seq, q_dtype, kv_dtype, v_scale, workspace,
                            workspace_bytes, stream);
}

pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_pool,
                                  const void* v_pool, const int32_t* block_tables,
                                  const int32_t* context_lens, float scale, int block_size,
                                  int n_q_heads, int n_kv_heads, int head_dim, int num_seqs,
                                  int max_blocks_per_seq, int num_blocks, pa_dtype q_dtype,
                                  pa_dtype kv_dtype, float k_scale, float v_scale,
                                  const int32_t* group_members, const int32_t* group_shared_blocks,
                                  const int32_t* seq_group, int n_groups, int group_width,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_err,
                                  void* stream) {
  if (n_groups < 0) return PA_ERR_INVALID_ARG;
  if (n_groups > 0) {
    if (!group_members || !group_shared_blocks || !seq_group || group_width < 1)
      return PA_ERR_INVALID_ARG;
    if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (n_kv_heads < 1 || n_q_heads % n_kv_heads != 0 ||
        group_width * (n_q_heads / n_kv_heads) > 32 || n_groups > 65535)
      return PA_ERR_UNSUPPORTED;
  }
  pa_status st = decode_parts_impl(out, q, k_pool, v_pool, block_tables, context_lens, scale,
                                   block_size, n_q_heads, n_kv_heads, head_dim, num_seqs, 1,
                                   max_blocks_per_seq, num_blocks, q_dtype, kv_dtype, k_scale,
                                   v_scale, workspace, workspace_bytes, dev_err, stream,
                                   group_members, group_shared_blocks, seq_group, n_groups,
                                   group_width);
  if (st != PA_OK) return st;
  return decode_reduce_impl(out, context_lens, n_q_heads, head_dim, num_seqs, max_blocks_per_seq,
                            q_dtype, kv_dtype, v_scale, workspace, workspace_bytes, stream);
}

pa_status pa_prefix_groups(const int32_t* block_tables, const int32_t* context_lens,
                           int num_seqs, int max_blocks_per_seq, int n_q_heads, int n_kv_heads,
                           pa_dtype kv_dtype, int32_t* group_members_out,
                           int32_t* group_shared_blocks_out, int32_t* seq_group_out,
                           int* n_groups_out, int* group_width_out) {
  if (!n_groups_out || !group_width_out || num_seqs < 0 || max_blocks_per_seq < 1 ||
      n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads != 0 || !valid_dtype(kv_dtype))
    return PA_ERR_INVALID_ARG;
  const int G = n_q_heads / n_kv_heads;
  if (G > 8) return PA_ERR_UNSUPPORTED;
  const int W = 32 / G;  // members per group: 4 column groups of 8 (member, head) pairs
  *n_groups_out = 0;
  *group_width_out = W;
  if (num_seqs == 0) return PA_OK;
  if (!block_tables || !context_lens || !group_members_out || !group_shared_blocks_out ||
      !seq_group_out)
    return PA_ERR_INVALID_ARG;
  const int part_blocks = pa::decode_part_tokens(kv_dtype) / 16;
  std::vector<int> full(num_seqs);
  for (int s = 0; s < num_seqs; s++) {
    const int c = context_lens[s] < 0 ? 0 : context_lens[s];
    full[s] = std::min(c / 16, max_blocks_per_seq);
    seq_group_out[s] = -1;
  }
  // sequences whose first block is the same, in index order
  std::unordered_map<int32_t, std::vector<int>> by_first;
  std::vector<int32_t> firsts;
  for (int s = 0; s < num_seqs; s++) {
    if (full[s] < part_blocks) continue;  // shares no whole partition
    const int32_t b = block_tables[(size_t)s * max_blocks_per_seq];
    auto it = by_first.find(b);
    if (it == by_first.end()) {
      firsts.push_back(b);
      by_first[b] = {s};
    } else {
      it->second.push_back(s);
    }
  }
  std::vector<std::pair<std::vector<int>, int>> groups;  // (members, shared blocks)
  for (int32_t b : firsts) {
    const std::vector<int>& cand = by_first[b];
    for (size_t c0 = 0; c0 < cand.size(); c0 += W) {
      const size_t n = std::min(cand.size() - c0, (size_t)W);
      if (n < 2) continue;
      const int s0 = cand[c0];
      int shared = full[s0];
      for (size_t k = 1; k < n; k++) {
        const int s = cand[c0 + k];
        int m = 0;
        const int lim = std::min(shared, full[s]);
        while (m < lim && block_tables[(size_t)s * max_blocks_per_seq + m] ==
                              block_tables[(size_t)s0 * max_blocks_per_seq + m])
          m++;
        shared = m;
      }
      if (shared < part_blocks) continue;
      groups.emplace_back(std::vector<int>(cand.begin() + c0, cand.begin() + c0 + n), shared);
    }
  }
  // rows as wide as the largest group, so the group pass has no empty columns
  int w = 0;
  for (auto& g : groups) w = std::max(w, (int)g.first.size());
  for (size_t g = 0; g < groups.size(); g++) {
    const auto& m = groups[g].first;
    for (int k = 0; k < w; k++) group_members_out[g * w + k] = k < (int)m.size() ? m[k] : -1;
    group_shared_blocks_out[g] = groups[g].second;
    for (int s : m) seq_group_out[s] = (int)g;
  }
  *n_groups_out = (int)groups.size();
  *group_width_out = groups.empty() ? W : w;
  return PA_OK;
}

size_t pa_prefill_workspace_size(int n_chunks, int n_kv_heads, int head_dim,
                                 int max_blocks_per_seq, int block_size) {
  if (n_chunks < 0 || n_kv_heads < 1 || head_dim != 128 || max_blocks_per_seq < 1 ||
      block_size != 16)
    return 0;
  // K and V: f16 [n_chunks][n_kv][stage_rows][head_dim]
  return 2 * (size_t)n_chunks * n_kv_heads * pa::prefill_stage_rows(max_blocks_per_seq) *
         head_dim * 2;
}

pa_status pa_prefill_paged(void* out, const void* q, const void* k_pool, const void* v_pool,
                           const int32_t* block_tables, const int32_t* query_start_loc,
                           const int32_t* context_lens, float scale, int block_size,
                           int n_q_heads, int n_kv_heads, int head_dim, int n_chunks,
                           int max_chunk_len, int max_blocks_per_seq, int num_blocks,
                           pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
                           void* workspace, size_t workspace_bytes, int32_t* dev_err,
                           void* stream) {
  if (block_size != 16 || head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (n_chunks < 0 || max_chunk_len < 1 || max_blocks_per_seq < 1 || num_blocks < 1)
    return PA_ERR_INVALID_ARG;
  if (n_chunks > 65535 || n_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
  if ((int64_t)max_blocks_per_seq * 16 >= (int64_t(1) << 30)) return PA_ERR_UNSUPPORTED;
  if ((int64_t)num_blocks * n_kv_heads * 16 >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  if (q_dtype != PA_BF16 || (kv_dtype != PA_BF16 && kv_dtype != PA_FP8_E4M3))
    return PA_ERR_UNSUPPORTED;
  if (!(scale == scale) || (kv_dtype == PA_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)))
    return PA_ERR_INVALID_ARG;
  if (n_chunks == 0) return PA_OK;
  if (!out || !q || !k_pool || !v_pool || !block_tables || !query_start_loc || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool))
    return PA_ERR_INVALID_ARG;
  const int grid_x = (max_chunk_len + (128 / G) - 1) / (128 / G);
  if (grid_x > 65535 * 32) return PA_ERR_UNSUPPORTED;
  const bool fp8 = kv_dtype == PA_FP8_E4M3;
  pa::PrefillParams p;
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.query_start_loc = query_start_loc;
  p.context_lens = context_lens;
  p.dev_err = dev_err;
  p.scale_log2 = scale * kLog2e * (fp8 ? k_scale : 1.f);
  // in-kernel widening takes fp8 V as code x 2^-8 (see below for the workspace)
  p.out_mul = fp8 ? v_scale * kFp8VUnscale : 1.f;
  p.n_q = n_q_heads;
  p.n_kv = n_kv_heads;
  p.group = G;
  p.n_chunks = n_chunks;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.max_chunk_len = max_chunk_len;
  p.stage_rows = static_cast<int>(pa::prefill_stage_rows(max_blocks_per_seq));
  p.fixed_q_len = 0;
  CUtensorMap tmk{}, tmv{};
  if (workspace != nullptr &&
      (!aligned16(workspace) ||
       workspace_bytes < pa_prefill_workspace_size(n_chunks, n_kv_heads, head_dim,
                                                   max_blocks_per_seq, block_size)))
    return PA_ERR_INVALID_ARG;
  if (!fp8) {
    // bf16 cache: the tensor cores take the pools' bf16 blocks as they are,
    // loaded by TMA through the block table; there is nothing to widen, so a
    // workspace is not used
    if (!kv_pool_map(k_pool, num_blocks, n_kv_heads, head_dim, kv_dtype, &tmk) ||
        !kv_pool_map(v_pool, num_blocks, n_kv_heads, head_dim, kv_dtype, &tmv))
      return PA_ERR_CUDA;
  } else if (workspace != nullptr) {
    // the history of every chunk is widened once into the workspace; both fp8
    // operands widen exactly there, so V needs no 2^-8 fold
    const uint64_t rows = (uint64_t)n_chunks * n_kv_heads * p.stage_rows;
    if (rows >= (uint64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    p.out_mul = fp8 ? v_scale : 1.f;
    const uint16_t* kst = static_cast<const uint16_t*>(workspace);
    if (!get_map(kst, rows, 128, 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B, &tmk) ||
        !get_map(kst + rows * 128, rows, 128, 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B, &tmv))
      return PA_ERR_CUDA;
  } else if (!kv_pool_map(k_pool, num_blocks, n_kv_heads, head_dim, kv_dtype, &tmk) ||
             !kv_pool_map(v_pool, num_blocks, n_kv_heads, head_dim, kv_dtype, &tmv)) {
    return PA_ERR_CUDA;
  }
  return cuda_status(pa::launch_prefill(p, kv_dtype, k_pool, v_pool, &tmk, &tmv, workspace,
                                        static_cast<cudaStream_t>(stream)));
}

pa_status pa_reshape_and_cache(void* k_pool, void* v_pool, const void* key, const void* value,
                               const int64_t* slot_mapping, int num_tokens, int n_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype src_dtype,
                               pa_dtype cache_dtype, float k_scale, float v_scale,
                               int32_t* dev_err, void* stream) {
  if (block_size != 16) return PA_ERR_UNSUPPORTED;
  if (num_tokens < 0 || n_kv_heads < 1 || head_dim < 1 || num_blocks < 1)
    return PA_ERR_INVALID_ARG;
  if (!valid_dtype(src_dtype) || !valid_dtype(cache_dtype) || src_dtype == PA_FP8_E4M3)
    return PA_ERR_UNSUPPORTED;
  if (cache_dtype != src_dtype && cache_dtype != PA_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  if ((head_dim * elem_bytes(src_dtype)) % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k_pool || !v_pool || !key || !value || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(key) || !aligned16(value))
    return PA_ERR_INVALID_ARG;
  if (cache_dtype == PA_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)) return PA_ERR_INVALID_ARG;
  pa::ScatterParams p;
  p.k_pool = k_pool;
  p.v_pool = v_pool;
  p.key = key;
  p.value = value;
  p.slot_mapping = slot_mapping;
  p.dev_err = dev_err;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.num_tokens = num_tokens;
  p.n_kv = n_kv_heads;
  p.head_dim = head_dim;
  p.num_blocks = num_blocks;
  return cuda_status(pa::launch_reshape_and_cache(p, src_dtype, cache_dtype,
                                                  static_cast<cudaStream_t>(stream)));
}

pa_status pa_copy_blocks(void* k_pool, void* v_pool, const int64_t* block_pairs, int n_pairs,
                         int n_kv_heads, int head_dim, int block_size, int num_blocks,
                         pa_dtype kv_dtype, int32_t* dev_err, void* stream) {
  if (block_size != 16) return PA_ERR_UNSUPPORTED;
  if (n_pairs < 0 || n_kv_heads < 1 || head_dim < 1 || num_blocks < 1 || !valid_dtype(kv_dtype))
    return PA_ERR_INVALID_ARG;
  const int64_t bb = (int64_t)n_kv_heads * 16 * head_dim * elem_bytes(kv_dtype);
  if (bb % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (n_pairs == 0) return PA_OK;
  if (!k_pool || !v_pool || !block_pairs || !aligned16(k_pool) || !aligned16(v_pool))
    return PA_ERR_INVALID_ARG;
  pa::CopyParams p;
  p.dst_k = k_pool;
  p.dst_v = v_pool;
  p.src_k = k_pool;
  p.src_v = v_pool;
  p.pairs = block_pairs;
  p.dev_err = dev_err;
  p.n_pairs = n_pairs;
  p.src_num_blocks = p.dst_num_blocks = num_blocks;
  p.block_bytes = bb;
  return cuda_status(pa::launch_copy_blocks(p, static_cast<cudaStream_t>(stream)));
}

// The address a kernel on the current device uses for `ptr`, which must be
// memory of that device or pinned host memory mapped into its address space
// (cudaHostAlloc / cudaMallocHost, or cudaHostRegister with
// cudaHostRegisterMapped); NULL for anything else (pageable host memory,
// another GPU's memory), which a kernel could not touch safely.
static const void* device_view(const void* ptr) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();  // clear the error this query left, so a later launch check is clean
    return nullptr;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (a.type == cudaMemoryTypeDevice) return a.device == dev ? ptr : nullptr;
  if (a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeManaged) return a.devicePointer;
  return nullptr;
}

pa_status pa_swap_blocks(void* dst_k_pool, void* dst_v_pool, const void* src_k_pool,
                         const void* src_v_pool, const int64_t* block_pairs, int n_pairs,
                         int n_kv_heads, int head_dim, int block_size, int src_num_blocks,
                         int dst_num_blocks, pa_dtype kv_dtype, int32_t* dev_err,
                         void* stream) {
  if (block_size != 16) return PA_ERR_UNSUPPORTED;
  if (n_pairs < 0 || n_kv_heads < 1 || head_dim < 1 || src_num_blocks < 1 ||
      dst_num_blocks < 1 || !valid_dtype(kv_dtype))
    return PA_ERR_INVALID_ARG;
  const int64_t bb = (int64_t)n_kv_heads * 16 * head_dim * elem_bytes(kv_dtype);
  if (bb % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (n_pairs == 0) return PA_OK;
  if (!dst_k_pool || !dst_v_pool || !src_k_pool || !src_v_pool || !block_pairs)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(dst_k_pool) || !aligned16(dst_v_pool) || !aligned16(src_k_pool) ||
      !aligned16(src_v_pool) || (reinterpret_cast<uintptr_t>(block_pairs) & 7u))
    return PA_ERR_INVALID_ARG;
  pa::CopyParams p;
  p.dst_k = const_cast<void*>(device_view(dst_k_pool));
  p.dst_v = const_cast<void*>(device_view(dst_v_pool));
  p.src_k = device_view(src_k_pool);
  p.src_v = device_view(src_v_pool);
  p.pairs = static_cast<const int64_t*>(device_view(block_pairs));
  if (!p.dst_k || !p.dst_v || !p.src_k || !p.src_v || !p.pairs) return PA_ERR_INVALID_ARG;
  p.dev_err = dev_err;
  p.n_pairs = n_pairs;
  p.src_num_blocks = src_num_blocks;
  p.dst_num_blocks = dst_num_blocks;
  p.block_bytes = bb;
  return cuda_status(pa::launch_copy_blocks(p, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
