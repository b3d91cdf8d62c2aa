/*
 * pa.h -- C ABI of the paged-KV attention library (libpa_b200.so, sm_100a).
 *
 * The operations follow three web pages on PagedAttention:
 *  [P1] "LLM inference optimization: KV cache & PagedAttention"
 *       (carlstack.gravito.dev)
 *  [P2] "vLLM explained" (jackchen890311.github.io)
 *  [P3] "Daily AI, 2026-07-31: inference serving" (k1-blog.pages.dev)
 *
 * Common conventions
 * ------------------
 *  - Pools.  k_pool and v_pool are separate device arrays laid out
 *    [num_blocks][n_kv_heads][block_size][head_dim] ("HND"): one physical block
 *    holds the 16 tokens of every KV head ([P2] "Block 的大小怎麼決定": a block
 *    spans all KV heads), and the 16 x head_dim tile of one (block, head) is
 *    contiguous.  block_size must be 16 ([P1] §三.1, [P2] "PagedAttention").
 *  - Block tables.  int32 [num_seqs][max_blocks_per_seq], row-major; entry j of
 *    a row is the physical block holding logical block j (tokens 16j..16j+15)
 *    of that sequence ([P1] §三.1 "Logical Block Table"; [P2] "PagedAttention",
 *    item 3).  Only the first ceil(context_len / 16) entries of a row are read.
 *  - Slots.  slot = physical_block * 16 + offset; a negative slot means "no
 *    slot" and is skipped.
 *  - GQA.  q head h reads kv head h / (n_q_heads / n_kv_heads) ([P2] "Block 的
 *    大小怎麼決定": GQA/MQA models have fewer KV heads).
 *  - Ownership.  Every pointer argument is owned by the caller.  Device
 *    pointers must stay valid until the work queued on `stream` has finished.
 *    The library allocates no device memory and never synchronises with the
 *    device on these paths; all work is queued on `stream` (a cudaStream_t;
 *    NULL means the legacy default stream).
 *  - Errors.  Argument errors are detected on the host before anything is
 *    launched and return PA_ERR_INVALID_ARG or PA_ERR_UNSUPPORTED.  A failed
 *    launch returns PA_ERR_CUDA.  Data-dependent faults that only the device
 *    can see (a block id outside [0, num_blocks), a slot outside the pool) are
 *    never trapped: the offending element is skipped and, when `dev_err` is
 *    non-NULL, bits of PA_DEVERR_* are OR-ed into *dev_err (a device int32 the
 *    caller zeroes).  Bounded waits inside kernels that give up set
 *    PA_DEVERR_TIMEOUT instead of hanging.
 *  - Thread safety.  The kernels' entry points may be called from several host
 *    threads.  A pa_alloc handle must not be used by two threads at once.
 */
#ifndef PA_B200_H
#define PA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ABI_VERSION 2

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,
    PA_ERR_UNSUPPORTED = 2,
    PA_ERR_OOM = 3,
    PA_ERR_CUDA = 4
} pa_status;

typedef enum {
    PA_F32 = 0,
    PA_F16 = 1,
    PA_BF16 = 2,
    PA_FP8_E4M3 = 3 /* OCP E4M3FN; stored value x per-tensor scale */
} pa_dtype;

/* bits OR-ed into *dev_err */
#define PA_DEVERR_BLOCK_ID 1  /* a block-table entry outside [0, num_blocks) */
#define PA_DEVERR_SLOT 2      /* a slot or block-pair id outside the pool */
#define PA_DEVERR_TIMEOUT 4   /* a bounded wait inside a kernel gave up */
#define PA_DEVERR_QUERY_LOC 8 /* inconsistent query_start_loc / context_lens */

int pa_abi_version(void);
const char* pa_status_string(pa_status s);

/* ------------------------------------------------------------------------- */
/* Decode attention                                                           */
/* ------------------------------------------------------------------------- */

/*
 * pa_decode -- one new query token per running sequence attends to that
 * sequence's whole cached context through its block table:
 *     out[s][h] = softmax(scale * q[s][h] . K_s^T) . V_s
 * ([P1] §二 Attention formula; [P1] §一.2: decode re-reads the whole KV cache
 * every step; [P2] "兩層實作": the kernel reads K/V by jumping through the
 * block table, and paging leaves the result equal to ordinary attention).
 * K_s / V_s are the first context_lens[s] tokens of sequence s; context_lens
 * includes the current token, whose K/V pa_reshape_and_cache wrote earlier in
 * the step.  A sequence with context 0 gets an all-zero output row.
 *
 *   out          device [num_seqs][n_q_heads][head_dim], dtype q_dtype
 *   q            device [num_seqs][n_q_heads][head_dim], dtype q_dtype
 *   k_pool/v_pool device pools (see conventions), dtype kv_dtype
 *   block_tables device int32 [num_seqs][max_blocks_per_seq]
 *   context_lens device int32 [num_seqs], each in [0, 16 * max_blocks_per_seq]
 *   scale        multiplies q . k (usually 1/sqrt(head_dim))
 *   k_scale, v_scale  per-tensor dequantisation scales, used only when
 *                kv_dtype is PA_FP8_E4M3 (an element's value is code x scale)
 *   workspace    device scratch of at least pa_decode_workspace_size(...)
 *                bytes, 16-byte aligned; contents need no initialisation
 *   dev_err      optional device int32 for PA_DEVERR_* bits
 *
 * Supported: block_size 16; head_dim 64 or 128; n_q_heads % n_kv_heads == 0
 * with group size n_q_heads / n_kv_heads <= 8; (q_dtype, kv_dtype) in
 * {(F32,F32), (F16,F16), (BF16,BF16), (F16,FP8_E4M3), (BF16,FP8_E4M3)}.
 * 16-bit caches multiply in the cache's type; with an fp8 cache the E4M3
 * values widen to f16 exactly and a bf16 query head is multiplied by a power
 * of two that puts its largest magnitude in [2^14, 2^15) before its f16
 * rounding, its scores by the inverse, so the whole bf16 range is taken.
 * Pointers must be 16-byte aligned.  Output rows are bit-identical under any
 * permutation of the physical blocks (partitioning and reduction order depend
 * only on logical positions).
 *
 * The work is split along the context into fixed partitions of 1024 tokens
 * (16-bit and fp32 caches) or 2048 tokens (fp8 caches): a partition kernel
 * writes per-partition (max, sum, unnormalised output) into the workspace and
 * a reduce kernel merges the partitions of sequences that have more than one.
 * pa_decode queues both; pa_decode_partitions and pa_decode_reduce queue them
 * one at a time (same arguments, same result).  pa_decode_workspace_size does
 * not depend on the dtypes (it is sized for 1024-token partitions) and is 0
 * when every sequence fits one partition; the workspace may then be NULL.
 */
size_t pa_decode_workspace_size(int num_seqs, int n_q_heads, int head_dim,
                                int max_blocks_per_seq);

pa_status pa_decode(void* out, const void* q, const void* k_pool, const void* v_pool,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    int block_size, int n_q_heads, int n_kv_heads, int head_dim,
                    int num_seqs, int max_blocks_per_seq, int num_blocks,
                    pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
                    void* workspace, size_t workspace_bytes, int32_t* dev_err,
                    void* stream);

pa_status pa_decode_partitions(void* out, const void* q, const void* k_pool,
                               const void* v_pool, const int32_t* block_tables,
                               const int32_t* context_lens, float scale, int block_size,
                               int n_q_heads, int n_kv_heads, int head_dim, int num_seqs,
                               int max_blocks_per_seq, int num_blocks, pa_dtype q_dtype,
                               pa_dtype kv_dtype, float k_scale, float v_scale,
                               void* workspace, size_t workspace_bytes, int32_t* dev_err,
                               void* stream);

pa_status pa_decode_reduce(void* out, const int32_t* context_lens, int n_q_heads,
                           int head_dim, int num_seqs, int max_blocks_per_seq,
                           pa_dtype q_dtype, pa_dtype kv_dtype, float v_scale,
                           const void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode_multi -- decode with q_len new queries per sequence, as when the
 * target model verifies K draft tokens in one forward pass ([P1] §五
 * "Speculative Decoding": the large model evaluates all K candidates in a
 * single pass; [P3] "推測解碼": the k guessed tokens are checked in parallel).
 * The K/V of all q_len tokens must already be in the cache
 * (pa_reshape_and_cache), so context_lens[s] counts them; query i of sequence
 * s (0 <= i < q_len) sits at position context_lens[s] - q_len + i and attends
 * causally to keys 0 .. context_lens[s] - q_len + i:
 *     out[s][i][h] = softmax(scale * q[s][i][h] . K_s[0..c_i]^T) . V_s[0..c_i]
 * A query whose position is negative (context_lens[s] < q_len - i) has no
 * keys and gets an all-zero row.  This is the causal chunk of
 * pa_prefill_paged with history context_lens[s] - q_len, and each K/V tile is
 * read once for all of a sequence's queries of a kv head.  Routes (head_dim
 * 128, group size 1, 2, 4 or 8, q_len >= 2):
 *  - bf16 or f16 queries over a cache of the same type: a multi-query
 *    tensor-core kernel.  The q_len x G (query, head) rows of a kv head are
 *    one 64-row tcgen05 tile; persistent CTAs, one per SM, take equal shares
 *    of the work measured in 128-key tiles (plus a fixed cost per (sequence,
 *    kv head)); a (sequence, kv head) whose keys are split between two CTAs
 *    leaves its partial results in the workspace (the slots of its 1024-token
 *    partitions) and a merge kernel combines them, all others are written
 *    whole.  P enters O += P V as a bf16 value plus its bf16 residual (f16
 *    queries: one f16 value).
 *  - bf16 queries over an fp8 cache: pa_prefill_paged's tensor-core kernel
 *    (one 128-row tile per (sequence, kv head); the workspace is not written).
 *  - otherwise: decode's partition and merge kernels with up to 32 (query,
 *    head) pairs per tile pass.
 *
 *   out, q       device [num_seqs][q_len][n_q_heads][head_dim], dtype q_dtype
 *   q_len        1 .. 8 (1 gives pa_decode's result)
 *   workspace    >= pa_decode_workspace_size(num_seqs, n_q_heads * q_len,
 *                head_dim, max_blocks_per_seq) bytes, 16-byte aligned (may be
 *                NULL when that size is 0); scratch, contents on entry
 *                ignored
 *   other arguments as pa_decode.
 *
 * Supported as pa_decode except q_dtype PA_F32 (PA_ERR_UNSUPPORTED);
 * q_len outside 1..8 is PA_ERR_INVALID_ARG.  Errors as pa_decode.
 */
pa_status pa_decode_multi(void* out, const void* q, const void* k_pool, const void* v_pool,
                          const int32_t* block_tables, const int32_t* context_lens, float scale,
                          int block_size, int n_q_heads, int n_kv_heads, int head_dim,
                          int num_seqs, int q_len, int max_blocks_per_seq, int num_blocks,
                          pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
                          void* workspace, size_t workspace_bytes, int32_t* dev_err,
                          void* stream);

/*
 * pa_decode_shared_prefix -- pa_decode's result, reading each block that a
 * group of sequences shares at the start of their tables once for the whole
 * group: the samples of one prompt share its blocks ([P1] §三.2: parallel
 * sampling forks share physical blocks; [P2] "帶來的好處"), so attention over
 * the shared prefix is one pass over those K/V for all members' queries (one
 * (member, head) pair per MMA column) instead of one pass per member.
 *
 * Group g has members group_members[g][0 .. group_width) (sequence indices;
 * -1 pads) whose tables hold the same ids in their first
 * group_shared_blocks[g] entries, all within every member's context;
 * seq_group[s] is the group of sequence s or -1.  The group pass computes the
 * context partitions (see pa_decode) that lie wholly inside a group's shared
 * blocks, for every member at once; each sequence's own pass computes its
 * other partitions; the merge is pa_decode's.  pa_prefix_groups builds these
 * arrays from host copies of the block tables.
 *
 *   group_members, group_shared_blocks, seq_group  device int32 arrays
 *   group_width  members per group; group_width x (n_q_heads / n_kv_heads)
 *                must be <= 32
 *   other arguments as pa_decode (same workspace size).
 * n_groups == 0 gives pa_decode.  Supported: q_dtype F16 or BF16 when
 * n_groups > 0.  Group arrays that break the contract above give wrong
 * results, not memory errors: every index is range-checked on the device.
 */
pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_pool,
                                  const void* v_pool, const int32_t* block_tables,
                                  const int32_t* context_lens, float scale, int block_size,
                                  int n_q_heads, int n_kv_heads, int head_dim, int num_seqs,
                                  int max_blocks_per_seq, int num_blocks, pa_dtype q_dtype,
                                  pa_dtype kv_dtype, float k_scale, float v_scale,
                                  const int32_t* group_members, const int32_t* group_shared_blocks,
                                  const int32_t* seq_group, int n_groups, int group_width,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_err,
                                  void* stream);

/*
 * pa_prefix_groups -- host helper for pa_decode_shared_prefix: groups the
 * sequences whose tables start with the same block (in index order, at most
 * 32 / (n_q_heads / n_kv_heads) per group) and records how many leading
 * blocks all members share, within their full blocks; groups sharing less
 * than one whole partition, and single sequences, are dropped.
 * *group_width_out is the largest group's size (the row stride of
 * group_members_out).
 *
 *   block_tables, context_lens  host copies ([num_seqs][max_blocks_per_seq],
 *                [num_seqs])
 *   group_members_out  host int32 of num_seqs x 32 / G entries
 *   group_shared_blocks_out, seq_group_out  host int32 [num_seqs]
 */
pa_status pa_prefix_groups(const int32_t* block_tables, const int32_t* context_lens,
                           int num_seqs, int max_blocks_per_seq, int n_q_heads, int n_kv_heads,
                           pa_dtype kv_dtype, int32_t* group_members_out,
                           int32_t* group_shared_blocks_out, int32_t* seq_group_out,
                           int* n_groups_out, int* group_width_out);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory and therefore have no workspace to pass: for example a plugin inside
 * a host program that owns all device memory and forbids cudaMalloc after
 * start-up, or a loop that cannot afford cudaMalloc's implicit device
 * synchronisation.  The pages have no counterpart to this: it is a packaging
 * of pa_decode, not part of the method.
 *
 * Same arguments and results as pa_decode without the workspace.  The
 * per-partition results go to a scratch array built into the library (a
 * file-scope __device__ array of pa_decode_noalloc_scratch_bytes() = 16 MiB;
 * every GPU that loads the library holds it until the process exits).  The
 * call makes no cudaMalloc, cudaFree or other allocating call.
 *  - Returns PA_ERR_UNSUPPORTED before any launch when the call would need more
 *    scratch than that, i.e. when pa_decode_workspace_size(num_seqs, n_q_heads,
 *    head_dim, max_blocks_per_seq) > pa_decode_noalloc_scratch_bytes().
 *  - The array's device address belongs to a CUDA context.  The first call
 *    made with a given context current (the device's primary context, or a
 *    driver-API context the caller made current) looks it up and caches it
 *    under that context's id; make that first call before any stream capture.
 *    A context created later (for instance after cudaDeviceReset) has a new
 *    id and gets a fresh lookup, so an address cached for a destroyed context
 *    is never used.
 *  - All calls share the one array, which keeps the last call's contents:
 *    calls whose work overlaps on the GPU (other streams, other host threads)
 *    race on it and must be ordered by the caller.  Nothing in it needs to
 *    start at zero.
 */
size_t pa_decode_noalloc_scratch_bytes(void);

pa_status pa_decode_noalloc(void* out, const void* q, const void* k_pool, const void* v_pool,
                            const int32_t* block_tables, const int32_t* context_lens,
                            float scale, int block_size, int n_q_heads, int n_kv_heads,
                            int head_dim, int num_seqs, int max_blocks_per_seq, int num_blocks,
                            pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
                            int32_t* dev_err, void* stream);

/*
 * pa_test_decode_timeout -- a test hook for the error path of the kernels'
 * bounded waits; the pages have no counterpart to it.  It queues pa_decode
 * (same arguments, q_dtype F16 or BF16) with every wait in the partition
 * kernel giving up after wait_limit_us microseconds (1 .. 1,000,000; the
 * library's own limit is 1 s) and with each CTA's producer warp leaving the
 * shared-memory stage of its tile `skip_tile` unfilled, as if its load had
 * never arrived.  The waits on that stage run out: the kernel sets
 * PA_DEVERR_TIMEOUT in *dev_err, lets the loads it did issue land, and
 * returns; the output is meaningless, the context stays usable, and the next
 * call computes normally.  PA_ERR_INVALID_ARG for skip_tile < 0 or a limit
 * out of range.
 */
pa_status pa_test_decode_timeout(void* out, const void* q, const void* k_pool,
                                 const void* v_pool, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, int block_size,
                                 int n_q_heads, int n_kv_heads, int head_dim, int num_seqs,
                                 int max_blocks_per_seq, int num_blocks, pa_dtype q_dtype,
                                 pa_dtype kv_dtype, float k_scale, float v_scale, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_err, void* stream,
                                 int skip_tile, uint32_t wait_limit_us);

/* ------------------------------------------------------------------------- */
/* Chunked prefill                                                            */
/* ------------------------------------------------------------------------- */

/*
 * pa_prefill_paged -- chunked prefill: a long prompt is cut into chunks that
 * are batched with decodes ([P1] §六.2 "Chunked Prefill"; [P2] "附錄與延伸").
 * Chunk c owns query rows query_start_loc[c] .. query_start_loc[c+1]-1 (L_c
 * rows) and its sequence holds context_lens[c] tokens including the chunk, so
 * its history is H_c = context_lens[c] - L_c.  The chunk's K/V must already be
 * in the pools (pa_reshape_and_cache).  Query i of the chunk sits at absolute
 * position H_c + i and attends causally to keys 0 .. H_c + i:
 *     out[r][h] = softmax(scale * q[r][h] . K^T, masked) . V
 * The prefill half of a batch is compute-bound ([P1] §一.1; [P3] "prefill 與
 * decode"); this kernel runs the two contractions on tcgen05 tensor cores.
 *
 *   out, q         device [total_q][n_q_heads][head_dim], dtype q_dtype,
 *                  total_q = query_start_loc[n_chunks]
 *   block_tables   device int32 [n_chunks][max_blocks_per_seq]
 *   query_start_loc device int32 [n_chunks + 1], non-decreasing, [0] = 0
 *   context_lens   device int32 [n_chunks], context_lens[c] >= L_c
 *   max_chunk_len  host bound on every L_c (sizes the grid; no device sync)
 *
 * Supported: block_size 16, head_dim 128, group size 1, 2, 4 or 8, q_dtype
 * BF16 and kv_dtype BF16 or FP8_E4M3.  Both products accumulate in fp32 and
 * take every input value exactly, over the whole bf16 range ([P2] "兩層實作":
 * paging leaves the math unchanged):
 *  - bf16 cache: q, K and V enter the tensor cores as bf16; the softmax
 *    weights P enter O += P V as a bf16 value plus its bf16 rounding residual
 *    (about 16 significant bits);
 *  - fp8 cache: E4M3 values widen to f16 exactly; each bf16 query row is
 *    multiplied by a power of two that puts its largest magnitude in
 *    [2^14, 2^15) before its f16 rounding and its scores by the inverse (an
 *    element below 2^-28 of its row's largest keeps an absolute precision of
 *    2^-39 of that largest); P is f16.
 * A block id outside [0, num_blocks) is flagged with PA_DEVERR_BLOCK_ID and
 * its keys read as zeros.  The output is written in q_dtype.
 * PA_ERR_UNSUPPORTED also when num_blocks * n_kv_heads * 16 >= 2^31 (the pools
 * are addressed as that many rows of head_dim elements).
 *
 *   workspace      NULL, or device memory of at least
 *                  pa_prefill_workspace_size(n_chunks, n_kv_heads, head_dim,
 *                  max_blocks_per_seq, block_size) bytes, 16-byte aligned,
 *                  owned by the caller and free for this call's duration.
 * fp8 cache: with NULL every query tile widens the K/V it reads to f16
 * itself; with a workspace a first kernel widens each chunk's history once
 * (per kv head) into it, and the tensor-core kernel streams the f16 operands
 * from there, every query tile of a chunk sharing them.  The results are
 * identical up to the order of the fp32 accumulation (the same f16 operands
 * either way).  bf16 cache: the kernel reads the pool's blocks directly and
 * a workspace, if given, is checked but not used.
 * PA_ERR_INVALID_ARG if the workspace is too small or misaligned;
 * PA_ERR_UNSUPPORTED if n_chunks * n_kv_heads * (max_blocks_per_seq * 16
 * rounded up to 128) >= 2^31.
 */
size_t pa_prefill_workspace_size(int n_chunks, int n_kv_heads, int head_dim,
                                 int max_blocks_per_seq, int block_size);
pa_status pa_prefill_paged(void* out, const void* q, const void* k_pool, const void* v_pool,
                           const int32_t* block_tables, const int32_t* query_start_loc,
                           const int32_t* context_lens, float scale, int block_size,
                           int n_q_heads, int n_kv_heads, int head_dim, int n_chunks,
                           int max_chunk_len, int max_blocks_per_seq, int num_blocks,
                           pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale,
                           float v_scale, void* workspace, size_t workspace_bytes,
                           int32_t* dev_err, void* stream);

/* ------------------------------------------------------------------------- */
/* Slot write and copy-on-write block copy                                    */
/* ------------------------------------------------------------------------- */

/*
 * pa_reshape_and_cache -- write each new token's K and V rows into the slot
 * its position maps to (the block table gives the block, the position modulo
 * 16 the offset; [P2] "PagedAttention" items 1-4, [P1] §三.1).
 *
 *   key, value   device [num_tokens][n_kv_heads][head_dim], dtype src_dtype
 *   slot_mapping device int64 [num_tokens]; < 0 skips the token; slots must be
 *                distinct (two tokens writing one slot race)
 *   cache_dtype  == src_dtype: bytes are copied;
 *                PA_FP8_E4M3 (src F16/BF16/F32): code = RNE_satfinite(x / scale)
 *                with the quotient taken in binary32, k_scale for K and
 *                v_scale for V ([P2] "Block 的大小怎麼決定": FP8 is 1 byte).
 * Out-of-range slots are skipped and flagged with PA_DEVERR_SLOT.
 */
pa_status pa_reshape_and_cache(void* k_pool, void* v_pool, const void* key, const void* value,
                               const int64_t* slot_mapping, int num_tokens, int n_kv_heads,
                               int head_dim, int block_size, int num_blocks,
                               pa_dtype src_dtype, pa_dtype cache_dtype, float k_scale,
                               float v_scale, int32_t* dev_err, void* stream);

/*
 * pa_copy_blocks -- the copy half of copy-on-write: when a branch is about to
 * write into a block it shares, the block is first copied to a private one
 * ([P1] §三.2; [P2] "帶來的好處").  For each pair (src, dst) the whole dst
 * block (every KV head, K and V) becomes a byte copy of the src block.
 *
 *   block_pairs  device int64 [n_pairs][2] = (src, dst); dst ids must be
 *                distinct and must not appear as a src (pa_alloc_prepare_write
 *                produces such pairs).  Ids outside [0, num_blocks) are skipped
 *                and flagged with PA_DEVERR_SLOT.
 */
pa_status pa_copy_blocks(void* k_pool, void* v_pool, const int64_t* block_pairs, int n_pairs,
                         int n_kv_heads, int head_dim, int block_size, int num_blocks,
                         pa_dtype kv_dtype, int32_t* dev_err, void* stream);

/*
 * pa_swap_blocks -- move whole blocks between two pools, e.g. a preempted
 * request's blocks from the GPU pool to a host pool and later back ([P2]
 * "KV cache 什麼時候可以被覆蓋": when memory runs short a request is
 * preempted by recomputation or by swapping its KV cache to the CPU).  For
 * each pair (src, dst), block dst of (dst_k_pool, dst_v_pool) becomes a byte
 * copy of block src of (src_k_pool, src_v_pool), every KV head, K and V.  One
 * kernel moves all pairs; host blocks cross the host link as the kernel's own
 * loads and stores.
 *
 *   pools        each either memory of the current device or pinned host
 *                memory mapped into the device's address space (cudaHostAlloc
 *                / cudaMallocHost, or cudaHostRegister with
 *                cudaHostRegisterMapped), [num_blocks][n_kv][16][head_dim],
 *                16-byte aligned; src and dst pools must not overlap
 *   block_pairs  int64 [n_pairs][2] = (src, dst) in the same kinds of memory;
 *                dst ids distinct.  Ids outside [0, src_num_blocks) /
 *                [0, dst_num_blocks) are skipped and flagged with
 *                PA_DEVERR_SLOT.
 * Pointers to pageable host memory or to another GPU's memory are refused
 * with PA_ERR_INVALID_ARG before any launch.
 */
pa_status pa_swap_blocks(void* dst_k_pool, void* dst_v_pool, const void* src_k_pool,
                         const void* src_v_pool, const int64_t* block_pairs, int n_pairs,
                         int n_kv_heads, int head_dim, int block_size, int src_num_blocks,
                         int dst_num_blocks, pa_dtype kv_dtype, int32_t* dev_err,
                         void* stream);

/* ------------------------------------------------------------------------- */
/* Host block allocator (not on the hot path)                                 */
/* ------------------------------------------------------------------------- */

/*
 * The memory-management layer: fixed-size blocks, a block table per
 * sequence, allocation on demand, release when a request finishes
 * ([P2] "PagedAttention" items 1-4, "兩層實作"), sharing by reference count and
 * copy-on-write ([P1] §三.2), and a block in use is never handed out again
 * ([P2] "KV cache 什麼時候可以被覆蓋").
 *
 * Free blocks are handed out FIFO from `initial_free_order` (NULL: 0..N-1;
 * otherwise a permutation of 0..N-1) and freed blocks join the back of the
 * queue, so the state after any call sequence is deterministic.  Every call is
 * all-or-nothing: PA_ERR_OOM or PA_ERR_INVALID_ARG leave the state unchanged.
 * Sequence ids are arbitrary int64 values.  Handles are not thread-safe.
 *
 * Prefix caching ([P2] "Prefix Caching：相同前綴只算一次"), off unless
 * pa_alloc_set_prefix_caching switches it on: a block is in use (count > 0),
 * free and empty, or free but holding cached content (count 0).  A full block
 * whose token ids are known (pa_alloc_admit, pa_alloc_append_tokens) is
 * registered under a 64-bit hash of its whole prefix, checked on a hit
 * against its stored 16 tokens and its parent's hash.  pa_alloc_admit reuses
 * the longest run of leading full blocks of a prompt held by a block in use
 * or cached.  A new block is an empty one (FIFO) if any is left, else the
 * least recently released cached block, whose registration is dropped; a
 * block in use is never taken.  When a request ends, its registered blocks
 * whose count reaches 0 become cached (the back of the LRU list) and the
 * others empty.  A block whose prefix is already registered by another block
 * stays unregistered; a partial last block is never registered.  Callers
 * write the K/V of a registered block's tokens before any attention reads
 * them (slot writes precede attention within a step).
 */
typedef struct pa_alloc pa_alloc;

/* NULL on invalid arguments (num_blocks < 1, block_size != 16, bad order) */
pa_alloc* pa_alloc_create(int num_blocks, int block_size, const int32_t* initial_free_order);
void pa_alloc_destroy(pa_alloc* a);

/* Reserve slots for n_tokens new tokens of `seq` (created on first use),
 * taking new blocks when the last one is full.  slots_out[n_tokens] receives
 * their slots (may be NULL when n_tokens == 0).  Refused with
 * PA_ERR_INVALID_ARG while the last block is partially filled and shared:
 * call pa_alloc_prepare_write first. */
pa_status pa_alloc_append(pa_alloc* a, int64_t seq, int n_tokens, int64_t* slots_out);

/* `child` (new id) gets the parent's table; every block's count goes up by 1. */
pa_status pa_alloc_fork(pa_alloc* a, int64_t parent, int64_t child);

/* If the last block of `seq` is partially filled and shared, move `seq` to a
 * fresh block and report the pair (old, new) that pa_copy_blocks must copy
 * before the next write; cow_pairs_out has room for one pair (2 int64).
 * *n_pairs_out is 0 or 1. */
pa_status pa_alloc_prepare_write(pa_alloc* a, int64_t seq, int64_t* cow_pairs_out,
                                 int* n_pairs_out);

/* Drop `seq`; each of its blocks' counts goes down by 1, last block first,
 * and a block whose count reaches 0 joins the back of the free queue (or,
 * with prefix caching, of the cached list if it is registered). */
pa_status pa_alloc_free_seq(pa_alloc* a, int64_t seq);

/* Copy the block table of `seq` (logical order) into out[cap]; *n_out gets
 * its length.  PA_ERR_INVALID_ARG if cap is too small or seq is unknown. */
pa_status pa_alloc_block_table(const pa_alloc* a, int64_t seq, int32_t* out, int cap,
                               int* n_out);
/* Copy the free queue of empty blocks (front first) into out[cap]. */
pa_status pa_alloc_free_list(const pa_alloc* a, int32_t* out, int cap, int* n_out);
int pa_alloc_num_tokens(const pa_alloc* a, int64_t seq); /* -1 if unknown */
int pa_alloc_refcount(const pa_alloc* a, int32_t block); /* -1 if out of range */
int pa_alloc_num_free(const pa_alloc* a);   /* empty free blocks */
int pa_alloc_num_seqs(const pa_alloc* a);

/* Switch prefix caching on (on != 0) or off; PA_ERR_INVALID_ARG while any
 * sequence exists. */
pa_status pa_alloc_set_prefix_caching(pa_alloc* a, int on);

/* Start sequence `seq` (a new id) with a prompt of n_tokens known token ids.
 * With prefix caching on, the longest run of the prompt's leading full blocks
 * whose prefixes are registered is reused (counts + 1, cached blocks back in
 * use); *n_cached_out = 16 x that run: those tokens' K/V are already in the
 * cache and need no prefill.  The rest get new blocks.  slots_out[n_tokens]
 * receives every token's slot, reused ones included.  PA_ERR_OOM when the new
 * blocks cannot all be had (state unchanged). */
pa_status pa_alloc_admit(pa_alloc* a, int64_t seq, const int32_t* tokens, int n_tokens,
                         int64_t* slots_out, int* n_cached_out);

/* pa_alloc_append for tokens whose ids are known: as long as every token of
 * `seq` has come with its id, blocks it fills are registered.  (Plain
 * pa_alloc_append makes a sequence's ids unknown from then on.) */
pa_status pa_alloc_append_tokens(pa_alloc* a, int64_t seq, const int32_t* tokens,
                                 int n_tokens, int64_t* slots_out);

/* Copy the cached blocks (count 0, content kept), least recently released
 * first, into out[cap]. */
pa_status pa_alloc_cached_list(const pa_alloc* a, int32_t* out, int cap, int* n_out);
int pa_alloc_num_cached(const pa_alloc* a);

#ifdef __cplusplus
}
#endif
#endif /* PA_B200_H */
