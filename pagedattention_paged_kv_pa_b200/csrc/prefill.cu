// Chunked prefill over the paged cache on tcgen05 tensor cores (sm_100a).
//
// A long prompt is cut into chunks that run next to decodes ("LLM inference
// optimization: KV cache & PagedAttention", §六.2; "vLLM explained",
// "附錄與延伸").  Chunk c holds L queries at absolute positions H..H+L-1 over
// a paged history of H tokens; query i attends causally to keys 0..H+i.  With
// many queries per chunk the two products are real dense contractions, so
// they run on the 5th-generation tensor cores with accumulators in TMEM.
//
// CTA tile: M = 128 rows = (128 / G) consecutive queries x the G query heads
// of one kv head (GQA packing: each K/V tile serves the whole group).  Keys
// are processed in tiles of 128 (8 blocks of 16 from the block table).
//
// The paged kernel must not change the math ("vLLM explained", "兩層實作"), so
// every operand reaches the tensor cores exactly:
//
// bf16 cache (kDirectBf16, 320 threads): Q, K and V stay bf16 and both
// products run as kind::f16 MMAs with bf16 operands.  A TMA warp loads each
// full 16-token block of a tile straight from the pools (two 64-column boxes
// per operand, the block table giving the row); the warp itself writes the
// rows of a block the context ends in (its valid rows, zeros after them), of
// blocks past the context and of blocks with an out-of-range id (zeros,
// flagged).  P = 2^(s - m) enters O += P V as a bf16 value plus its bf16
// rounding residual (two MMAs into the same TMEM accumulator): ~16
// significant bits, where one bf16 P would cost up to 2^-9 |v - o| on short
// contexts.  No workspace is needed.
//
// fp8 cache: E4M3 values widen to f16 exactly, so the products run in f16.  A
// bf16 query row is multiplied by the power of two 2^e that brings its largest
// magnitude into [2^14, 2^15) before it is rounded to f16 (every element at
// least 2^-28 of the row's largest keeps all of its bits; smaller ones keep
// an absolute precision of 2^-39 of it), and that row's score scale is
// multiplied by 2^-e -- exact, and free in the loop.  P is f16 (11
// significant bits).  The operands come one of two ways:
//
// With a workspace (kStaged, 320 threads): prefill_widen_kernel first writes
// each chunk's history, per kv head, as f16 rows (zeros past the context), so
// the 16 query tiles of a 512-query chunk share one widening instead of each
// doing its own, and a TMA warp streams two 64-column boxes per operand into
// 3 K and 2 V stages.
//
// Without one (kWidenFp8, 320 threads): one softmax warp per row (warps 0-3)
// and converter warps 4-7 that widen each tile themselves and write both
// operands as [key][d] rows in the 128-byte-swizzled layout (K-major for K,
// MN-major for V, so V needs no transpose): K on the conversion pipe, V on the
// integer pipe as code x 2^-8 (folded into the output scale); warp 9 brings
// each tile's raw rows into a 2-stage shared-memory ring by TMA, two tiles
// ahead.
//
// Two-warps-per-row softmax (kDirectBf16, kStaged): warps w and w+4 own rows
// 32 (w%4) .. +31 (TMEM lanes) and take half a key tile each; they read S from
// TMEM, mask, keep an online max/sum (the halves' maxima meet in shared
// memory at a named barrier), write P back to TMEM, rescale their half of the
// TMEM output only when the max grew by more than 2^8, and write the
// normalised output at the end.  Warp 8 owns TMEM and issues the MMAs from one
// lane: S = Q K^T into a double-buffered TMEM score tile, O += P V into TMEM
// with P read from TMEM.  K stages are released as soon as S = Q K^T has read
// them, V stages once O += P V has.  S(j+1) is issued before O += P(j) V(j),
// so the next tile's QK^T overlaps this tile's softmax.  All waits are
// bounded; a wait that gives up flags PA_DEVERR_TIMEOUT, the CTA drains its
// tensor-core work and loads in flight and frees its TMEM before returning.
#include <type_traits>
#include <utility>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int D = 128;       // head dim
constexpr int BM = 128;      // rows per CTA tile
constexpr int BN = 128;      // keys per tile
// TMEM columns: S[2] (2 x 128 fp32), O (128 fp32), then P: two buffers of 64
// columns of f16 pairs (fp8 cache), or one buffer of bf16 pairs with its
// residual pairs in the next 64 columns (bf16 cache)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (factor 256)

// Where the K/V operands come from:
//   kWidenFp8: warps 4-7 widen each tile's fp8 rows to f16 in shared memory,
//     after a tenth warp has brought the raw rows into a 2-stage ring by TMA;
//   kStaged: the chunk's fp8 history was widened once into an f16 workspace by
//     prefill_widen_kernel (all query tiles of a chunk and kv head share it),
//     and a TMA warp streams ready operands; there are no converter warps;
//   kDirectBf16: a TMA warp streams the bf16 pool's blocks themselves.
enum Mode : int { kWidenFp8 = 0, kStaged = 1, kDirectBf16 = 2 };

// shared-memory map (offsets from a 1024-aligned base)
constexpr int kOpBytes = BM * D * 2;  // one 128x128 16-bit operand = 32 KiB
constexpr int kRawBytes = BN * D;     // one tile's fp8 K (or V) rows = 16 KiB
constexpr int kMaxKStages = 3, kMaxVStages = 2, kRawStages = 2;
template <int MODE>
struct Layout {
  static constexpr bool kTmaOps = MODE != kWidenFp8;  // operands arrive by TMA, no converters
  static constexpr bool kRawRing = MODE == kWidenFp8;
  static constexpr bool kBf16 = MODE == kDirectBf16;  // bf16 MMAs, P as value + residual
  static constexpr int kPBufs = kBf16 ? 1 : 2;         // P buffers in TMEM
  // TMA-fed kernels split each row's softmax over kParts warps (4 kParts
  // softmax warps, kParts per TMEM lane quadrant); the in-kernel widening
  // keeps one softmax warp per quadrant and 4 converter warps
  static constexpr bool kSplitSoftmax = kTmaOps;
  // parts per row: the length of a softmax warp's chain per tile is what
  // bounds it.  bf16 (also multi-query decode, whose few rows fill only
  // two TMEM lane quadrants, i.e. two of the four SM sub-partitions): 4
  // parts of 32 keys; fp8 from the workspace (all quadrants busy): 2 of 64,
  // which measured faster than 4 there
  static constexpr int kParts = !kSplitSoftmax ? 1 : (kBf16 ? 4 : 2);
  // two parts per row keep independent softmax states, each with its own O
  // accumulator (the two 128-column O tiles take the TMEM the P buffers had;
  // P goes over the part's own S columns), so no per-tile max exchange ties
  // the row's two warps together; they merge once at the end
  static constexpr bool kIndep = kSplitSoftmax && kParts == 2;
  static constexpr int kSoftWarps = 4 * kParts;
  static constexpr int kMmaWarp = kSplitSoftmax ? kSoftWarps : 8;
  // one load warp takes K then V of each tile (a second warp for V measured
  // no faster, and with 4 parts it would cut the registers a thread may hold)
  static constexpr int kLoadWarp = kMmaWarp + 1;
  static constexpr int kThreads = (kLoadWarp + 1) * 32;
  static constexpr int kKStages = kTmaOps ? 3 : 2;
  static constexpr int kVStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kOpBytes;             // K stages
  static constexpr int kVOff = kKOff + kKStages * kOpBytes;  // V stages
  static constexpr int kRawOff = kVOff + kVStages * kOpBytes;  // raw fp8 K, V stages
  // split softmax: row maxima of the parts [2 parities][kParts][BM], then
  // the parts' row sums [kParts][BM]
  static constexpr int kRedOff = kRawOff + (kRawRing ? kRawStages * 2 * kRawBytes : 0);
  // per-row score scale (scale x log2 e x the row's 2^-e) [BM]
  static constexpr int kRowScaleOff = kRedOff + (kSplitSoftmax ? 3 * kParts * BM * 4 : 0);
  static constexpr int kBarOff = kRowScaleOff + BM * 4;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

// 128x128 16-bit operand with the 128-byte swizzle: 128-byte rows of 64
// elements in two 16 KiB halves; chunk = 8 consecutive elements of a row
// (0..15).  Read K-major (Q, K, P rows along K) or MN-major (V: rows are keys,
// the 64-dim halves are the MN atoms, 8-row groups the K atoms).
__device__ __forceinline__ uint32_t op_off(int row, int chunk) {
  return (chunk >> 3) * 16384 + row * 128 + ((((chunk & 7) ^ (row & 7))) << 4);
}
// ------------------------------------------------------------- tcgen05 ops
// shared-memory matrix descriptor, 128-byte swizzle: K-major operands use only
// the 8-row group stride (1 KiB); the MN-major V operand also needs the stride
// between its two 64-element MN halves (16 KiB) as the leading-dimension offset
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo = 16) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
// same with A (M x K, 16-bit pairs along K in consecutive columns) read from TMEM
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                          uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// named barrier `id` over `n` threads that also ORs a flag across them
__device__ __forceinline__ bool named_bar_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %3, 0;\n\t"
      "bar.red.or.pred p, %1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(id), "r"(n), "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
// barrier over the 128 converter threads that also ORs a flag across them
__device__ __forceinline__ bool conv_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
// KP/2 columns (KP = 32 or 64 keys as pairs) from v
template <int KP>
__device__ __forceinline__ void tmem_st_pairs(uint32_t taddr, const uint32_t* v) {
  if constexpr (KP == 64)
    tmem_st32(taddr, reinterpret_cast<const float*>(v));
  else
    tmem_st16(taddr, reinterpret_cast<const float*>(v));
}
// 2^x with the hardware approximation (relative error far below f16's 2^-11;
// results below 2^-126 flush to zero, which P can afford)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct Bars {
  uint64_t k_full[kMaxKStages], k_empty[kMaxKStages], v_full[kMaxVStages], v_empty[kMaxVStages];
  uint64_t raw_full[kRawStages], raw_empty[kRawStages];
  uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2], done;
  uint64_t pp_full[2][2];  // independent parts: P of part h in S buffer b written
  uint32_t tmem_base;
  int abort_flag;
};

// bounded wait that also honours the CTA-wide abort flag
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Bars* B,
                                              int32_t* dev_err) {
  if (mbar_wait(bar, parity)) return true;
  flag_error(dev_err, PA_DEVERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&B->abort_flag) = 1;
  return false;
}
__device__ __forceinline__ bool aborted(Bars* B) {
  return *reinterpret_cast<volatile int*>(&B->abort_flag) != 0;
}

// Rows of a block that the TMA cannot load whole (the block the context ends
// in, blocks past the context, blocks with an out-of-range id), written by
// the load warp into operand stage `op` at rows 16 m .. 16 m + 15: rows below
// `nvalid` are copied from the pool row `src_row` on, the rest are zeros.
// 16-byte chunks, eight per lane.
__device__ __forceinline__ void write_block_rows(uint8_t* op, int m, const uint8_t* pool,
                                                 long long src_row, int nvalid, int lane) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int idx = lane + 32 * u, r = idx >> 4, cc = idx & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < nvalid)
      v = __ldg(reinterpret_cast<const uint4*>(pool + (src_row + r) * (D * 2) + cc * 16));
    *reinterpret_cast<uint4*>(op + op_off(16 * m + r, cc)) = v;
  }
}

// tmk / tmv: with kWidenFp8 maps over the fp8 pools ([token rows][128]
// bytes, 16 x 128-byte boxes); with kStaged maps over the f16 workspace
// ([rows][128] f16, 64 x 128-element boxes); with kDirectBf16 maps over the
// bf16 pools ([token rows][128] bf16, 64 x 16-element boxes)
template <int MODE>
__global__ void __launch_bounds__(Layout<MODE>::kThreads, 1)
    prefill_tc_kernel(const PrefillParams p, const void* __restrict__ k_pool,
                      const void* __restrict__ v_pool, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
  using LY = Layout<MODE>;
  constexpr int kKStages = LY::kKStages, kVStages = LY::kVStages, kPB = LY::kPBufs;
  constexpr int kMmaWarp = LY::kMmaWarp, kLoadWarp = LY::kLoadWarp;
  // stage "full" barriers: a TMA transaction count or the 128 converters
  constexpr uint32_t kFullCount = LY::kTmaOps ? 1 : 128;
  constexpr int kQOff = LY::kQOff, kKOff = LY::kKOff, kVOff = LY::kVOff, kBarOff = LY::kBarOff;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars* B = reinterpret_cast<Bars*>(smem + kBarOff);
  const uint32_t sbase = smem_u32(smem);

  // query tiles later in a chunk see more keys (causal): they are launched
  // first, so the shorter ones fill the last wave
  const int tile = gridDim.x - 1 - blockIdx.x, kvh = blockIdx.y, c = blockIdx.z;
  const int G = p.group;
  const int QT = BM / G;  // queries per CTA tile
  int q0, L, ctx;
  if (p.fixed_q_len > 0) {
    // multi-query decode: sequence c's fixed_q_len queries are the last
    // positions of its context; a query before the context's start sees no
    // key.  A context beyond the table is flagged and clamped, as in decode.
    L = p.fixed_q_len;
    q0 = c * L;
    ctx = p.context_lens[c];
    if (ctx > p.max_blocks * 16) {
      if (threadIdx.x == 0 && tile == 0 && kvh == 0) flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
      ctx = p.max_blocks * 16;
    }
    ctx = max(ctx, 0);
  } else {
    q0 = p.query_start_loc[c];
    L = p.query_start_loc[c + 1] - q0;
    ctx = p.context_lens[c];
    if (L < 0 || L > p.max_chunk_len || ctx < L || ctx > p.max_blocks * 16) {
      if (threadIdx.x == 0 && tile == 0 && kvh == 0) flag_error(p.dev_err, PA_DEVERR_QUERY_LOC);
      return;
    }
  }
  const int H = ctx - L;  // negative only in multi-query decode
  const int i0 = tile * QT;
  if (i0 >= L) return;
  const int i_end = min(L, i0 + QT);
  const int n_keys = max(0, H + i_end);
  const int nkt = (n_keys + BN - 1) / BN;
  if (nkt == 0) {  // no query of this tile sees a key: all-zero rows
    for (int idx = threadIdx.x; idx < BM * (D / 8); idx += blockDim.x) {
      const int r = idx / (D / 8), i = i0 + r / G;
      if (i < L)
        reinterpret_cast<uint4*>(p.out)[((size_t)(q0 + i) * p.n_q + (size_t)kvh * G + r % G) *
                                            (D / 8) + idx % (D / 8)] = make_uint4(0, 0, 0, 0);
    }
    return;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  if (tid == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&B->k_full[s], kFullCount);
      mbar_init(&B->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&B->v_full[s], kFullCount);
      mbar_init(&B->v_empty[s], 1);
    }
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(&B->raw_full[s], 1);
      mbar_init(&B->raw_empty[s], 128);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B->s_full[s], 1);
      mbar_init(&B->s_empty[s], LY::kSoftWarps * 32);
      mbar_init(&B->p_full[s], LY::kSoftWarps * 32);
      mbar_init(&B->pp_full[0][s], LY::kSoftWarps * 16);  // the 4 warps of a part
      mbar_init(&B->pp_full[1][s], LY::kSoftWarps * 16);
      mbar_init(&B->pv_done[s], 1);
    }
    mbar_init(&B->done, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&B->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // Q tile -> shared (K-major, swizzled), one row per thread of warps 0-3.
  // bf16 cache: the bf16 row as it is.  fp8 cache: the row times 2^e, e
  // chosen from its largest magnitude, rounded to f16; the row's score scale
  // takes the 2^-e.
  float* row_scale = reinterpret_cast<float*>(smem + LY::kRowScaleOff);
  if (tid < BM) {
    const int r = tid, i = i0 + r / G, g = r % G;
    const bool valid = i < L;
    const uint4* src = reinterpret_cast<const uint4*>(
        reinterpret_cast<const __nv_bfloat16*>(p.q) +
        ((size_t)(q0 + (valid ? i : 0)) * p.n_q + (size_t)kvh * G + g) * D);
    if constexpr (LY::kBf16) {
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const uint4 v = valid ? src[ch] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(smem + kQOff + op_off(r, ch)) = v;
      }
      row_scale[r] = p.scale_log2;
    } else {
      uint4 v[16];
      uint32_t mag = 0;  // largest |x| of the row, as bf16 bits (order-preserving)
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        v[ch] = valid ? src[ch] : make_uint4(0, 0, 0, 0);
        mag = max(mag, bf16x2_max_mag(v[ch].x));
        mag = max(mag, bf16x2_max_mag(v[ch].y));
        mag = max(mag, bf16x2_max_mag(v[ch].z));
        mag = max(mag, bf16x2_max_mag(v[ch].w));
      }
      const int e = f16_row_shift(mag);
      const float up = exp2i(e);
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const uint4 w = make_uint4(bf16x2_to_f16x2_scaled(v[ch].x, up),
                                   bf16x2_to_f16x2_scaled(v[ch].y, up),
                                   bf16x2_to_f16x2_scaled(v[ch].z, up),
                                   bf16x2_to_f16x2_scaled(v[ch].w, up));
        *reinterpret_cast<uint4*>(smem + kQOff + op_off(r, ch)) = w;
      }
      row_scale[r] = p.scale_log2 * exp2i(-e);
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 256, tP = tmem + 384;

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kind::f16: D f32, N = 128, M = 128; A and B bf16 (bf16 cache) or f16
      // (fp8 cache, and P with it); B K-major for S = Q K^T, MN-major (bit
      // 16) for O += P V
      constexpr uint32_t kAB = LY::kBf16 ? ((1u << 7) | (1u << 10)) : 0u;
      const uint32_t idesc =
          (1u << 4) | kAB | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
      const uint32_t idesc_pv = idesc | (1u << 16);
      const uint32_t aQ = sbase + kQOff;
      bool ok = true;
      if constexpr (LY::kIndep) {
        // S(j) goes into TMEM buffer j % 2 once both parts' O += P V of tile
        // j - 2 -- whose P was written over that buffer -- has completed.
        // Then per tile: each part's O_h += P_h V_h (its 64 keys) as soon as
        // that part's P is written.
        auto issue_s = [&](int j) -> bool {
          const int s = j & 1, sk = j % kKStages;
          if (!wait_or_abort(&B->k_full[sk], (j / kKStages) & 1, B, p.dev_err)) return false;
          if (j >= 2 && !wait_or_abort(&B->pv_done[s], ((j - 2) >> 1) & 1, B, p.dev_err))
            return false;
          tc_fence_after();
          const uint32_t bK = sbase + kKOff + sk * kOpBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc_mma(tS + s * BN, smem_desc(aQ + off), smem_desc(bK + off), idesc, kk > 0);
          }
          tc_commit(&B->s_full[s]);
          tc_commit(&B->k_empty[sk]);  // the K stage is free once S(j) is done
          return true;
        };
        ok = issue_s(0) && (nkt < 2 || issue_s(1));
        for (int jp = 0; jp < nkt && ok; ++jp) {
          const int b = jp & 1, sv = jp % kVStages;
          ok = wait_or_abort(&B->v_full[sv], (jp / kVStages) & 1, B, p.dev_err);
          const uint32_t bV = sbase + kVOff + sv * kOpBytes;
          for (int h = 0; h < 2 && ok; ++h) {
            ok = wait_or_abort(&B->pp_full[h][b], (jp >> 1) & 1, B, p.dev_err);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // keys 64 h + 16 kk ..: two 8-row groups
              tc_mma_ts(tO + h * 128, tS + b * BN + h * 64 + kk * 8,
                        smem_desc(bV + (4 * h + kk) * 2048, 16384), idesc_pv, (jp > 0 || kk > 0));
          }
          if (!ok) break;
          tc_commit(&B->pv_done[b]);
          tc_commit(&B->v_empty[sv]);
          if (jp + 2 < nkt) ok = issue_s(jp + 2);
        }
      }
      for (int j = 0; j <= nkt && ok && !LY::kIndep; ++j) {
        if (j < nkt) {  // S(j) = Q K(j)^T into TMEM buffer j % 2
          const int s = j & 1, sk = j % kKStages;
          ok = wait_or_abort(&B->k_full[sk], (j / kKStages) & 1, B, p.dev_err);
          if (ok && j >= 2) ok = wait_or_abort(&B->s_empty[s], ((j - 2) >> 1) & 1, B, p.dev_err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bK = sbase + kKOff + sk * kOpBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc_mma(tS + s * BN, smem_desc(aQ + off), smem_desc(bK + off), idesc, kk > 0);
          }
          tc_commit(&B->s_full[s]);
          tc_commit(&B->k_empty[sk]);  // the K stage is free once S(j) is done
        }
        if (j >= 1) {  // O += P(j-1) V(j-1), P from TMEM
          const int jp = j - 1, b = jp % kPB, sv = jp % kVStages;
          ok = wait_or_abort(&B->v_full[sv], (jp / kVStages) & 1, B, p.dev_err);
          if (ok) ok = wait_or_abort(&B->p_full[b], (jp / kPB) & 1, B, p.dev_err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bV = sbase + kVOff + sv * kOpBytes;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {  // 16 keys = two 8-row groups per step
            const uint64_t vd = smem_desc(bV + kk * 2048, 16384);
            tc_mma_ts(tO, tP + b * (BN / 2) + kk * 8, vd, idesc_pv, (jp > 0 || kk > 0));
            if constexpr (LY::kBf16)  // the residual of P, into the same accumulator
              tc_mma_ts(tO, tP + BN / 2 + kk * 8, vd, idesc_pv, 1u);
          }
          tc_commit(&B->pv_done[b]);
          tc_commit(&B->v_empty[sv]);
        }
      }
      // everything issued above has completed before TMEM is released
      tc_commit(&B->done);
      mbar_wait(&B->done, 0);
    }
  } else if (warp == kLoadWarp) {
    if constexpr (LY::kTmaOps) {
      // TMA-fed operands: K then V of each tile.  issue(j, v) loads operand v
      // of tile j into its stage once the stage is free; false when the CTA
      // gives up.
      const int32_t* bt = p.block_tables + (size_t)c * p.max_blocks;
      int issued[2] = {0, 0};
      if (lane == 0) {
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
      }
      // launched as a programmatic dependent of the widening pass: the
      // prologue above overlapped it; the workspace is read only after it
      // has completed (a no-op for other launches)
      if (MODE == kStaged) pdl_wait();
      auto issue = [&](int j, bool vop) -> bool {
        const int NS = vop ? kVStages : kKStages;
        const int st = j % NS;
        uint64_t* full = vop ? &B->v_full[st] : &B->k_full[st];
        uint64_t* empty = vop ? &B->v_empty[st] : &B->k_empty[st];
        const CUtensorMap* map = vop ? &tmv : &tmk;
        uint8_t* d = smem + (vop ? kVOff : kKOff) + st * kOpBytes;
        if constexpr (MODE == kStaged) {
          // tile j of this chunk and kv head is rows row0 + 128 j .. + 127 of
          // the workspace; an operand is two 64-column boxes (its two 16 KiB
          // halves, 128-byte swizzled), counted on the stage's full barrier
          int ok = 1;
          if (lane == 0) {
            if (j >= NS)
              ok = wait_or_abort(empty, ((j - NS) / NS) & 1, B, p.dev_err) && !aborted(B);
            if (ok) {
              const int row = (c * p.n_kv + kvh) * p.stage_rows + j * BN;
              mbar_arrive_expect_tx(full, kOpBytes);
              tma_load_2d(d, map, full, 0, row);
              tma_load_2d(d + kOpBytes / 2, map, full, 64, row);
            }
          }
          return __shfl_sync(0xffffffffu, ok, 0) != 0;
        } else {
          // bf16 blocks straight from the pool: lane m < 8 holds block m of
          // tile j.  A whole block of the context with an id in range is two
          // 64-column boxes (rows 16 m .. 16 m + 15 of the stage's halves),
          // counted on the stage's full barrier; the rows of every other
          // block (the one the context ends in, those past it, those with an
          // out-of-range id) the warp writes itself before that barrier's
          // arrival, so the MMA reads them too: zeros past the context, so
          // that 0 x garbage never reaches O.
          constexpr uint32_t kBlockBytes = 16u * D * 2u;  // one operand's rows of a block
          const int blk = j * 8 + lane;
          const bool in_ctx = lane < 8 && blk * 16 < ctx;
          const int phys = in_ctx ? __ldg(&bt[blk]) : -1;
          const bool in_range = phys >= 0 && phys < p.num_blocks;
          if (!vop && in_ctx && !in_range) flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
          const bool whole = in_ctx && in_range && blk * 16 + 16 <= ctx;
          const uint32_t whole_m = __ballot_sync(0xffffffffu, whole);
          const uint32_t part_m = __ballot_sync(0xffffffffu, lane < 8 && !whole);
          const int y = whole ? (phys * p.n_kv + kvh) * 16 : 0;  // row in the [rows][D] view
          if (j >= NS) {
            const bool ok =
                wait_or_abort(empty, ((j - NS) / NS) & 1, B, p.dev_err) && !aborted(B);
            if (!__all_sync(0xffffffffu, ok)) return false;
          }
          const uint8_t* pool = static_cast<const uint8_t*>(vop ? v_pool : k_pool);
          for (uint32_t pm = part_m; pm; pm &= pm - 1) {
            const int m = __ffs(pm) - 1;
            const int ph = __shfl_sync(0xffffffffu, phys, m);
            const bool ok_id = ph >= 0 && ph < p.num_blocks;
            const int nvalid = ok_id ? max(0, min(16, ctx - (j * 8 + m) * 16)) : 0;
            write_block_rows(d, m, pool, ok_id ? (long long)(ph * p.n_kv + kvh) * 16 : 0,
                             nvalid, lane);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_expect_tx(full, __popc(whole_m) * kBlockBytes);
          __syncwarp();
          if (whole) {
            tma_load_2d(d + lane * 2048, map, full, 0, y);
            tma_load_2d(d + kOpBytes / 2 + lane * 2048, map, full, 64, y);
          }
          return true;
        }
      };
      for (int j = 0; j < nkt; ++j) {
        if (!issue(j, false)) break;
        issued[0] = j + 1;
        if (!issue(j, true)) break;
        issued[1] = j + 1;
      }
      // loads still in flight when the CTA gives up land before it exits
      if (lane == 0) {
        for (int t = max(0, issued[0] - kKStages); t < issued[0]; ++t)
          mbar_wait(&B->k_full[t % kKStages], (t / kKStages) & 1);
        for (int t = max(0, issued[1] - kVStages); t < issued[1]; ++t)
          mbar_wait(&B->v_full[t % kVStages], (t / kVStages) & 1);
      }
    } else {
      // ----------------------------------------------- raw fp8 tiles by TMA
      // Lane m < 8 loads block m of tile t: its 16 K rows and 16 V rows of
      // 128 bytes, one box each, into raw stage t % 2 with the 128-byte
      // swizzle.  Blocks past the context and out-of-range ids are not
      // loaded; the converters zero those keys.
      const int32_t* bt = p.block_tables + (size_t)c * p.max_blocks;
      if (lane == 0) {
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
      }
      int issued = 0;
      for (int t = 0; t < nkt; ++t) {
        const int rs = t % kRawStages;
        // the stage is free once every converter has read tile t-2 out of it
        // (each lane waits, so each load it issues is ordered after those reads)
        const bool ok = t < kRawStages ||
                        (wait_or_abort(&B->raw_empty[rs], ((t - kRawStages) / kRawStages) & 1,
                                       B, p.dev_err) &&
                         !aborted(B));
        if (!__all_sync(0xffffffffu, ok)) break;
        const int blk = t * 8 + lane;
        const int phys = (lane < 8 && blk * 16 < ctx) ? __ldg(&bt[blk]) : -1;
        const bool valid = phys >= 0 && phys < p.num_blocks;
        const uint32_t vm = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) mbar_arrive_expect_tx(&B->raw_full[rs], __popc(vm) * 2u * 16u * D);
        __syncwarp();
        if (valid) {
          uint8_t* dst = smem + LY::kRawOff + rs * 2 * kRawBytes + lane * 16 * D;
          const int y = (phys * p.n_kv + kvh) * 16;  // row of the pool's [token rows][D] view
          tma_load_2d(dst, &tmk, &B->raw_full[rs], 0, y);
          tma_load_2d(dst + kRawBytes, &tmv, &B->raw_full[rs], 0, y);
        }
        issued = t + 1;
      }
      // loads still in flight when the CTA gives up land before it exits
      if (lane == 0)
        for (int t = max(0, issued - kRawStages); t < issued; ++t)
          mbar_wait(&B->raw_full[t % kRawStages], (t / kRawStages) & 1);
    }
  } else if (warp >= LY::kSoftWarps) {
    // ------------------------------------------------------------ converters
    if constexpr (LY::kRawRing) {
    const int ct = tid - LY::kSoftWarps * 32;  // 0..127
    const int32_t* bt = p.block_tables + (size_t)c * p.max_blocks;
    // block ids of a tile's 8 blocks (-1 past the context); the next tile's
    // are loaded a tile ahead so the K/V reads never wait on the block table
    auto load_ids = [&](int j, int (&ids)[8]) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int blk = j * 8 + m;
        ids[m] = (blk * 16 < ctx) ? __ldg(&bt[blk]) : -1;
      }
    };
    int id_cur[8], id_nxt[8];  // ids of tile j and of tile j+1
    load_ids(0, id_cur);
    if (nkt > 1) load_ids(1, id_nxt);
    for (int j = 0; j < nkt; ++j) {
      const int s = j % kKStages, sv = j % kVStages;
      uint8_t* kop = smem + kKOff + s * kOpBytes;
      uint8_t* vop = smem + kVOff + sv * kOpBytes;
      // wait for the raw tile
      const int rs = j % kRawStages;
      const uint8_t* raw = smem + LY::kRawOff + rs * 2 * kRawBytes;
      const bool raw_stop = !wait_or_abort(&B->raw_full[rs], (j / kRawStages) & 1, B, p.dev_err);
      // Pass m covers block m of the tile: thread ct takes key ct/8, 16-byte
      // chunk ct%8 of the stored K and V rows.  The reads of all 8 passes go
      // out before the operand stages are released, so their latency overlaps
      // the tensor-core work still reading them.
      uint4 kr[8], vr[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int kib = ct >> 3;  // key in block
        const int cc = ct & 7;    // 16-byte chunk in the row
        const int key = j * BN + m * 16 + kib;
        kr[m] = make_uint4(0, 0, 0, 0);
        vr[m] = make_uint4(0, 0, 0, 0);
        if (key < ctx) {
          const int phys = id_cur[m];
          if (phys < 0 || phys >= p.num_blocks) {
            if (kib == 0 && cc == 0) flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
          } else if (!raw_stop) {  // row kib of block m in the swizzled raw stage
            const uint32_t ro = m * 16 * D + swz128(kib * 128 + cc * 16);
            kr[m] = *reinterpret_cast<const uint4*>(raw + ro);
            vr[m] = *reinterpret_cast<const uint4*>(raw + kRawBytes + ro);
          }
        }
      }
      // the K stage is free once S(j-2) is done, the V stage once O += P V of
      // tile j - kVStages is
      mbar_arrive(&B->raw_empty[rs]);  // raw tile j read
      bool stop = raw_stop || (j >= kKStages && !wait_or_abort(&B->k_empty[s],
                                                               ((j - kKStages) / kKStages) & 1,
                                                               B, p.dev_err));
      stop = stop || (j >= kVStages &&
                      !wait_or_abort(&B->v_empty[sv], ((j - kVStages) / kVStages) & 1, B,
                                     p.dev_err));
      if (conv_bar_or(stop || aborted(B))) break;  // all converters stop together
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int kib = ct >> 3, cc = ct & 7;
        const int key_t = m * 16 + kib;  // key within tile
        // 16 codes -> 16 f16 = 16-bit chunks 2cc, 2cc+1 (dims 16cc..16cc+15)
        uint32_t kh[8], vh[8];
        const uint32_t kw[4] = {kr[m].x, kr[m].y, kr[m].z, kr[m].w};
        const uint32_t vw[4] = {vr[m].x, vr[m].y, vr[m].z, vr[m].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kh[2 * e] = e4m3x2_to_f16x2(kw[e] & 0xffffu);
          kh[2 * e + 1] = e4m3x2_to_f16x2(kw[e] >> 16);
          vh[2 * e] = e4m3x2_to_f16x2_div256(vw[e], 0x4140u);      // codes 0, 1
          vh[2 * e + 1] = e4m3x2_to_f16x2_div256(vw[e], 0x4342u);  // codes 2, 3
        }
        *reinterpret_cast<uint4*>(kop + op_off(key_t, 2 * cc)) =
            make_uint4(kh[0], kh[1], kh[2], kh[3]);
        *reinterpret_cast<uint4*>(kop + op_off(key_t, 2 * cc + 1)) =
            make_uint4(kh[4], kh[5], kh[6], kh[7]);
        *reinterpret_cast<uint4*>(vop + op_off(key_t, 2 * cc)) =
            make_uint4(vh[0], vh[1], vh[2], vh[3]);
        *reinterpret_cast<uint4*>(vop + op_off(key_t, 2 * cc + 1)) =
            make_uint4(vh[4], vh[5], vh[6], vh[7]);
      }
      fence_async_smem();
      mbar_arrive(&B->k_full[s]);
      mbar_arrive(&B->v_full[sv]);
#pragma unroll
      for (int m = 0; m < 8; ++m) id_cur[m] = id_nxt[m];
      if (j + 2 < nkt) load_ids(j + 2, id_nxt);  // a whole tile ahead of its first use
    }
    }
  } else if constexpr (LY::kIndep) {
    // ------------------------------ softmax, two independent parts per row
    // Warps w and w + 4 share rows 32 (w % 4) .. + 31 (the TMEM lanes warp
    // w % 4 may access); part hh takes keys 64 hh .. 64 hh + 63 of every tile
    // with its own running max, sum and O accumulator O_hh (TMEM columns
    // 256 + 128 hh), writes its P over the first half of its own S columns,
    // and rescales only O_hh.  Nothing is exchanged per tile; at the end the
    // two parts' (max, sum) meet in shared memory and each thread writes half
    // of its row from both accumulators.
    const int q4 = warp & 3, hh = warp >> 2;
    const int r = q4 * 32 + lane;  // row = TMEM lane
    const int i = i0 + r / G, g = r % G;
    const bool row_valid = i < L;
    const bool live = i0 + (q4 * 32) / G < L;  // see the split softmax below
    const int lim = H + i;                      // last visible key
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tOh = tO + hh * 128 + lane_base;
    const float sl = row_scale[r];  // > 0 exactly when the scale is
    float m_used = -INFINITY, l = 0.f;
    bool fail = false;  // warp-uniform
    for (int j = 0; j < nkt; ++j) {
      const int s = j & 1;
      fail = __any_sync(0xffffffffu, !wait_or_abort(&B->s_full[s], (j >> 1) & 1, B, p.dev_err));
      if (fail) break;
      tc_fence_after();
      const int kbase = j * BN + hh * 64;  // first key of this part
      const uint32_t tSrow = tS + lane_base + s * BN + hh * 64;
      const bool full =
          __all_sync(0xffffffffu, row_valid && kbase + 63 <= lim) && p.scale_log2 > 0.f;
      float x[64];
      float mx = -INFINITY;
      if (live) {  // this part's scores and their max
        tmem_ld32(tSrow, x);
        tmem_ld32(tSrow + 32, x + 32);
        tmem_wait_ld();
        float m4[4] = {mx, -INFINITY, -INFINITY, -INFINITY};  // 4 chains, not 1
        if (full) {
#pragma unroll
          for (int e = 0; e < 64; ++e) m4[e & 3] = fmaxf(m4[e & 3], x[e]);
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            const bool vis = !row_valid || (kbase + e <= lim);
            m4[e & 3] = fmaxf(m4[e & 3], vis ? (row_valid ? x[e] * sl : 0.f) : -INFINITY);
          }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
      }
      // lazy rescale: only when this part's max grew by more than 2^8
      const float m_new = fmaxf(m_used, mx);
      const bool rescale = m_new > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (rescale) {
        alpha = exp2f(m_used - m_new);  // 0 on the first tile
        l *= alpha;
        m_used = m_new;
      }
      float r4[4] = {0.f, 0.f, 0.f, 0.f};  // the row sum in 4 chains
      uint32_t pk[32];
      // a row that has seen no key yet exponentiates against 0 (P = 0, not NaN)
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      if (live) {
        if (full) {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float a = fast_exp2(fmaf(x[e], sl, neg_m));
            const float bb = fast_exp2(fmaf(x[e + 1], sl, neg_m));
            r4[(e >> 1) & 3] += a + bb;
            pk[e / 2] = pack2<false>(a, bb);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const int k0 = kbase + e;
            const float v0 = row_valid ? (k0 <= lim ? x[e] * sl : -INFINITY) : 0.f;
            const float v1 = row_valid ? (k0 + 1 <= lim ? x[e + 1] * sl : -INFINITY) : 0.f;
            const float a = fast_exp2(v0 + neg_m), bb = fast_exp2(v1 + neg_m);
            r4[(e >> 1) & 3] += a + bb;
            pk[e / 2] = pack2<false>(a, bb);
          }
        }
      }
      l += (r4[0] + r4[1]) + (r4[2] + r4[3]);
      // O_hh is rescaled (rarely) once O_hh += P V of tile j-1 has completed
      if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
        fail = __any_sync(0xffffffffu, !wait_or_abort(&B->pv_done[(j - 1) & 1],
                                                      ((j - 1) >> 1) & 1, B, p.dev_err));
        if (fail) break;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          tmem_ld32(tOh + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tOh + cc * 32, o);
        }
        tmem_wait_st();
      }
      if (live) {
        // the pair (key 2c, 2c+1) of this part in column c of its S columns
        tc_fence_after();
        tmem_st32(tSrow, reinterpret_cast<const float*>(pk));
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&B->pp_full[hh][s]);
    }
    // epilogue: both parts' (max, sum) meet in shared memory once their last
    // O += P V has completed; every softmax thread reaches the barrier once
    if (!fail)
      fail = __any_sync(0xffffffffu, !wait_or_abort(&B->pv_done[(nkt - 1) & 1],
                                                    ((nkt - 1) >> 1) & 1, B, p.dev_err));
    float2* red = reinterpret_cast<float2*>(smem + LY::kRedOff);  // [2][BM]
    red[hh * BM + r] = make_float2(m_used, l);
    if (!named_bar_or(2, LY::kSoftWarps * 32, fail)) {
      tc_fence_after();
      const float2 other = red[(hh ^ 1) * BM + r];
      const float M = fmaxf(m_used, other.x);
      const float w_me = m_used == -INFINITY ? 0.f : exp2f(m_used - M);
      const float w_ot = other.x == -INFINITY ? 0.f : exp2f(other.x - M);
      const float lt = w_me * l + w_ot * other.y;
      const float inv = (lt > 0.f) ? p.out_mul / lt : 0.f;
      const float w0 = (hh == 0 ? w_me : w_ot) * inv, w1 = (hh == 0 ? w_ot : w_me) * inv;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) +
                           ((size_t)(q0 + (row_valid ? i : 0)) * p.n_q + (size_t)kvh * G + g) * D +
                           hh * 64;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        float o0[32], o1[32];
        tmem_ld32(tO + lane_base + hh * 64 + cc * 32, o0);
        tmem_ld32(tO + 128 + lane_base + hh * 64 + cc * 32, o1);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack2<true>(o0[e] * w0 + o1[e] * w1, o0[e + 1] * w0 + o1[e + 1] * w1);
            v.y = pack2<true>(o0[e + 2] * w0 + o1[e + 2] * w1, o0[e + 3] * w0 + o1[e + 3] * w1);
            v.z = pack2<true>(o0[e + 4] * w0 + o1[e + 4] * w1, o0[e + 5] * w0 + o1[e + 5] * w1);
            v.w = pack2<true>(o0[e + 6] * w0 + o1[e + 6] * w1, o0[e + 7] * w0 + o1[e + 7] * w1);
            *reinterpret_cast<uint4*>(out + cc * 32 + e) = v;
          }
        }
      }
    }
  } else if constexpr (LY::kSplitSoftmax) {
    // -------------------------------------- softmax, kParts warps per row
    // The kParts warps w, w + 4, ... share rows 32 (w % 4) .. + 31 (the TMEM
    // lanes warp w % 4 may access); part hh takes keys KW hh .. KW hh + KW - 1
    // of every tile and O columns OW hh .. OW hh + OW - 1.  The row max of a
    // tile is combined through shared memory at a named barrier over all the
    // softmax threads, which also ORs their failure flags so that all of them
    // leave the loop at the same barrier; the row sum is combined once at the
    // end.  Several warps per sub-partition hide each other's latencies (the
    // TMEM loads, the exponentials, the barrier).
    constexpr int NP = LY::kParts;
    constexpr int KW = BN / NP;  // keys per part and tile
    constexpr int OW = D / NP;   // O columns per part
    const int q4 = warp & 3, hh = warp >> 2;
    const int r = q4 * 32 + lane;  // row = TMEM lane
    const int i = i0 + r / G, g = r % G;
    const bool row_valid = i < L;
    // a warp whose 32 rows are all past the chunk's queries (the tail of the
    // last query tile; most of the tile in multi-query decode) computes no P:
    // those rows of P and O are never read out, so it only keeps the barriers
    const bool live = i0 + (q4 * 32) / G < L;
    const int lim = H + i;  // last visible key
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    float* red_max = reinterpret_cast<float*>(smem + LY::kRedOff);  // [2][NP][BM]
    float* red_sum = red_max + 2 * NP * BM;                         // [NP][BM]
    const float sl = row_scale[r];  // > 0 exactly when the scale is
    float m_used = -INFINITY, l = 0.f;
    bool fail = false;  // warp-uniform
    auto load_s = [&](uint32_t ta, float* x) {
#pragma unroll
      for (int c32 = 0; c32 < KW / 32; ++c32) tmem_ld32(ta + c32 * 32, x + c32 * 32);
      tmem_wait_ld();
    };
    for (int j = 0; j < nkt; ++j) {
      const int s = j & 1;
      fail = __any_sync(0xffffffffu,
                        fail || !wait_or_abort(&B->s_full[s], (j >> 1) & 1, B, p.dev_err));
      tc_fence_after();
      const int kbase = j * BN + hh * KW;  // first key of this part
      const uint32_t tSrow = tS + lane_base + s * BN + hh * KW;
      const bool full =
          __all_sync(0xffffffffu, row_valid && kbase + KW - 1 <= lim) && p.scale_log2 > 0.f;
      float mx = -INFINITY;
      // this part's scores, read from TMEM once: the loads are slow while the
      // tensor core works on the same TMEM, so pass 2 reuses the registers
      float x[KW];
      if (!fail && live) {  // pass 1: this part's max
        load_s(tSrow, x);
        float m4[4] = {mx, -INFINITY, -INFINITY, -INFINITY};  // 4 chains, not 1
        if (full) {
#pragma unroll
          for (int e = 0; e < KW; ++e) m4[e & 3] = fmaxf(m4[e & 3], x[e]);
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
        } else {
#pragma unroll
          for (int e = 0; e < KW; ++e) {
            const bool vis = !row_valid || (kbase + e <= lim);
            m4[e & 3] = fmaxf(m4[e & 3], vis ? (row_valid ? x[e] * sl : 0.f) : -INFINITY);
          }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
      }
      float* rm = red_max + (j & 1) * NP * BM;
      rm[hh * BM + r] = mx;
      if (named_bar_or(2, LY::kSoftWarps * 32, fail || aborted(B))) {
        fail = true;
        break;
      }
#pragma unroll
      for (int o = 1; o < NP; ++o) mx = fmaxf(mx, rm[((hh + o) % NP) * BM + r]);
      // O and l are rescaled lazily: only when the max grew by more than 2^8;
      // all parts of a row take the same decision
      const float m_new = fmaxf(m_used, mx);
      const bool rescale = m_new > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (rescale) {
        alpha = exp2f(m_used - m_new);  // 0 on the first tile
        l *= alpha;
        m_used = m_new;
      }
      // pass 2: P = 2^(s*scale - m) as f16 pairs, or as bf16 pairs plus the
      // bf16 pairs of their rounding residuals
      float r4[4] = {0.f, 0.f, 0.f, 0.f};  // the row sum in 4 chains
      // (the residual pairs go to x[0 .. KW/2), scores already consumed)
      uint32_t pk[KW / 2];
      auto put = [&](int e, float a, float bb) {
        if constexpr (LY::kBf16) {
          const uint32_t h = pack2<true>(a, bb);
          const float2 hf = unpack2<true>(h);
          pk[e / 2] = h;
          x[e / 2] = __uint_as_float(pack2<true>(a - hf.x, bb - hf.y));
        } else {
          pk[e / 2] = pack2<false>(a, bb);
        }
      };
      // a row that has seen no key yet (multi-query decode) exponentiates
      // against 0, so that its masked scores give P = 0, not NaN
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      if (live) {
        if (full) {
#pragma unroll
          for (int e = 0; e < KW; e += 2) {
            const float a = fast_exp2(fmaf(x[e], sl, neg_m));
            const float bb = fast_exp2(fmaf(x[e + 1], sl, neg_m));
            r4[(e >> 1) & 3] += a + bb;
            put(e, a, bb);
          }
        } else {
#pragma unroll
          for (int e = 0; e < KW; e += 2) {
            const int k0 = kbase + e;
            const float v0 = row_valid ? (k0 <= lim ? x[e] * sl : -INFINITY) : 0.f;
            const float v1 = row_valid ? (k0 + 1 <= lim ? x[e + 1] * sl : -INFINITY) : 0.f;
            const float a = fast_exp2(v0 + neg_m), bb = fast_exp2(v1 + neg_m);
            r4[(e >> 1) & 3] += a + bb;
            put(e, a, bb);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&B->s_empty[s]);  // S buffer s may be overwritten by S(j+2)
      l += (r4[0] + r4[1]) + (r4[2] + r4[3]);
      const int b = j % kPB;
      // P buffer b is free once O += P V of tile j - kPB has completed
      if (j >= kPB)
        fail = __any_sync(0xffffffffu, !wait_or_abort(&B->pv_done[b], ((j - kPB) / kPB) & 1, B,
                                                      p.dev_err));
      // O (this part's columns) is rescaled, rarely, once O += P V of tile
      // j-1 has completed (with one P buffer, the wait above saw to that)
      if (!fail && j >= 1 && __any_sync(0xffffffffu, rescale)) {
        if constexpr (kPB == 2)
          fail = __any_sync(0xffffffffu, !wait_or_abort(&B->pv_done[b ^ 1], ((j - 1) >> 1) & 1,
                                                        B, p.dev_err));
        if (!fail) {
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < OW / 32; ++cc) {
            float o[32];
            const uint32_t ta = tO + lane_base + hh * OW + cc * 32;
            tmem_ld32(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(ta, o);
          }
          tmem_wait_st();
        }
      }
      if (!fail) {
        if (live) {
          tc_fence_after();
          // column c of P buffer b holds the pair (key 2c, 2c+1); this part
          // writes columns KW/2 hh .. KW/2 hh + KW/2 - 1 (and the residuals
          // 64 further)
          tmem_st_pairs<KW>(tP + lane_base + b * (BN / 2) + hh * (KW / 2), pk);
          if constexpr (LY::kBf16)
            tmem_st_pairs<KW>(tP + lane_base + BN / 2 + hh * (KW / 2),
                              reinterpret_cast<const uint32_t*>(x));
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&B->p_full[b]);
      }
    }
    // epilogue: O / l after the last O += P V; every softmax thread reaches
    // this barrier once, whether the loop ended or was left together
    if (!fail)
      fail = __any_sync(0xffffffffu, !wait_or_abort(&B->pv_done[(nkt - 1) % kPB],
                                                    ((nkt - 1) / kPB) & 1, B, p.dev_err));
    red_sum[hh * BM + r] = l;
    if (!named_bar_or(2, LY::kSoftWarps * 32, fail)) {
      tc_fence_after();
      float lt = l;
#pragma unroll
      for (int o = 1; o < NP; ++o) lt += red_sum[((hh + o) % NP) * BM + r];
      const float inv = (lt > 0.f) ? p.out_mul / lt : 0.f;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) +
                           ((size_t)(q0 + (row_valid ? i : 0)) * p.n_q + (size_t)kvh * G + g) * D +
                           hh * OW;
#pragma unroll
      for (int cc = 0; cc < OW / 32; ++cc) {
        float o[32];
        tmem_ld32(tO + lane_base + hh * OW + cc * 32, o);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack2<true>(o[e] * inv, o[e + 1] * inv);
            v.y = pack2<true>(o[e + 2] * inv, o[e + 3] * inv);
            v.z = pack2<true>(o[e + 4] * inv, o[e + 5] * inv);
            v.w = pack2<true>(o[e + 6] * inv, o[e + 7] * inv);
            *reinterpret_cast<uint4*>(out + cc * 32 + e) = v;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = tid;  // row = TMEM lane
    const int i = i0 + r / G, g = r % G;
    const bool row_valid = i < L;
    const bool live = i0 + (warp * 32) / G < L;  // see the split softmax
    const int lim = H + i;  // last visible key
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl = row_scale[r];  // > 0 exactly when the scale is
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt && ok; ++j) {
      const int s = j & 1;
      ok = __all_sync(0xffffffffu, wait_or_abort(&B->s_full[s], (j >> 1) & 1, B, p.dev_err));
      if (!ok) break;
      tc_fence_after();
      const int kbase = j * BN;
      const uint32_t tSrow = tS + lane_base + s * BN;
      // a tile every key of which is visible to every row of this warp needs no
      // mask: its max is taken on the raw scores (the scale is positive)
      const bool full =
          __all_sync(0xffffffffu, row_valid && kbase + BN - 1 <= lim) && p.scale_log2 > 0.f;
      // pass 1: the row's max over this tile, 32 columns at a time
      float mx = -INFINITY;
      if (!live) {
      } else if (full) {
#pragma unroll 1
        for (int cc = 0; cc < 4; cc += 2) {  // two TMEM loads in flight
          float x[64];
          tmem_ld32(tSrow + cc * 32, x);
          tmem_ld32(tSrow + cc * 32 + 32, x + 32);
          tmem_wait_ld();
          float m4[4] = {mx, -INFINITY, -INFINITY, -INFINITY};  // 4 chains, not 1
#pragma unroll
          for (int e = 0; e < 64; ++e) m4[e & 3] = fmaxf(m4[e & 3], x[e]);
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        mx *= sl;
      } else {
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float x[32];
          tmem_ld32(tSrow + cc * 32, x);
          tmem_wait_ld();
          float m4[4] = {mx, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const bool vis = !row_valid || (kbase + cc * 32 + e <= lim);
            m4[e & 3] = fmaxf(m4[e & 3], vis ? (row_valid ? x[e] * sl : 0.f) : -INFINITY);
          }
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
      }
      // O and l are rescaled lazily: only when the max grew by more than 2^8
      const float m_new = fmaxf(m_used, mx);
      const bool rescale = m_new > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (rescale) {
        alpha = exp2f(m_used - m_new);  // 0 on the first tile
        l *= alpha;
        m_used = m_new;
      }
      // pass 2: P = 2^(s*scale - m) as f16, kept in registers until the P
      // buffer is free
      float r4[4] = {0.f, 0.f, 0.f, 0.f};  // the row sum in 4 chains
      uint32_t pk[BN / 2];
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;  // see the split softmax
      if (!live) {
      } else if (full) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float x[32];
          tmem_ld32(tSrow + cc * 32, x);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float a = fast_exp2(fmaf(x[e], sl, neg_m));
            const float bb = fast_exp2(fmaf(x[e + 1], sl, neg_m));
            r4[(e >> 1) & 3] += a + bb;
            pk[cc * 16 + e / 2] = pack2<false>(a, bb);
          }
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float x[32];
          tmem_ld32(tSrow + cc * 32, x);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int k0 = kbase + cc * 32 + e;
            const float v0 = row_valid ? (k0 <= lim ? x[e] * sl : -INFINITY) : 0.f;
            const float v1 = row_valid ? (k0 + 1 <= lim ? x[e + 1] * sl : -INFINITY) : 0.f;
            const float a = fast_exp2(v0 + neg_m), bb = fast_exp2(v1 + neg_m);
            r4[(e >> 1) & 3] += a + bb;
            pk[cc * 16 + e / 2] = pack2<false>(a, bb);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&B->s_empty[s]);  // S buffer s may be overwritten by S(j+2)
      l += (r4[0] + r4[1]) + (r4[2] + r4[3]);
      const int b = j & 1;
      // P buffer b is free once O += P V of tile j-2 has completed
      if (j >= 2) {
        ok = __all_sync(0xffffffffu,
                        wait_or_abort(&B->pv_done[b], ((j - 2) >> 1) & 1, B, p.dev_err));
        if (!ok) break;
      }
      // O is rescaled (rarely) once O += P V of tile j-1 has completed
      if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
        ok = __all_sync(0xffffffffu, wait_or_abort(&B->pv_done[b ^ 1], ((j - 1) >> 1) & 1, B,
                                                   p.dev_err));
        if (!ok) break;
        tc_fence_after();
        {
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            tmem_ld32(tO + lane_base + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tO + lane_base + cc * 32, o);
          }
          tmem_wait_st();
        }
      }
      if (live) {
        tc_fence_after();
        // P row -> TMEM: column c of buffer b holds the f16 pair (key 2c, 2c+1)
        tmem_st32(tP + lane_base + b * (BN / 2), reinterpret_cast<const float*>(pk));
        tmem_st32(tP + lane_base + b * (BN / 2) + 32, reinterpret_cast<const float*>(pk + 32));
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&B->p_full[b]);
    }
    // epilogue: O / l after the last O += P V
    if (ok && __all_sync(0xffffffffu, wait_or_abort(&B->pv_done[(nkt - 1) & 1],
                                                    ((nkt - 1) >> 1) & 1, B, p.dev_err))) {
      tc_fence_after();
      const float inv = (l > 0.f) ? p.out_mul / l : 0.f;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) +
                           ((size_t)(q0 + (row_valid ? i : 0)) * p.n_q + (size_t)kvh * G + g) * D;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float o[32];
        tmem_ld32(tO + lane_base + cc * 32, o);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack2<true>(o[e] * inv, o[e + 1] * inv);
            v.y = pack2<true>(o[e + 2] * inv, o[e + 3] * inv);
            v.z = pack2<true>(o[e + 4] * inv, o[e + 5] * inv);
            v.w = pack2<true>(o[e + 6] * inv, o[e + 7] * inv);
            *reinterpret_cast<uint4*>(out + cc * 32 + e) = v;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// ------------------------------------------------------------- widen pass
// Writes keys 0 .. round_up(ctx_c, 128) - 1 of chunk c's fp8 history for kv
// head h as f16 rows of the workspace: K to kst[(c n_kv + h) stage_rows +
// key][d], V likewise to vst.  Keys at or past the context, and the keys of a
// block whose id is out of range (flagged PA_DEVERR_BLOCK_ID), are written as
// zeros, so the attention kernel reads finite values everywhere.  Both
// operands widen exactly (code x 1).  One CTA per 128-key tile; 16-byte loads
// and stores, a warp covering whole stored rows.
__global__ void __launch_bounds__(256)
    prefill_widen_kernel(const PrefillParams p, const void* __restrict__ k_pool,
                         const void* __restrict__ v_pool, uint16_t* __restrict__ kst,
                         uint16_t* __restrict__ vst) {
  const int t = blockIdx.x, kvh = blockIdx.y, c = blockIdx.z;
  // launched as a programmatic dependent: whatever ran before (the slot
  // write) completes first; then the attention kernel may start its prologue
  pdl_wait();
  pdl_launch_dependents();
  const int ctx = p.context_lens[c];
  if (ctx < 0 || ctx > p.max_blocks * 16) return;  // the attention kernel flags it
  const int k0 = t * BN;
  if (k0 >= ctx) return;
  const int32_t* bt = p.block_tables + (size_t)c * p.max_blocks;
  constexpr int kCh = D / 16;  // 16-byte chunks per stored fp8 row
  const size_t row0 = ((size_t)c * p.n_kv + kvh) * p.stage_rows + k0;
  for (int idx = threadIdx.x; idx < BN * kCh; idx += blockDim.x) {
    const int r = idx / kCh, cc = idx % kCh;
    const int key = k0 + r;
    uint4 kr = make_uint4(0, 0, 0, 0), vr = make_uint4(0, 0, 0, 0);
    if (key < ctx) {
      const int phys = __ldg(&bt[key >> 4]);
      if (phys < 0 || phys >= p.num_blocks) {
        if ((key & 15) == 0 && cc == 0) flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
      } else {
        const size_t off = (((size_t)phys * p.n_kv + kvh) * 16 + (key & 15)) * D + (size_t)cc * 16;
        kr = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(k_pool) + off));
        vr = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(v_pool) + off));
      }
    }
    uint4* kd = reinterpret_cast<uint4*>(kst + (row0 + r) * D);
    uint4* vd = reinterpret_cast<uint4*>(vst + (row0 + r) * D);
    // 16 codes -> 16 f16 (elements 16 cc .. 16 cc + 15)
    const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w}, vw[4] = {vr.x, vr.y, vr.z, vr.w};
    uint32_t kh[8], vh[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kh[2 * e] = e4m3x2_to_f16x2(kw[e] & 0xffffu);
      kh[2 * e + 1] = e4m3x2_to_f16x2(kw[e] >> 16);
      vh[2 * e] = e4m3x2_to_f16x2(vw[e] & 0xffffu);
      vh[2 * e + 1] = e4m3x2_to_f16x2(vw[e] >> 16);
    }
    kd[2 * cc] = make_uint4(kh[0], kh[1], kh[2], kh[3]);
    kd[2 * cc + 1] = make_uint4(kh[4], kh[5], kh[6], kh[7]);
    vd[2 * cc] = make_uint4(vh[0], vh[1], vh[2], vh[3]);
    vd[2 * cc + 1] = make_uint4(vh[4], vh[5], vh[6], vh[7]);
  }
}

// a launch that may begin before the previous kernel in the stream has
// finished (programmatic dependent launch; the kernel calls pdl_wait before
// it reads what that kernel wrote)
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int MODE>
cudaError_t launch_tc(const PrefillParams& p, const void* k_pool, const void* v_pool,
                      const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t st) {
  using LY = Layout<MODE>;
  static cudaError_t attr = cudaFuncSetAttribute(
      prefill_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  const int QT = BM / p.group;
  dim3 grid((p.max_chunk_len + QT - 1) / QT, p.n_kv, p.n_chunks);
  if constexpr (MODE == kStaged)  // right after the widening pass
    return launch_dependent(prefill_tc_kernel<MODE>, grid, dim3(LY::kThreads), LY::kSmemBytes,
                            st, p, k_pool, v_pool, *tmk, *tmv);
  prefill_tc_kernel<MODE>
      <<<grid, LY::kThreads, LY::kSmemBytes, st>>>(p, k_pool, v_pool, *tmk, *tmv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, pa_dtype kv_dt, const void* k_pool,
                           const void* v_pool, const CUtensorMap* tmk, const CUtensorMap* tmv,
                           void* workspace, cudaStream_t st) {
  if (p.n_chunks == 0) return cudaSuccess;
  // a bf16 cache is read as it is: no widening, no workspace
  if (kv_dt != PA_FP8_E4M3) return launch_tc<kDirectBf16>(p, k_pool, v_pool, tmk, tmv, st);
  if (workspace == nullptr) return launch_tc<kWidenFp8>(p, k_pool, v_pool, tmk, tmv, st);
  uint16_t* kst = static_cast<uint16_t*>(workspace);
  uint16_t* vst = kst + (size_t)p.n_chunks * p.n_kv * p.stage_rows * D;
  const dim3 grid(p.stage_rows / BN, p.n_kv, p.n_chunks);
  const cudaError_t e =
      launch_dependent(prefill_widen_kernel, grid, dim3(256), 0, st, p, k_pool, v_pool, kst, vst);
  if (e != cudaSuccess) return e;
  return launch_tc<kStaged>(p, k_pool, v_pool, tmk, tmv, st);
}

size_t prefill_stage_rows(int max_blocks) {
  return ((size_t)max_blocks * 16 + BN - 1) / BN * BN;
}

}  // namespace pa
