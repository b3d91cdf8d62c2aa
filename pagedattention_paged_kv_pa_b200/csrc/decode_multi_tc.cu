// Multi-query decode on tcgen05 tensor cores (sm_100a): the target model
// checks q_len guessed tokens in one pass ("LLM inference optimization: KV
// cache & PagedAttention", §五 "Speculative Decoding"; "Daily AI, 2026-07-31:
// inference serving", "推測解碼").  With the K/V of all q_len new tokens in
// the cache, query i of a sequence with context c sits at position
// c - q_len + i and attends to keys 0 .. c - q_len + i.
//
// Tiles.  For one (sequence, kv head) the q_len x G (query, head) pairs are
// the rows of one 64-row MMA tile (row r = query r / G, head r % G; rows past
// q_len x G stay zero) and every 128-key K/V tile serves all of them.  With
// M = 64 the tensor core keeps accumulator row r in TMEM lane
// 32 (r / 16) + r % 16, so each of four softmax warps -- one per TMEM lane
// quadrant, i.e. one per SM sub-partition -- owns 16 whole rows: it reads them
// with the 16x256b shape (thread t: rows t / 4 and t / 4 + 8, two adjacent
// keys of every 8), needs no other warp for a row's max or sum, and rescales
// its own rows of O.  P goes to shared memory by stmatrix as the K-major A
// operand of O += P V: for bf16 a bf16 value plus its bf16 rounding residual
// (two MMAs into the same accumulator, ~16 significant bits, as in chunked
// prefill), for f16 one f16 value.  S = Q K^T and O live in TMEM, each double
// buffered (S(t+1) overlaps tile t's softmax; O of the next run of tiles
// accumulates while the last one is written out); P has one buffer, which
// tile t's softmax fills once O += P V of tile t - 1 is done.
//
// Work split.  Persistent CTAs, one per SM.  The work is the (sequence, kv
// head, 1024-token partition) units laid end to end in that order, measured
// in key tiles plus a fixed cost per (sequence, kv head); CTA c takes the
// units that start in [c T / C, (c + 1) T / C) (T in all, C CTAs), so every
// CTA gets about the same time's worth of K/V streaming.  Consecutive
// partitions of one (sequence, kv head) in a CTA form one segment,
// accumulated without a break.  A segment that covers its whole (sequence, kv
// head) writes the normalised output; a segment of a (sequence, kv head)
// split between CTAs writes its unnormalised output and (max, sum) to the
// workspace slot of its first partition and an empty state (max -inf) to its
// other partitions' slots, and mq_merge_kernel combines them.  Sequences with
// no context get all-zero rows.
//
// Roles: warps 0-3 softmax, warp 4 owns TMEM and issues the MMAs from one
// lane, warp 5 loads Q (one 3-D TMA box per 64-column half) and the K tiles
// into 3 stages, warp 6 the V tiles into 2 (two 64-column TMA boxes per whole
// 16-token block; a load warp writes the rows of the block the context ends
// in, zeros after them, and zeros for blocks past the context or with an
// out-of-range id, which the K warp flags).  Separate K and V warps keep a K
// load from waiting for a V stage: K stages free up when S = Q K^T is done, V
// stages only when O += P V is.  Every wait is bounded; a CTA that gives up
// flags PA_DEVERR_TIMEOUT, drains its MMAs and loads and frees TMEM.
#include <type_traits>

#include "mq_tc.h"
#include "tc_ops.cuh"

namespace pa {

namespace {

constexpr int D = 128;   // head dim
constexpr int BM = 64;   // MMA rows: (query, head) pairs of a kv head
constexpr int BN = 128;  // keys per tile
constexpr int kPT = kPart16 / BN;  // tiles per workspace partition (8)
constexpr int kKS = 3, kVS = 2;    // K and V stages
constexpr uint32_t kTmemCols = 512;  // S[2] at 0 and 128, O[2] at 256 and 384
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (factor 256)
constexpr int kSoftWarps = 4, kMmaWarp = 4, kKWarp = 5, kVWarp = 6;
constexpr int kThreads = 224;

// shared memory (offsets from a 1024-aligned base)
constexpr int kQBytes = BM * D * 2;   // one Q tile: 16 KiB
constexpr int kOpBytes = BN * D * 2;  // one K or V tile: 32 KiB
constexpr int kPBytes = BM * BN * 2;  // one P tile: 16 KiB (value, then residual)
constexpr int kQOff = 0;                                // Q[2]
constexpr int kKOff = kQOff + 2 * kQBytes;              // K stages
constexpr int kVOff = kKOff + kKS * kOpBytes;           // V stages
constexpr int kPOff = kVOff + kVS * kOpBytes;           // P: value, residual
constexpr int kBarOff = kPOff + 2 * kPBytes;
constexpr int kSmemBytes = kBarOff + 512 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

// A operand (Q, P): 64 rows of 128 16-bit elements, 128-byte swizzle, the two
// 64-element halves 8 KiB apart; chunk = 8 consecutive elements (0..15)
__device__ __forceinline__ uint32_t a_off(int row, int chunk) {
  return (chunk >> 3) * 8192 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}
// B operand (K, V): 128 rows, halves 16 KiB apart
__device__ __forceinline__ uint32_t b_off(int row, int chunk) {
  return (chunk >> 3) * 16384 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

struct Bars {
  uint64_t k_full[kKS], k_empty[kKS], v_full[kVS], v_empty[kVS];
  uint64_t q_full[2], q_empty[2], s_full[2], s_empty[2], p_full, pv_done[2], o_free[2];
  uint64_t done;
  long long gbase0;  // position of (s0, kv head 0) in the shares
  long long gend;    // end of this CTA's share
  int s0, h0, p00;   // the first unit of the share (s0 >= num_seqs: none)
  uint32_t tmem_base;
  int abort_flag;
};

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

__device__ __forceinline__ int clamp_ctx(const MQParams& p, int s) {
  const int c = __ldg(&p.context_lens[s]);
  return c < 0 ? 0 : min(c, p.max_blocks * 16);
}
__device__ __forceinline__ int ctx_tiles(int ctx) { return (ctx + BN - 1) / BN; }
// The shares are measured in key tiles plus kSegCost tiles' worth of time per
// (sequence, kv head) -- a segment's fixed costs (its query load, its first
// S, its epilogue after the last O += P V) -- so that a CTA whose share holds
// many short sequences takes fewer tiles.  A (sequence, kv head) with nt key
// tiles spans nt + kSegCost positions; its partition p starts at position
// kSegCost + 8 p.
constexpr int kSegCost = 3;
__device__ __forceinline__ int seq_weight(int nt) { return nt > 0 ? nt + kSegCost : 0; }

// A run of consecutive partitions p0 .. p1 (tiles t0 .. t1 - 1) of one
// (sequence s, kv head h) inside this CTA's share.
struct Seg {
  int s, h, p0, p1, t0, t1, ctx, nt, np;
  long long gbase;  // position of (s, kv head 0) in the CTAs' shares
  bool whole;       // p0 .. p1 are all of (s, h)'s partitions
};

// Settle on the segment that starts at (s, h, p0) or at the next unit after
// it; false when no unit starting before gend is left.
__device__ bool seg_settle(const MQParams& p, Seg& g, long long gend) {
  for (;;) {
    if (g.s >= p.num_seqs) return false;
    g.np = (g.nt + kPT - 1) / kPT;
    if (g.p0 < g.np) break;
    g.p0 = 0;
    if (++g.h == p.n_kv) {
      g.h = 0;
      g.gbase += (long long)p.n_kv * seq_weight(g.nt);
      if (++g.s >= p.num_seqs) return false;
      g.ctx = clamp_ctx(p, g.s);
      g.nt = ctx_tiles(g.ctx);
    }
  }
  // position of (s, h)'s partition 0
  const long long gsh = g.gbase + (long long)g.h * seq_weight(g.nt) + kSegCost;
  if (gsh + (long long)kPT * g.p0 >= gend) return false;
  const long long last = (gend - 1 - gsh) / kPT;  // last partition starting in the share
  g.p1 = (int)min((long long)(g.np - 1), last);
  g.t0 = g.p0 * kPT;
  g.t1 = min(g.nt, (g.p1 + 1) * kPT);
  g.whole = g.p0 == 0 && g.p1 == g.np - 1;
  return true;
}
__device__ __forceinline__ bool seg_first(const MQParams& p, const Bars* B, Seg& g) {
  g.s = B->s0;
  g.h = B->h0;
  g.p0 = B->p00;
  g.gbase = B->gbase0;
  if (g.s >= p.num_seqs) return false;
  g.ctx = clamp_ctx(p, g.s);
  g.nt = ctx_tiles(g.ctx);
  return seg_settle(p, g, B->gend);
}
__device__ __forceinline__ bool seg_next(const MQParams& p, const Bars* B, Seg& g) {
  if (g.p1 < g.np - 1) return false;  // the share ends inside this (sequence, kv head)
  g.p0 = g.np;
  return seg_settle(p, g, B->gend);
}

// T = n_kv x the sum of the sequences' weights (seq_weight), by one warp;
// flags contexts beyond the table (once, from CTA 0 when `report`).
__device__ long long total_weight(const MQParams& p, int lane, bool report) {
  long long part = 0;
  bool over = false;
  // four independent loads in flight per lane
  for (int s0 = lane; s0 < p.num_seqs; s0 += 128) {
    int c[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = s0 + 32 * u;
      c[u] = s < p.num_seqs ? __ldg(&p.context_lens[s]) : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      over |= c[u] > p.max_blocks * 16;
      part += seq_weight(ctx_tiles(c[u] < 0 ? 0 : min(c[u], p.max_blocks * 16)));
    }
  }
  if (report && blockIdx.x == 0 && __any_sync(0xffffffffu, over) && lane == 0)
    flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
  return part * p.n_kv;
}
// Start of share c of C: floor(c T / C) without overflow.
__device__ __forceinline__ long long share_start(long long T, long long c, long long C) {
  return (T / C) * c + (T % C) * c / C;
}
// The sequence s whose span of positions [gs, gs + n_kv w) contains X < T,
// its position gs and its weight w, by one warp (the same values in every
// lane); false when no sequence does.
__device__ bool locate(const MQParams& p, long long X, int lane, int& s_out, long long& gs_out,
                       int& w_out) {
  long long acc = 0;  // position of the chunk's first sequence
  // the next chunk's context length is loaded while this one is scanned
  int c_next = lane < p.num_seqs ? __ldg(&p.context_lens[lane]) : 0;
  for (int base = 0; base < p.num_seqs; base += 32) {
    const int s = base + lane;
    const int c = c_next;
    c_next = s + 32 < p.num_seqs ? __ldg(&p.context_lens[s + 32]) : 0;
    const int cc = c < 0 ? 0 : min(c, p.max_blocks * 16);
    const int n = s < p.num_seqs ? seq_weight(ctx_tiles(cc)) : 0;
    int incl = n;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, m);
      if (lane >= m) incl += v;
    }
    const long long gs = acc + (long long)(incl - n) * p.n_kv;
    const long long ge = acc + (long long)incl * p.n_kv;
    const uint32_t hit = __ballot_sync(0xffffffffu, gs <= X && X < ge);
    if (hit) {
      const int src = __ffs(hit) - 1;
      s_out = __shfl_sync(0xffffffffu, s, src);
      gs_out = __shfl_sync(0xffffffffu, gs, src);
      w_out = __shfl_sync(0xffffffffu, n, src);
      return true;
    }
    acc += (long long)__shfl_sync(0xffffffffu, incl, 31) * p.n_kv;
  }
  return false;
}

// This CTA's share [c T / C, (c + 1) T / C), found by one warp; its first
// unit is the first partition that starts at or after the share's start.
__device__ void find_share(const MQParams& p, Bars* B, int lane) {
  const long long T = total_weight(p, lane, true);
  const long long C = gridDim.x, c = blockIdx.x;
  const long long gbeg = share_start(T, c, C), gend = share_start(T, c + 1, C);
  int s0 = p.num_seqs, h0 = 0, p00 = 0, w = 0;
  long long gb = 0;
  if (gbeg < gend && locate(p, gbeg, lane, s0, gb, w)) {
    const long long local = gbeg - gb;
    h0 = (int)(local / w);
    p00 = (int)((max(0LL, local % w - kSegCost) + kPT - 1) / kPT);
  } else {
    s0 = p.num_seqs;
  }
  if (lane == 0) {
    B->s0 = s0;
    B->h0 = h0;
    B->p00 = p00;
    B->gbase0 = gb;
    B->gend = gend;
  }
}

// Rows of a block that the TMA cannot load whole (the block the context ends
// in, blocks past the context, blocks with an out-of-range id), written by
// the load warp into operand stage `op` at rows 16 m .. 16 m + 15: rows below
// `nvalid` are copied from pool row `src_row` on, the rest are zeros.
__device__ __forceinline__ void write_block_rows(uint8_t* op, int m, const uint8_t* pool,
                                                 long long src_row, int nvalid, int lane) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int idx = lane + 32 * u, r = idx >> 4, cc = idx & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < nvalid)
      v = __ldg(reinterpret_cast<const uint4*>(pool + (src_row + r) * (D * 2) + cc * 16));
    *reinterpret_cast<uint4*>(op + b_off(16 * m + r, cc)) = v;
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    mq_tc_kernel(const MQParams p, const void* __restrict__ k_pool,
                 const void* __restrict__ v_pool, const __grid_constant__ CUtensorMap tmq,
                 const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  using T16 = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars* B = reinterpret_cast<Bars*>(smem + kBarOff);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group, nrows = p.q_len * G;
  const int nlive = (nrows + 15) / 16;  // softmax warps with rows
  const uint32_t live_threads = 32u * nlive;

  // the merge kernel may be scheduled now; it waits for this grid to finish
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKS; ++s) {
      mbar_init(&B->k_full[s], 1);
      mbar_init(&B->k_empty[s], 1);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(&B->v_full[s], 1);
      mbar_init(&B->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B->q_full[s], 1);
      mbar_init(&B->q_empty[s], 1);
      mbar_init(&B->s_full[s], 1);
      mbar_init(&B->s_empty[s], live_threads);
      mbar_init(&B->pv_done[s], 1);
      mbar_init(&B->o_free[s], live_threads);
    }
    mbar_init(&B->p_full, live_threads);
    mbar_init(&B->done, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::alloc(&B->tmem_base, kTmemCols);
  if (warp == kKWarp) find_share(p, B, lane);
  if (warp < kSoftWarps) {
    // Q rows past q_len x G stay zero in both Q buffers
    for (int idx = threadIdx.x; idx < 2 * kQBytes / 16; idx += kSoftWarps * 32)
      reinterpret_cast<uint4*>(smem + kQOff)[idx] = make_uint4(0, 0, 0, 0);
    tc::fence_async_smem();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = B->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 256;

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // per tile t: S(t) = Q K(t)^T into S buffer t % 2, then O += P(t-1) V(t-1)
    // of the previous tile (its P is written by then, or soon)
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_f16(BF16, false, BM, BN);
      constexpr uint32_t idesc_pv = tc::idesc_f16(BF16, true, BM, D);
      Seg g;
      bool have = seg_first(p, B, g), ok = true, issued = false;
      int t = 0, n = 0;
      int pend_t = -1, pend_n = 0;
      bool pend_first = false;
      auto issue_pv = [&]() -> bool {
        const int pb = pend_t & 1, sv = pend_t % kVS, ob = pend_n & 1;  // pv_done[pb]
        // O buffer ob is free once the run of tiles two back has been read out
        if (pend_first && pend_n >= 2 &&
            !wait_or_abort(&B->o_free[ob], ((pend_n - 2) >> 1) & 1, B, p.dev_err))
          return false;
        if (!wait_or_abort(&B->v_full[sv], (pend_t / kVS) & 1, B, p.dev_err) ||
            !wait_or_abort(&B->p_full, pend_t & 1, B, p.dev_err))
          return false;
        tc::fence_after();
        const uint32_t aP = sbase + kPOff;
        const uint32_t bV = sbase + kVOff + sv * kOpBytes;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {  // 16 keys = two 8-row groups of V
          const uint32_t pa = (kk >> 2) * 8192 + (kk & 3) * 32;
          const uint64_t vd = tc::smem_desc(bV + kk * 2048, 16384);
          tc::mma(tO + ob * 128, tc::smem_desc(aP + pa), vd, idesc_pv,
                  (pend_first && kk == 0) ? 0u : 1u);
          if constexpr (BF16)  // P's rounding residual, into the same accumulator
            tc::mma(tO + ob * 128, tc::smem_desc(aP + kPBytes + pa), vd, idesc_pv, 1u);
        }
        tc::commit(&B->pv_done[pb]);
        tc::commit(&B->v_empty[sv]);
        return true;
      };
      for (; have && ok; have = seg_next(p, B, g), ++n) {
        const int qb = n & 1;
        ok = wait_or_abort(&B->q_full[qb], (n >> 1) & 1, B, p.dev_err);
        const uint32_t aQ = sbase + kQOff + qb * kQBytes;
        for (int jj = g.t0; jj < g.t1 && ok; ++jj, ++t) {
          const int sb = t & 1, sk = t % kKS;
          ok = wait_or_abort(&B->k_full[sk], (t / kKS) & 1, B, p.dev_err) &&
               (t < 2 || wait_or_abort(&B->s_empty[sb], ((t - 2) >> 1) & 1, B, p.dev_err));
          if (!ok) break;
          tc::fence_after();
          const uint32_t bK = sbase + kKOff + sk * kOpBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma(tS + sb * BN, tc::smem_desc(aQ + (kk >> 2) * 8192 + (kk & 3) * 32),
                    tc::smem_desc(bK + (kk >> 2) * 16384 + (kk & 3) * 32), idesc_s, kk > 0);
          issued = true;
          tc::commit(&B->s_full[sb]);
          tc::commit(&B->k_empty[sk]);  // the K stage is free once S(t) is done
          if (jj == g.t1 - 1) tc::commit(&B->q_empty[qb]);
          if (pend_t >= 0 && !(ok = issue_pv())) break;
          pend_t = t;
          pend_n = n;
          pend_first = jj == g.t0;
        }
      }
      if (ok && pend_t >= 0) issue_pv();
      // everything issued above has completed before TMEM is released
      if (issued) {
        tc::commit(&B->done);
        mbar_wait(&B->done, 0);
      }
    }
  } else if (warp == kKWarp || warp == kVWarp) {
    // ------------------------------------------------------------ loads
    // warp 5: Q of each segment and the K tiles; warp 6: the V tiles
    const bool vop = warp == kVWarp;
    const int NS = vop ? kVS : kKS;
    if (lane == 0) {
      if (!vop) prefetch_tensormap(&tmq);
      prefetch_tensormap(vop ? &tmv : &tmk);
    }
    const uint64_t ef = l2_policy_evict_first();  // K/V are read once
    const CUtensorMap* map = vop ? &tmv : &tmk;
    const uint8_t* pool = static_cast<const uint8_t*>(vop ? v_pool : k_pool);
    Seg g;
    bool have = seg_first(p, B, g), ok = true;
    int t = 0, n = 0, issued = 0;
    constexpr uint32_t kBlockBytes = 16u * D * 2u;  // one operand's rows of a block
    for (; have && ok; have = seg_next(p, B, g), ++n) {
      if (!vop) {
        // Q of this segment: the q_len x G rows of kv head h, one 3-D box
        // (64 columns x G heads x q_len queries) per half
        const int qb = n & 1;
        if (lane == 0) {
          ok = n < 2 || (wait_or_abort(&B->q_empty[qb], ((n - 2) >> 1) & 1, B, p.dev_err) &&
                         !aborted(B));
          if (ok) {
            uint8_t* dq = smem + kQOff + qb * kQBytes;
            mbar_arrive_expect_tx(&B->q_full[qb], (uint32_t)nrows * 256u);
            tc::tma_load_3d(dq, &tmq, &B->q_full[qb], 0, g.h * G, g.s * p.q_len);
            tc::tma_load_3d(dq + 8192, &tmq, &B->q_full[qb], 64, g.h * G, g.s * p.q_len);
          }
        }
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      }
      const int32_t* bt = p.block_tables + (size_t)g.s * p.max_blocks;
      for (int jj = g.t0; jj < g.t1 && ok; ++jj, ++t) {
        // lane m < 8: block m of the tile.  A whole block of the context with
        // an id in range is two 64-column boxes; the warp writes the rows of
        // every other block itself before the stage's arrival
        const int blk = jj * 8 + lane;
        const bool in_ctx = lane < 8 && blk * 16 < g.ctx;
        const int phys = in_ctx ? __ldg(&bt[blk]) : -1;
        const bool in_range = phys >= 0 && phys < p.num_blocks;
        if (!vop && in_ctx && !in_range) flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
        const bool whole = in_ctx && in_range && blk * 16 + 16 <= g.ctx;
        const uint32_t whole_m = __ballot_sync(0xffffffffu, whole);
        const uint32_t part_m = __ballot_sync(0xffffffffu, lane < 8 && !whole);
        const int y = whole ? (phys * p.n_kv + g.h) * 16 : 0;  // row of the [rows][D] view
        const int st = t % NS;
        uint64_t* full = vop ? &B->v_full[st] : &B->k_full[st];
        uint64_t* empty = vop ? &B->v_empty[st] : &B->k_empty[st];
        if (t >= NS) {
          const bool w = wait_or_abort(empty, ((t - NS) / NS) & 1, B, p.dev_err) && !aborted(B);
          ok = __all_sync(0xffffffffu, w);
          if (!ok) break;
        }
        uint8_t* d = smem + (vop ? kVOff : kKOff) + st * kOpBytes;
        for (uint32_t pm = part_m; pm; pm &= pm - 1) {
          const int m = __ffs(pm) - 1;
          const int ph = __shfl_sync(0xffffffffu, phys, m);
          const bool ok_id = ph >= 0 && ph < p.num_blocks;
          const int nvalid = ok_id ? max(0, min(16, g.ctx - (jj * 8 + m) * 16)) : 0;
          write_block_rows(d, m, pool, ok_id ? (long long)(ph * p.n_kv + g.h) * 16 : 0,
                           nvalid, lane);
        }
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(full, __popc(whole_m) * kBlockBytes);
        __syncwarp();
        if (whole) {
          tma_load_2d_hint(d + lane * 2048, map, full, 0, y, ef);
          tma_load_2d_hint(d + kOpBytes / 2 + lane * 2048, map, full, 64, y, ef);
        }
        issued = t + 1;
      }
    }
    // loads still in flight when the CTA gives up land before it exits
    if (lane == 0)
      for (int u = max(0, issued - NS); u < issued; ++u)
        mbar_wait(vop ? &B->v_full[u % kVS] : &B->k_full[u % kKS], (u / NS) & 1);
  } else {
    // ------------------------------------------------------------ softmax
    // sequences without context: all-zero rows (strided over the CTAs)
    for (int s = blockIdx.x; s < p.num_seqs; s += gridDim.x) {
      if (clamp_ctx(p, s) > 0) continue;
      uint4* o = reinterpret_cast<uint4*>(static_cast<T16*>(p.out) +
                                          (size_t)s * p.q_len * p.n_q * D);
      for (int idx = threadIdx.x; idx < p.q_len * p.n_q * D / 8; idx += kSoftWarps * 32)
        o[idx] = make_uint4(0, 0, 0, 0);
    }
    if (warp < nlive) {
      const int ra = 16 * warp + (lane >> 2), rb = ra + 8;  // this thread's two rows
      const int ia = ra / G, ga = ra % G, ib = rb / G, gb = rb % G;
      const bool va = ra < nrows, vb = rb < nrows;
      const int cpair = 2 * (lane & 3);  // key (and dim) offset inside each 8
      const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
      // stmatrix: lane l addresses row l % 8 of matrix l / 8; matrices 0..3 of
      // a store are (rows a, chunk 2u), (rows b, 2u), (a, 2u+1), (b, 2u+1)
      const int sm_row = 16 * warp + 8 * ((lane >> 3) & 1) + (lane & 7);
      const int sm_chunk = lane >> 4;
      const float sl = p.scale_log2;
      Seg g;
      bool have = seg_first(p, B, g), fail = false;
      int t = 0, n = 0;
      auto all_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, wait_or_abort(bar, parity, B, p.dev_err));
      };
      for (; have && !fail; have = seg_next(p, B, g), ++n) {
        const int ob = n & 1;
        const int H = g.ctx - p.q_len;  // keys before the first query; may be negative
        const int lim_a = va ? H + ia : 0x7fffffff, lim_b = vb ? H + ib : 0x7fffffff;
        float m_a = -INFINITY, m_b = -INFINITY;  // log2-domain max used so far
        float l_a = 0.f, l_b = 0.f;  // this thread's share of the row sums
        for (int jj = g.t0; jj < g.t1; ++jj, ++t) {
          const int sb = t & 1;
          if (!all_wait(&B->s_full[sb], (t >> 1) & 1)) {
            fail = true;
            break;
          }
          tc::fence_after();
          // x[32 hf + 4 k + e]: column 64 hf + 8 k + cpair + (e & 1) of row
          // a (e < 2) or b (e >= 2)
          uint32_t xr[64];
          tc::ld16x256b_x8(tS + sb * BN + lane_base, xr);
          tc::ld16x256b_x8(tS + sb * BN + 64 + lane_base, xr + 32);
          tc::wait_ld();
          tc::fence_before();
          mbar_arrive(&B->s_empty[sb]);  // S buffer sb may take S(t + 2)
          float x[64];
#pragma unroll
          for (int e = 0; e < 64; ++e) x[e] = __uint_as_float(xr[e]);
          const int kbase = jj * BN;
          const bool full = __all_sync(0xffffffffu, kbase + BN - 1 <= min(lim_a, lim_b)) &&
                            sl > 0.f;
          float xa = -INFINITY, xb = -INFINITY, sle = sl;
          if (full) {
            float ma[2] = {-INFINITY, -INFINITY}, mb[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              ma[q & 1] = fmaxf(ma[q & 1], fmaxf(x[4 * q], x[4 * q + 1]));
              mb[q & 1] = fmaxf(mb[q & 1], fmaxf(x[4 * q + 2], x[4 * q + 3]));
            }
            xa = fmaxf(ma[0], ma[1]) * sl;
            xb = fmaxf(mb[0], mb[1]) * sl;
          } else {
            // scores times the scale, -inf past a row's last visible key
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int key = kbase + 64 * (q >> 3) + 8 * (q & 7) + cpair;
              x[4 * q] = key <= lim_a ? x[4 * q] * sl : -INFINITY;
              x[4 * q + 1] = key + 1 <= lim_a ? x[4 * q + 1] * sl : -INFINITY;
              x[4 * q + 2] = key <= lim_b ? x[4 * q + 2] * sl : -INFINITY;
              x[4 * q + 3] = key + 1 <= lim_b ? x[4 * q + 3] * sl : -INFINITY;
              xa = fmaxf(xa, fmaxf(x[4 * q], x[4 * q + 1]));
              xb = fmaxf(xb, fmaxf(x[4 * q + 2], x[4 * q + 3]));
            }
            sle = 1.f;
          }
          // the row's four threads
          xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 1));
          xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 1));
          xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 2));
          xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 2));
          // lazy rescale: only when a row's max grew by more than 2^8
          const float mna = fmaxf(m_a, xa), mnb = fmaxf(m_b, xb);
          const bool ra_ = mna > m_a + kRescaleLog2, rb_ = mnb > m_b + kRescaleLog2;
          float alpha_a = 1.f, alpha_b = 1.f;
          if (ra_) {
            alpha_a = exp2f(m_a - mna);  // 0 on a row's first keys
            l_a *= alpha_a;
            m_a = mna;
          }
          if (rb_) {
            alpha_b = exp2f(m_b - mnb);
            l_b *= alpha_b;
            m_b = mnb;
          }
          // a row that has seen no key yet exponentiates against 0 (P = 0)
          const float nma = m_a == -INFINITY ? 0.f : -m_a;
          const float nmb = m_b == -INFINITY ? 0.f : -m_b;
          // P pairs: pv[2 c] row a, pv[2 c + 1] row b, keys 8 c + cpair, + 1
          uint32_t pv[32], pr[32];
          float sa[2] = {0.f, 0.f}, sbm[2] = {0.f, 0.f};
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float a0 = tc::ex2(fmaf(x[4 * q], sle, nma));
            const float a1 = tc::ex2(fmaf(x[4 * q + 1], sle, nma));
            const float b0 = tc::ex2(fmaf(x[4 * q + 2], sle, nmb));
            const float b1 = tc::ex2(fmaf(x[4 * q + 3], sle, nmb));
            sa[q & 1] += a0 + a1;
            sbm[q & 1] += b0 + b1;
            pv[2 * q] = pack2<BF16>(a0, a1);
            pv[2 * q + 1] = pack2<BF16>(b0, b1);
            if constexpr (BF16) {
              const float2 ha = unpack2<true>(pv[2 * q]), hb = unpack2<true>(pv[2 * q + 1]);
              pr[2 * q] = pack2<true>(a0 - ha.x, a1 - ha.y);
              pr[2 * q + 1] = pack2<true>(b0 - hb.x, b1 - hb.y);
            }
          }
          l_a += sa[0] + sa[1];
          l_b += sbm[0] + sbm[1];
          // the P buffer is free, and O may be rescaled, once O += P V of
          // tile t - 1 has completed
          if (t >= 1 && !all_wait(&B->pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1)) {
            fail = true;
            break;
          }
          // this warp's rows of O are rescaled (rarely); the first tile of a
          // segment starts O afresh
          if (jj > g.t0 && __any_sync(0xffffffffu, ra_ || rb_)) {
            tc::fence_after();
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
              uint32_t o[32];
              const uint32_t ta = tO + ob * 128 + 64 * hf + lane_base;
              tc::ld16x256b_x8(ta, o);
              tc::wait_ld();
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                o[4 * q] = __float_as_uint(__uint_as_float(o[4 * q]) * alpha_a);
                o[4 * q + 1] = __float_as_uint(__uint_as_float(o[4 * q + 1]) * alpha_a);
                o[4 * q + 2] = __float_as_uint(__uint_as_float(o[4 * q + 2]) * alpha_b);
                o[4 * q + 3] = __float_as_uint(__uint_as_float(o[4 * q + 3]) * alpha_b);
              }
              tc::st16x256b_x8(ta, o);
            }
            tc::wait_st();
          }
          const uint32_t pbase = sbase + kPOff;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t ad = pbase + a_off(sm_row, 2 * u + sm_chunk);
            tc::stsm_x4(ad, pv[4 * u], pv[4 * u + 1], pv[4 * u + 2], pv[4 * u + 3]);
            if constexpr (BF16)
              tc::stsm_x4(ad + kPBytes, pr[4 * u], pr[4 * u + 1], pr[4 * u + 2], pr[4 * u + 3]);
          }
          tc::fence_async_smem();
          tc::fence_before();
          mbar_arrive(&B->p_full);
        }
        if (fail) break;
        // ------------------------------------------------ segment epilogue
        const int tl = t - 1;  // the segment's last tile
        if (!all_wait(&B->pv_done[tl & 1], (tl >> 1) & 1)) {
          fail = true;
          break;
        }
        tc::fence_after();
        uint32_t o[64];
        tc::ld16x256b_x8(tO + ob * 128 + lane_base, o);
        tc::ld16x256b_x8(tO + ob * 128 + 64 + lane_base, o + 32);
        tc::wait_ld();
        tc::fence_before();
        mbar_arrive(&B->o_free[ob]);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
        // rows of out / the workspace: [seq][query][q head]
        const size_t rowa = ((size_t)g.s * p.q_len + ia) * p.n_q + (size_t)g.h * G + ga;
        const size_t rowb = ((size_t)g.s * p.q_len + ib) * p.n_q + (size_t)g.h * G + gb;
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // row a, then row b
          const bool v = half ? vb : va;
          if (!v) continue;
          const size_t row = half ? rowb : rowa;
          const float l = half ? l_b : l_a, m = half ? m_b : m_a;
          if (g.whole) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint32_t* out = reinterpret_cast<uint32_t*>(static_cast<T16*>(p.out) + row * D);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int e = 32 * (q >> 3) + 4 * (q & 7) + 2 * half;
              out[(64 * (q >> 3) + 8 * (q & 7) + cpair) / 2] =
                  pack2<BF16>(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
            }
          } else {
            float* wo = p.ws_o + (row * p.n_parts_max + g.p0) * D;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int e = 32 * (q >> 3) + 4 * (q & 7) + 2 * half;
              *reinterpret_cast<float2*>(wo + 64 * (q >> 3) + 8 * (q & 7) + cpair) =
                  make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1]));
            }
            if ((lane & 3) == 0) {
              p.ws_ml[row * p.n_parts_max + g.p0] = make_float2(m, l);
              for (int pp = g.p0 + 1; pp <= g.p1; ++pp)
                p.ws_ml[row * p.n_parts_max + pp] = make_float2(-INFINITY, 0.f);
            }
          }
        }
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc::dealloc(tmem, kTmemCols);
  }
}

// Combines the segments of the (sequence, kv head) pairs split between CTAs.
// Merge CTA c (the grid is the attention kernel's) looks at the boundary
// between shares c and c + 1: if the (sequence, kv head) whose span holds
// that boundary has partitions starting on both sides of it, and its first
// partition lies in share c, this CTA merges its q_len x G rows -- so each
// split pair is merged once, by the CTA of its first partition.  One warp per
// row; the row's partition slots in increasing order, empty ones (max -inf)
// skipped.  Every other row was written whole by the attention kernel.
template <typename OutT>
__global__ void __launch_bounds__(256) mq_merge_kernel(const MQParams p) {
  __shared__ int sh_s, sh_h, sh_np;
  // finding the pair reads only the context lengths, so it overlaps the
  // attention kernel (this grid is its programmatic dependent); the
  // workspace is read after pdl_wait
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  if (warp == 0) {
    int s = -1, h = 0, np = 0;
    const long long C = gridDim.x, c = blockIdx.x;
    if (c + 1 < C) {
      const long long T = total_weight(p, lane, false);
      const long long X = share_start(T, c + 1, C);
      int s0, w;
      long long gs;
      if (X < T && locate(p, X, lane, s0, gs, w)) {
        const long long local = X - gs;
        const int hh = (int)(local / w);
        const long long r = local % w;  // X's offset in (s0, hh)'s span
        const int npp = (w - kSegCost + kPT - 1) / kPT;
        const int before = r <= kSegCost ? 0 : (int)((r - kSegCost + kPT - 1) / kPT);
        if (before >= 1 && before < npp && gs + (long long)hh * w + kSegCost >= share_start(T, c, C)) {
          s = s0;
          h = hh;
          np = npp;
        }
      }
    }
    if (lane == 0) {
      sh_s = s;
      sh_h = h;
      sh_np = np;
    }
  }
  __syncthreads();
  pdl_wait();  // the attention kernel's results
  if (sh_s < 0) return;
  const int np = sh_np;
  for (int k = warp; k < p.q_len * G; k += 8) {
    const long long gw = ((long long)sh_s * p.q_len + k / G) * p.n_q + (long long)sh_h * G + k % G;
    const float2* ml = p.ws_ml + gw * p.n_parts_max;
    float M = -INFINITY;
    for (int pp = lane; pp < np; pp += 32) M = fmaxf(M, ml[pp].x);
    M = warp_max_xor(M, 1);
    float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float* wo = p.ws_o + gw * p.n_parts_max * D + lane * 4;
    for (int pp = 0; pp < np; ++pp) {
      const float2 v = ml[pp];
      if (v.x == -INFINITY) continue;
      const float wt = exp2f(v.x - M);
      L += wt * v.y;
      const float4 x = *reinterpret_cast<const float4*>(wo + (size_t)pp * D);
      acc[0] += wt * x.x;
      acc[1] += wt * x.y;
      acc[2] += wt * x.z;
      acc[3] += wt * x.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    constexpr bool kBf = std::is_same<OutT, __nv_bfloat16>::value;
    uint2 o;
    o.x = pack2<kBf>(acc[0] * inv, acc[1] * inv);
    o.y = pack2<kBf>(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(reinterpret_cast<OutT*>(p.out) + gw * D + lane * 4) = o;
  }
}

int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1)
      v = 148;
    n[dev] = v;
  }
  return n[dev];
}

template <bool BF16>
cudaError_t launch_t(const MQParams& p, const void* k_pool, const void* v_pool,
                     const CUtensorMap* tmq, const CUtensorMap* tmk, const CUtensorMap* tmv,
                     bool merge, cudaStream_t st) {
  using T16 = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  static cudaError_t attr = cudaFuncSetAttribute(
      mq_tc_kernel<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (attr != cudaSuccess) return attr;
  mq_tc_kernel<BF16><<<sm_count(), kThreads, kSmemBytes, st>>>(p, k_pool, v_pool, *tmq, *tmk,
                                                                *tmv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !merge) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sm_count());  // one merge CTA per share boundary
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mq_merge_kernel<T16>, p);
}

}  // namespace

cudaError_t launch_mq_tc(const MQParams& p, bool bf16, const void* k_pool, const void* v_pool,
                         const CUtensorMap* tmq, const CUtensorMap* tmk, const CUtensorMap* tmv,
                         bool merge, cudaStream_t st) {
  if (p.num_seqs == 0) return cudaSuccess;
  return bf16 ? launch_t<true>(p, k_pool, v_pool, tmq, tmk, tmv, merge, st)
              : launch_t<false>(p, k_pool, v_pool, tmq, tmk, tmv, merge, st);
}

}  // namespace pa
