// Paged decode attention for sm_100a.
//
// One new query token per sequence attends to its whole cached context,
// softmax(scale * q . K^T) . V ("LLM inference optimization: KV cache &
// PagedAttention", §二), reading K/V block by block through the sequence's
// block table ("vLLM explained", "兩層實作").  Decode re-reads the whole cache
// each step and is bound by HBM bandwidth (same page, §一.2), so the design
// goal is to keep enough bytes in flight and to touch every byte once.
//
// Split-context scheme.  Grid = (context partition, kv head, sequence); a
// partition is 1024 consecutive logical tokens (64 blocks) with 16-bit caches
// and 2048 with fp8 caches.  Each CTA:
//   * one producer warp streams the partition's 16-token K and V tiles with
//     2-D TMA loads (no multicast) into an 8-stage shared-memory ring guarded
//     by mbarriers -- the block table indirection becomes one TMA row
//     coordinate per tile;
//   * four consumer warps take blocks round-robin; each keeps an online
//     max / sum / output state for all G query heads of the kv head, so every
//     K/V byte loaded serves the whole GQA group;
//   * the warps' states are merged in shared memory; a sequence with one
//     partition is written straight to `out`, otherwise the partition's
//     (max, sum, unnormalised output) goes to the workspace and the reduce
//     kernel merges partitions in fixed order.
// Work assignment depends only on logical positions, so results are the same
// bits for any permutation of the physical blocks.
//
// Per-block math (16-bit and fp8 caches): S^T[16 tok][8 heads] = K . Q^T and
// O^T[d][8 heads] += V^T . P^T, each as m16n8k16 warp MMAs with the GQA group
// as N=8 (fp32 accumulate; with 16-bit caches P enters as a 16-bit value plus
// its 16-bit rounding residual).  For fp8 caches the E4M3 codes are widened to f16
// exactly in registers after ldmatrix (no shared-memory round trip), and the
// per-tensor scales are applied to the scores and to the final output.  fp32
// inputs use a CUDA-core path with fp32 arithmetic throughout.
#include <type_traits>
#include <utility>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kNW = 4;  // consumer warps
constexpr int kThreads = (kNW + 1) * 32;
constexpr int kStages = 8;
constexpr int kMaxGroup = 8;

template <int D, bool FP8>
struct MmaLayout {
  static constexpr int kPart = FP8 ? kPartFp8 : kPart16;  // tokens per partition
  static constexpr int kPartBlocks = kPart / 16;
  static_assert(kPartBlocks <= kThreads, "one thread per block id");
  static constexpr int kTileBytes = 16 * D * (FP8 ? 1 : 2);  // one (block, head) tile
  static constexpr int kStageBytes = 2 * kTileBytes;          // K + V
  static constexpr int kIdsOff = kStages * kStageBytes;
  static constexpr int kBarOff = kIdsOff + kPartBlocks * 4;
  static constexpr int kSmemBytes = kBarOff + 2 * kStages * 8 + 1024;  // + align slack
  static constexpr int kMergeFloats = kNW * 8 * D + 3 * kNW * 8 + 2 * 32;
  static_assert(kMergeFloats * 4 <= kIdsOff, "merge scratch must fit in the ring");
  static_assert(kStageBytes % 1024 == 0, "1024-B aligned tiles");
};

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// Clamp a context length into [0, capacity]; a length beyond the table's
// capacity is a caller error that is flagged, never read past.
__device__ __forceinline__ int clamp_ctx(int ctx, int cap, int32_t* dev_err, bool report) {
  if (ctx > cap) {
    if (report) flag_error(dev_err, PA_DEVERR_BLOCK_ID);
    return cap;
  }
  return ctx < 0 ? 0 : ctx;
}

// Row of q / out (and of the workspace) that MMA column c of a CTA serves.  A
// CTA's 8 columns are (query, head) pairs 8cg .. 8cg+7 of the sequence's
// q_len x G pairs for its kv head, pair m being query m / G, head m % G of the
// group; rows are laid out [seq][query][q head].  With one query per sequence
// (decode) column c is simply head kvh*G + c.
__device__ __forceinline__ size_t col_row(const DecodeParams& p, int seq, int kvh, int cg,
                                          int c) {
  const int m = 8 * cg + c, i = m / p.group;
  return ((size_t)seq * p.q_len + i) * p.n_q + (size_t)kvh * p.group + (m - i * p.group);
}

// Group CTA of the shared-prefix decode: column c of column group cg is
// head m % G of member m / G of group grp (m = 8cg + c); -1 for a column of an
// unused member slot.  *member receives the member's sequence.
__device__ __forceinline__ long long grp_col_row(const DecodeParams& p, int grp, int kvh, int cg,
                                                 int c, int* member) {
  const int m = 8 * cg + c, i = m / p.group;
  int s = i < p.grp_width ? p.grp_members[(size_t)grp * p.grp_width + i] : -1;
  if (s >= p.n_seqs_all) s = -1;  // not a sequence: the column is left out
  *member = s;
  if (s < 0) return -1;
  return (long long)s * p.n_q + (long long)kvh * p.group + (m - i * p.group);
}

// Merge the consumer warps' (m, l, O) states held in shared memory and write
// the partition result.  The CTA's nvc columns are "virtual columns"
// vc = 8 gi + c of its column groups gi (group cg0 + gi of the sequence's
// (query, head) pairs); group gi's state is spread over the wpg warps
// w = gi + cpc2 * ph.  Plain decode: one group (cg0 = 0, cpc2 = 1) over all
// kNW warps, nvc = G.  mo: [kNW][8][D], mm/ml/wgt: [kNW][8] (log2-domain max,
// running sum, merge weight), Ls/Ms: [32].  Called by every thread of the CTA.
template <int D, typename OutT, bool MQ>
__device__ __forceinline__ void merge_and_store(float* mo, float* mm, float* ml, float* wgt,
                                                float* Ls, float* Ms, int nthreads,
                                                const DecodeParams& p, int seq, int kvh,
                                                int cg0, int cpc2, int wpg, int nvc, int part,
                                                int n_parts_seq, int part_tokens, bool grp) {
  const int tid = threadIdx.x;
  if (tid < nvc) {
    const int gi = tid >> 3, c = tid & 7;
    float M = -INFINITY;
    for (int ph = 0; ph < wpg; ++ph) M = fmaxf(M, mm[(gi + cpc2 * ph) * 8 + c]);
    float L = 0.f;
    for (int ph = 0; ph < wpg; ++ph) {
      const int w = gi + cpc2 * ph;
      const float wv = (M == -INFINITY) ? 0.f : exp2f(mm[w * 8 + c] - M);
      wgt[w * 8 + c] = wv;
      L += wv * ml[w * 8 + c];
    }
    Ls[tid] = L;
    Ms[tid] = M;
  }
  __syncthreads();
  // the row of a virtual column and how many partitions its sequence has
  // (in a group CTA each column has its own member sequence)
  auto target = [&](int vc, int& np) -> long long {
    if constexpr (!MQ) {  // plain decode: the G heads of the kv head
      np = n_parts_seq;
      return ((long long)seq * p.n_q + (long long)kvh * p.group) + vc;
    }
    if (grp) {
      int ms;
      const long long r = grp_col_row(p, seq, kvh, cg0 + (vc >> 3), vc & 7, &ms);
      if (r >= 0) {
        const int c = max(0, min(p.context_lens[ms], p.max_blocks * 16));
        np = (c + part_tokens - 1) / part_tokens;
      }
      return r;
    }
    np = n_parts_seq;
    return (long long)col_row(p, seq, kvh, cg0 + (vc >> 3), vc & 7);
  };
  for (int idx = tid; idx < nvc * D; idx += nthreads) {
    const int vc = idx / D, dd = idx % D;
    const int gi = vc >> 3, c = vc & 7;
    int np = 1;
    const long long row = target(vc, np);
    if (row < 0) continue;
    float acc = 0.f;
    for (int ph = 0; ph < wpg; ++ph) {
      const int w = gi + cpc2 * ph;
      acc += wgt[w * 8 + c] * mo[(w * 8 + c) * D + dd];
    }
    if (np == 1) {
      const float L = Ls[vc];
      reinterpret_cast<OutT*>(p.out)[row * D + dd] =
          from_f32<OutT>(L > 0.f ? acc / L * p.out_mul : 0.f);
    } else {
      p.ws_o[(row * p.n_parts_max + part) * D + dd] = acc;
    }
  }
  if (tid < nvc) {
    int np = 1;
    const long long row = target(tid, np);
    if (row >= 0 && np > 1)
      p.ws_ml[row * p.n_parts_max + part] = make_float2(Ms[tid], Ls[tid]);
  }
}
// ---------------------------------------------------------------------------
// tensor-core engine: 16-bit caches (MMA in the cache's type) and fp8 caches
// (MMA in f16); Q_BF16 selects the query / output type.
// ---------------------------------------------------------------------------
// MQ: several queries per sequence (multi-query decode, e.g. verifying draft
// tokens): query i of q_len sits at position ctx - q_len + i and sees keys
// 0 .. ctx - q_len + i.  A CTA takes up to 4 column groups of its kv head
// (blockIdx.y = kv head x group quad); with cpc groups (cpc2 = cpc rounded up
// to 1, 2 or 4) consumer warp w takes group w % cpc2 and every (4 / cpc2)-th
// block, so one K/V stage serves all of the CTA's groups.
// Registers: 96 with 16-bit caches (three CTAs per SM, a shared-memory
// limit); 80 with fp8 caches, so that five CTAs fit an SM (96 allowed four):
// the fp8 kernel is bound by its warps' per-block latency, and the fifth CTA
// hides more of it than the few spilled registers cost (measured 403 against
// 440 us on the mixed-step decode; 64 registers, six CTAs: 473 us).
template <int D, bool FP8, bool Q_BF16, bool MQ>
__global__ void __launch_bounds__(kThreads) __maxnreg__(FP8 ? 80 : 96) decode_mma_kernel(
    const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
    const DecodeParams p) {
  using L = MmaLayout<D, FP8>;
  using QT = typename std::conditional<Q_BF16, __nv_bfloat16, __half>::type;
  constexpr bool kMmaBf16 = Q_BF16 && !FP8;
  constexpr int KS = D / 16;  // 16-wide k steps over the head dim / m tiles of O^T

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  // the merge kernel may be scheduled as this grid drains (it waits for it)
  pdl_launch_dependents();

  const int part = blockIdx.x;
  const int G = p.group;
  // shared-prefix decode: the first n_groups z-indices are groups, whose CTAs
  // take every member's queries over the group's shared blocks (K/V through
  // the first member's table, whole shared partitions only, no causal mask);
  // the rest are sequences.
  const bool grp = MQ && p.grp_members != nullptr && (int)blockIdx.z < p.n_groups;
  const int seq = (MQ && p.grp_members && !grp) ? (int)blockIdx.z - p.n_groups : (int)blockIdx.z;
  const int n_pairs = grp ? p.grp_width * G : G * p.q_len;  // (query or member, head) pairs
  const int n_cg = (n_pairs + 7) >> 3;
  int kvh = blockIdx.y, cg0 = 0, cpc = 1, cpc2 = 1;
  if constexpr (MQ) {
    const int nquad = (p.n_cg + 3) >> 2;  // the grid's quads per kv head
    kvh = (int)blockIdx.y / nquad;
    cg0 = 4 * ((int)blockIdx.y - kvh * nquad);
    if (cg0 >= n_cg) return;
    cpc = min(4, n_cg - cg0);
    cpc2 = cpc == 1 ? 1 : (cpc == 2 ? 2 : 4);
  }
  const int wpg = kNW / cpc2;  // warps per column group
  // virtual columns in use: 8 per full group, the last group's remainder
  const int nvc = MQ ? min(8 * cpc, n_pairs - 8 * cg0) : G;
  constexpr int kPart = L::kPart;
  int tseq = seq, ctx;
  if (grp) {
    tseq = p.grp_members[(size_t)seq * p.grp_width];
    const int sb = p.grp_shared_blocks[seq];
    if (tseq < 0 || tseq >= p.n_seqs_all || sb < 0 || sb > p.max_blocks) {
      if (threadIdx.x == 0 && part == 0 && blockIdx.y == 0) flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
      return;
    }
    ctx = (sb * 16 / kPart) * kPart;
    if (part * kPart >= ctx) return;
  } else {
    ctx = clamp_ctx(p.context_lens[seq], p.max_blocks * 16, p.dev_err,
                    threadIdx.x == 0 && part == 0 && blockIdx.y == 0);
  }
  const int tok0 = part * kPart;
  if (MQ && !grp && p.seq_group && tok0 < ctx) {  // partitions the group CTAs compute
    const int gi = p.seq_group[seq];
    if (gi >= p.n_groups) {
      if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
    } else if (gi >= 0) {
      const int sb = p.grp_shared_blocks[gi];
      if (sb >= 0 && sb <= p.max_blocks && part < sb * 16 / kPart) return;
    }
  }
  if (tok0 >= ctx) {
    if (part == 0) {  // empty context: all-zero output rows
      QT* out = reinterpret_cast<QT*>(p.out);
      for (int idx = threadIdx.x; idx < nvc * D; idx += kThreads) {
        const int vc = idx / D;
        const size_t row = MQ ? col_row(p, seq, kvh, cg0 + (vc >> 3), vc & 7)
                              : (size_t)seq * p.n_q + (size_t)kvh * G + vc;
        out[row * D + idx % D] = from_f32<QT>(0.f);
      }
    }
    return;
  }
  const int ntok = min(kPart, ctx - tok0);
  const int nblk = (ntok + 15) >> 4;
  const int n_parts_seq = (ctx + kPart - 1) / kPart;

  int32_t* ids = reinterpret_cast<int32_t*>(smem + L::kIdsOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x < nblk) {
    int id = p.block_tables[(size_t)tseq * p.max_blocks + (tok0 >> 4) + threadIdx.x];
    if (id < 0 || id >= p.num_blocks) {
      flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
      id = -1;
    }
    ids[threadIdx.x] = id;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], cpc);  // released by every group that reads the stage
    }
    fence_mbar_init();
  }
  __syncthreads();

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[KS][4];
#pragma unroll
  for (int i = 0; i < KS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  const int g = lane >> 2, t = lane & 3;

  if (warp == kNW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      const uint64_t pol = l2_policy_evict_first();
      // the cache may have been written by the kernel before this one (the
      // step's slot write, launched ahead of us): wait for it before reading
      pdl_wait();
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait(&empty[s], ((j / kStages) - 1) & 1, p.wait_ns)) {
          flag_error(p.dev_err, PA_DEVERR_TIMEOUT);
          break;
        }
        const int id = ids[j];
        uint8_t* kt = smem + s * L::kStageBytes;
        uint8_t* vt = kt + L::kTileBytes;
        if (j == p.skip_tile) {
          // test hook (pa_test_decode_timeout): the stage is never filled, so
          // the waits on it run out
        } else if (id >= 0) {
          mbar_arrive_expect_tx(&full[s], 2 * L::kTileBytes);
          const int row = (id * p.n_kv + kvh) * 16;
          if (FP8 || D == 64) {
            tma_load_2d_hint(kt, &tmk, &full[s], 0, row, pol);
            tma_load_2d_hint(vt, &tmv, &full[s], 0, row, pol);
          } else {
            tma_load_2d_hint(kt, &tmk, &full[s], 0, row, pol);
            tma_load_2d_hint(kt + 2048, &tmk, &full[s], 64, row, pol);
            tma_load_2d_hint(vt, &tmv, &full[s], 0, row, pol);
            tma_load_2d_hint(vt + 2048, &tmv, &full[s], 64, row, pol);
          }
        } else {
          mbar_arrive(&full[s]);
        }
        issued = j + 1;
      }
      // Before the ring is reused as merge scratch, make sure no load issued
      // here is still landing (only matters if a consumer gave up early).
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        mbar_wait(&full[j % kStages], (j / kStages) & 1, p.wait_ns);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int gi = warp % cpc2, ph = warp / cpc2;  // column group, block phase
    const int cg = cg0 + gi;
    const int ncols = MQ ? min(8, n_pairs - 8 * cg) : G;  // this warp's columns
    const bool active = !MQ || gi < cpc;
    // Q as the B operand (k = head dim, n = query head of the group); heads
    // beyond the group size are zero.  The fp8 path pairs MMA k-index
    // (2t, 2t+1 | 2t+8, 2t+9) with dims (4t, 4t+1 | 4t+2, 4t+3) of each
    // 16-dim step so that K can be read as whole 32-bit words; Q uses the
    // same pairing, which leaves the dot products unchanged.
    uint32_t qb[KS][2];
    float col_scale;  // scale x log2 e (x k_scale) x 2^-e of column g
    {
      bool hv = g < ncols;
      size_t r = 0;
      if (grp) {
        int ms;
        const long long gr = hv ? grp_col_row(p, seq, kvh, cg, g, &ms) : -1;
        hv = gr >= 0;
        r = hv ? (size_t)gr : 0;
      } else if constexpr (MQ) {
        r = col_row(p, seq, kvh, cg, hv ? g : 0);
      } else {
        r = (size_t)seq * p.n_q + (size_t)kvh * G + (hv ? g : 0);
      }
      const QT* qrow = reinterpret_cast<const QT*>(p.q) + r * D;
      // fp8 cache with bf16 queries: the column's row enters the f16 MMAs
      // times 2^e (its largest magnitude in [2^14, 2^15)); its scores are
      // scaled by 2^-e.  The four lanes t of a column hold all of its dims.
      int e = 0;
      if constexpr (FP8 && Q_BF16) {
        uint32_t mag = 0;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const uint2 w = *reinterpret_cast<const uint2*>(qrow + 16 * kk + 4 * t);
          mag = max(mag, max(bf16x2_max_mag(w.x), bf16x2_max_mag(w.y)));
        }
        mag = hv ? mag : 0u;
        mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, 1));
        mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, 2));
        e = f16_row_shift(mag);
      }
      const float up = exp2i(e);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        if constexpr (FP8) {
          const int d0 = 16 * kk + 4 * t;
          qb[kk][0] = pack2<false>(to_f32(qrow[d0]) * up, to_f32(qrow[d0 + 1]) * up);
          qb[kk][1] = pack2<false>(to_f32(qrow[d0 + 2]) * up, to_f32(qrow[d0 + 3]) * up);
        } else {
          qb[kk][0] = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * t);
          qb[kk][1] = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 8 + 2 * t);
        }
        if (!hv) qb[kk][0] = qb[kk][1] = 0u;
      }
      col_scale = p.scale_log2 * exp2i(-e);
    }
    // score scales of the lane's two columns 2t, 2t+1 (held by lanes g = 2t, 2t+1)
    const float sl_a = __shfl_sync(0xffffffffu, col_scale, 8 * t);
    const float sl_b = __shfl_sync(0xffffffffu, col_scale, 8 * t + 4);
    const uint32_t sbase = smem_u32(smem);
    const int q4 = lane >> 3;
    // multi-query causal limits: keys at positions >= lim are masked for the
    // lane's two columns (2t, 2t+1); columns not in use keep the full context
    int lim_a = ctx, lim_b = ctx;
    const int lim_min = ctx - p.q_len + 1;  // the first query's limit
    if constexpr (MQ) {
      if (2 * t < ncols) lim_a = lim_min + (8 * cg + 2 * t) / G;
      if (2 * t + 1 < ncols) lim_b = lim_min + (8 * cg + 2 * t + 1) / G;
    }

    for (int j = active ? ph : nblk; j < nblk; j += wpg) {
      const int s = j % kStages;
      if (!mbar_wait(&full[s], (j / kStages) & 1, p.wait_ns)) {
        flag_error(p.dev_err, PA_DEVERR_TIMEOUT);
        break;
      }
      if (ids[j] >= 0) {
        const int valid = min(16, ntok - 16 * j);
        const uint32_t kt = sbase + s * L::kStageBytes;
        // ---- scores S^T = K . Q^T  (16 tokens x 8 heads)
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (!FP8) {
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            const int row = (lane & 7) + ((q4 & 1) << 3);
            const int C = 2 * kk + (q4 >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kt + swz128((C >> 3) * 2048 + row * 128 + (C & 7) * 16), a0, a1, a2, a3);
            mma_16816<kMmaBf16>(sc, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
          }
        } else {
          // the fp8 tile read as 16-bit pairs: ldmatrix hands lane (g, t) the 4
          // codes of dims 4t..4t+3 of a 16-dim step for tokens g and g+8 --
          // the permuted k pairing the Q fragments were built with
#pragma unroll
          for (int k2 = 0; k2 < KS / 2; ++k2) {
            const int row = (lane & 7) + ((q4 & 1) << 3);
            const uint32_t off = row * D + (2 * k2 + (q4 >> 1)) * 16;
            uint32_t r0, r1, r2, r3;
            ldsm_x4(kt + (D == 128 ? swz128(off) : swz64(off)), r0, r1, r2, r3);
            mma_16816<false>(sc, e4m3x2_to_f16x2(r0 & 0xffffu), e4m3x2_to_f16x2(r1 & 0xffffu),
                             e4m3x2_to_f16x2(r0 >> 16), e4m3x2_to_f16x2(r1 >> 16),
                             qb[2 * k2][0], qb[2 * k2][1]);
            mma_16816<false>(sc, e4m3x2_to_f16x2(r2 & 0xffffu), e4m3x2_to_f16x2(r3 & 0xffffu),
                             e4m3x2_to_f16x2(r2 >> 16), e4m3x2_to_f16x2(r3 >> 16),
                             qb[2 * k2 + 1][0], qb[2 * k2 + 1][1]);
          }
        }
        // ---- online softmax (log2 domain); lane holds tokens g, g+8 of heads 2t, 2t+1
        float x0 = sc[0] * sl_a, x1 = sc[1] * sl_b, x2 = sc[2] * sl_a, x3 = sc[3] * sl_b;
        if (valid < 16) {
          if (g >= valid) x0 = x1 = -INFINITY;
          if (g + 8 >= valid) x2 = x3 = -INFINITY;
        }
        if constexpr (MQ) {
          const int kb = tok0 + 16 * j;  // position of the block's first key
          if (!grp && kb + 16 > lim_min) {  // (a group launch has no causal mask)
            const int k0 = kb + g, k1 = k0 + 8;
            if (k0 >= lim_a) x0 = -INFINITY;
            if (k0 >= lim_b) x1 = -INFINITY;
            if (k1 >= lim_a) x2 = -INFINITY;
            if (k1 >= lim_b) x3 = -INFINITY;
          }
        }
        float b0m = fmaxf(x0, x2), b1m = fmaxf(x1, x3);
        b0m = warp_max_xor(b0m, 4);
        b1m = warp_max_xor(b1m, 4);
        const float n0 = fmaxf(m0, b0m), n1 = fmaxf(m1, b1m);
        // with several queries a column can have every key so far masked
        // (max -inf); exponentiate against 0 then so that c = p = 0, not NaN
        const float e0 = (MQ && n0 == -INFINITY) ? 0.f : n0;
        const float e1 = (MQ && n1 == -INFINITY) ? 0.f : n1;
        const float c0 = exp2f(m0 - e0), c1 = exp2f(m1 - e1);
        const float p0 = exp2f(x0 - e0), p1 = exp2f(x1 - e1);
        const float p2 = exp2f(x2 - e0), p3 = exp2f(x3 - e1);
        l0 = l0 * c0 + (p0 + p2);
        l1 = l1 * c1 + (p1 + p3);
        m0 = n0;
        m1 = n1;
        if (__any_sync(0xffffffffu, c0 != 1.f || c1 != 1.f)) {  // a running max grew
#pragma unroll
          for (int i = 0; i < KS; ++i) {
            o[i][0] *= c0;
            o[i][1] *= c1;
            o[i][2] *= c0;
            o[i][3] *= c1;
          }
        }
        // P^T as the B operand: transpose the two 8x8 (token x head) halves.
        // With 16-bit caches P is split into a rounded part and its rounding
        // residual (two MMAs), which keeps ~16 significant bits of P: a single
        // bf16 P would cost up to 2^-9 |v - o| on short contexts.
        const uint32_t ph01 = pack2<kMmaBf16>(p0, p1), ph23 = pack2<kMmaBf16>(p2, p3);
        const uint32_t pb0 = movmatrix_t(ph01);
        const uint32_t pb1 = movmatrix_t(ph23);
        uint32_t pl0 = 0u, pl1 = 0u;
        if constexpr (!FP8) {
          const float2 h01 = unpack2<kMmaBf16>(ph01), h23 = unpack2<kMmaBf16>(ph23);
          pl0 = movmatrix_t(pack2<kMmaBf16>(p0 - h01.x, p1 - h01.y));
          pl1 = movmatrix_t(pack2<kMmaBf16>(p2 - h23.x, p3 - h23.y));
        }
        // ---- V^T tiles (A operand), O^T += V^T . P^T; tokens past the context
        // are masked out of V (their bytes are not part of the sequence)
        uint32_t mk01 = 0xffffffffu, mk23 = 0xffffffffu;
        if (valid < 16) {
          mk01 = ((2 * t < valid) ? 0x0000ffffu : 0u) | ((2 * t + 1 < valid) ? 0xffff0000u : 0u);
          mk23 = ((2 * t + 8 < valid) ? 0x0000ffffu : 0u) |
                 ((2 * t + 9 < valid) ? 0xffff0000u : 0u);
        }
        // the masks are applied only in a partition's partial last block
        auto pv = [&](auto masked) {
          constexpr bool kMask = decltype(masked)::value;
          if constexpr (!FP8) {
            const uint32_t vbase = kt + L::kTileBytes;
#pragma unroll
            for (int i = 0; i < KS; ++i) {
              const int row = (lane & 7) + ((q4 >> 1) << 3);
              const int C = 2 * i + (q4 & 1);
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(vbase + swz128((C >> 3) * 2048 + row * 128 + (C & 7) * 16), a0, a1, a2,
                        a3);
              if constexpr (kMask) {
                a0 &= mk01;
                a1 &= mk01;
                a2 &= mk23;
                a3 &= mk23;
              }
              mma_16816<kMmaBf16>(o[i], a0, a1, a2, a3, pb0, pb1);
              mma_16816<kMmaBf16>(o[i], a0, a1, a2, a3, pl0, pl1);
            }
          } else {
            // the fp8 V tile read as 16-bit pairs with ldmatrix.trans: a lane gets
            // the codes of dims (2g, 2g+1) of a 16-dim step for tokens (2t, 2t+1);
            // byte permutes split them into one V^T row per dim.  MMA row g holds
            // dim 16i+2g and row g+8 dim 16i+2g+1 (undone when O is written out).
            const uint32_t vbase = kt + L::kTileBytes;
#pragma unroll
            for (int i2 = 0; i2 < KS / 2; ++i2) {
              const int row = (lane & 7) + ((q4 & 1) << 3);
              const uint32_t off = row * D + (2 * i2 + (q4 >> 1)) * 16;
              uint32_t r[4];
              ldsm_x4_t(vbase + (D == 128 ? swz128(off) : swz64(off)), r[0], r[1], r[2], r[3]);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint32_t lo = r[2 * h], hi = r[2 * h + 1];  // tokens 0-7 / 8-15
                // widened on the integer pipe (x 2^-8, folded into the output
                // scale) so that K's hardware conversions have the
                // conversion pipe to themselves
                uint32_t a0 = e4m3x2_to_f16x2_div256(lo, 0x4240u);
                uint32_t a1 = e4m3x2_to_f16x2_div256(lo, 0x4341u);
                uint32_t a2 = e4m3x2_to_f16x2_div256(hi, 0x4240u);
                uint32_t a3 = e4m3x2_to_f16x2_div256(hi, 0x4341u);
                if constexpr (kMask) {
                  a0 &= mk01;
                  a1 &= mk01;
                  a2 &= mk23;
                  a3 &= mk23;
                }
                mma_16816<false>(o[2 * i2 + h], a0, a1, a2, a3, pb0, pb1);
              }
            }
          }
        };
        if (valid < 16)
          pv(std::true_type{});
        else
          pv(std::false_type{});
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 4);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 8);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 16);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 4);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 8);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 16);
  }
  __syncthreads();  // ring free: reuse it as merge scratch

  float* mo = reinterpret_cast<float*>(smem);
  float* mm = mo + kNW * 8 * D;
  float* ml = mm + kNW * 8;
  float* wgt = ml + kNW * 8;
  float* Ls = wgt + kNW * 8;
  float* Ms = Ls + 32;
  if (warp < kNW) {
    float* mw = mo + warp * 8 * D;
    // O^T row g / g+8 of m-tile i is dim 16i+g / 16i+g+8 (16-bit caches) or
    // dim 16i+2g / 16i+2g+1 (fp8 caches)
    const int d_lo = FP8 ? 2 * g : g, d_hi = FP8 ? 2 * g + 1 : g + 8;
#pragma unroll
    for (int i = 0; i < KS; ++i) {
      mw[(2 * t) * D + 16 * i + d_lo] = o[i][0];
      mw[(2 * t + 1) * D + 16 * i + d_lo] = o[i][1];
      mw[(2 * t) * D + 16 * i + d_hi] = o[i][2];
      mw[(2 * t + 1) * D + 16 * i + d_hi] = o[i][3];
    }
    if (g == 0) {
      mm[warp * 8 + 2 * t] = m0;
      mm[warp * 8 + 2 * t + 1] = m1;
      ml[warp * 8 + 2 * t] = l0;
      ml[warp * 8 + 2 * t + 1] = l1;
    }
  }
  __syncthreads();
  merge_and_store<D, QT, MQ>(mo, mm, ml, wgt, Ls, Ms, kThreads, p, seq, kvh, cg0, cpc2, wpg, nvc,
                             part, n_parts_seq, kPart, grp);
}

// ---------------------------------------------------------------------------
// CUDA-core engine for fp32 inputs (exact fp32 arithmetic; small workloads).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kNW * 32) decode_simt_f32_kernel(const DecodeParams p) {
  constexpr int VPL = D / 32;  // dims per lane
  constexpr int kPart = kPart16;
  static_assert(kPart / 16 <= kNW * 32, "one thread per block id");
  __shared__ int32_t ids[kPart / 16];
  __shared__ float mo[kNW * 8 * D];
  __shared__ float mm[kNW * 8], ml[kNW * 8], wgt[kNW * 8], Ls[8], Ms[8];

  const int part = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
  const int G = p.group;
  const int ctx = clamp_ctx(p.context_lens[seq], p.max_blocks * 16, p.dev_err,
                            threadIdx.x == 0 && part == 0 && kvh == 0);
  const int tok0 = part * kPart;
  if (tok0 >= ctx) {
    if (part == 0) {
      float* out = reinterpret_cast<float*>(p.out);
      const size_t head0 = (size_t)seq * p.n_q + (size_t)kvh * G;
      for (int idx = threadIdx.x; idx < G * D; idx += kNW * 32) out[head0 * D + idx] = 0.f;
    }
    return;
  }
  const int ntok = min(kPart, ctx - tok0);
  const int nblk = (ntok + 15) >> 4;
  const int n_parts_seq = (ctx + kPart - 1) / kPart;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < nblk) {
    int id = p.block_tables[(size_t)seq * p.max_blocks + (tok0 >> 4) + threadIdx.x];
    if (id < 0 || id >= p.num_blocks) {
      flag_error(p.dev_err, PA_DEVERR_BLOCK_ID);
      id = -1;
    }
    ids[threadIdx.x] = id;
  }
  __syncthreads();

  const float* qp = reinterpret_cast<const float*>(p.q) + ((size_t)seq * p.n_q + (size_t)kvh * G) * D;
  float qv[kMaxGroup][VPL], o[kMaxGroup][VPL], m[kMaxGroup], l[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      qv[h][i] = h < G ? qp[h * D + lane * VPL + i] : 0.f;
      o[h][i] = 0.f;
    }
  }
  const float* kpool = reinterpret_cast<const float*>(p.k_pool);
  const float* vpool = reinterpret_cast<const float*>(p.v_pool);
  for (int j = warp; j < nblk; j += kNW) {
    const int id = ids[j];
    if (id < 0) continue;
    const int valid = min(16, ntok - 16 * j);
    const size_t base = ((size_t)id * p.n_kv + kvh) * 16 * D;
    for (int tt = 0; tt < valid; ++tt) {
      float kr[VPL], vr[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        kr[i] = kpool[base + tt * D + lane * VPL + i];
        vr[i] = vpool[base + tt * D + lane * VPL + i];
      }
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= G) break;
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < VPL; ++i) s = fmaf(qv[h][i], kr[i], s);
#pragma unroll
        for (int msk = 16; msk >= 1; msk >>= 1) s += __shfl_xor_sync(0xffffffffu, s, msk);
        s *= p.scale_log2;
        const float mn = fmaxf(m[h], s);
        const float c = exp2f(m[h] - mn), pr = exp2f(s - mn);
        l[h] = l[h] * c + pr;
#pragma unroll
        for (int i = 0; i < VPL; ++i) o[h][i] = fmaf(pr, vr[i], o[h][i] * c);
        m[h] = mn;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) mo[(warp * 8 + h) * D + lane * VPL + i] = o[h][i];
    if (lane == 0) {
      mm[warp * 8 + h] = m[h];
      ml[warp * 8 + h] = l[h];
    }
  }
  __syncthreads();
  merge_and_store<D, float, false>(mo, mm, ml, wgt, Ls, Ms, kNW * 32, p, seq, kvh, 0, 1, kNW, G,
                                   part, n_parts_seq, kPart, false);
}

// ---------------------------------------------------------------------------
// partition merge: one warp per (sequence, q head) with more than one
// partition; partitions combined in increasing order.
// ---------------------------------------------------------------------------
template <int D, typename OutT>
__global__ void __launch_bounds__(256) decode_reduce_kernel(const ReduceParams r) {
  pdl_wait();  // the partition results of the kernel before this one
  constexpr int VPL = D / 32;
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= r.num_seqs * r.n_q) return;
  const int seq = gw / r.n_q;
  int ctx = r.context_lens[seq];
  ctx = ctx < 0 ? 0 : min(ctx, r.max_blocks * 16);
  const int np = (ctx + r.part_tokens - 1) / r.part_tokens;
  if (np <= 1) return;
  const float2* ml = r.ws_ml + (size_t)gw * r.n_parts_max;
  float M = -INFINITY;
  for (int pp = lane; pp < np; pp += 32) M = fmaxf(M, ml[pp].x);
  M = warp_max_xor(M, 1);
  float L = 0.f, acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  const float* wo = r.ws_o + (size_t)gw * r.n_parts_max * D + lane * VPL;
  for (int pp = 0; pp < np; ++pp) {
    const float2 v = ml[pp];
    const float w = (v.x == -INFINITY) ? 0.f : exp2f(v.x - M);
    L += w * v.y;
    if constexpr (VPL == 4) {
      const float4 x = *reinterpret_cast<const float4*>(wo + (size_t)pp * D);
      acc[0] += w * x.x;
      acc[1] += w * x.y;
      acc[2] += w * x.z;
      acc[3] += w * x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2*>(wo + (size_t)pp * D);
      acc[0] += w * x.x;
      acc[1] += w * x.y;
    }
  }
  OutT* out = reinterpret_cast<OutT*>(r.out) + (size_t)gw * D + lane * VPL;
#pragma unroll
  for (int i = 0; i < VPL; ++i) out[i] = from_f32<OutT>(L > 0.f ? acc[i] / L * r.out_mul : 0.f);
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream is still running (see pdl_wait).
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
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

template <int D, bool FP8, bool Q_BF16, bool MQ>
cudaError_t launch_mma_(const DecodeParams& p, const CUtensorMap* tmk, const CUtensorMap* tmv,
                        cudaStream_t st) {
  using L = MmaLayout<D, FP8>;
  static cudaError_t attr = set_smem(decode_mma_kernel<D, FP8, Q_BF16, MQ>, L::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  dim3 grid(p.n_parts_grid, p.n_kv * (MQ ? (p.n_cg + 3) / 4 : 1), p.num_seqs);
  return launch_pdl(decode_mma_kernel<D, FP8, Q_BF16, MQ>, grid, dim3(kThreads), L::kSmemBytes,
                    st, *tmk, *tmv, p);
}

template <int D, bool FP8, bool Q_BF16>
cudaError_t launch_mma(const DecodeParams& p, const CUtensorMap* tmk, const CUtensorMap* tmv,
                       cudaStream_t st) {
  return (p.q_len > 1 || p.grp_members) ? launch_mma_<D, FP8, Q_BF16, true>(p, tmk, tmv, st)
                                        : launch_mma_<D, FP8, Q_BF16, false>(p, tmk, tmv, st);
}

template <int D>
cudaError_t launch_simt(const DecodeParams& p, cudaStream_t st) {
  dim3 grid(p.n_parts_grid, p.n_kv, p.num_seqs);
  decode_simt_f32_kernel<D><<<grid, kNW * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

int decode_num_parts(int max_blocks_per_seq, int part_tokens) {
  return (int)(((int64_t)max_blocks_per_seq * 16 + part_tokens - 1) / part_tokens);
}

bool decode_uses_tma(pa_dtype q_dt, pa_dtype kv_dt) { return q_dt != PA_F32; }

cudaError_t launch_decode_partitions(const DecodeParams& p, int D, pa_dtype q_dt,
                                     pa_dtype kv_dt, const CUtensorMap* tmk,
                                     const CUtensorMap* tmv, cudaStream_t st) {
  const bool fp8 = kv_dt == PA_FP8_E4M3;
  if (q_dt == PA_F32) return D == 64 ? launch_simt<64>(p, st) : launch_simt<128>(p, st);
  if (q_dt == PA_BF16) {
    if (fp8) return D == 64 ? launch_mma<64, true, true>(p, tmk, tmv, st)
                            : launch_mma<128, true, true>(p, tmk, tmv, st);
    return D == 64 ? launch_mma<64, false, true>(p, tmk, tmv, st)
                   : launch_mma<128, false, true>(p, tmk, tmv, st);
  }
  if (fp8) return D == 64 ? launch_mma<64, true, false>(p, tmk, tmv, st)
                          : launch_mma<128, true, false>(p, tmk, tmv, st);
  return D == 64 ? launch_mma<64, false, false>(p, tmk, tmv, st)
                 : launch_mma<128, false, false>(p, tmk, tmv, st);
}

cudaError_t launch_decode_reduce(const ReduceParams& r, int D, pa_dtype out_dt,
                                 cudaStream_t st) {
  const int blocks = (r.num_seqs * r.n_q + 7) / 8;
  if (blocks == 0) return cudaSuccess;
#define PA_RED(DD, T) launch_pdl(decode_reduce_kernel<DD, T>, dim3(blocks), dim3(256), 0, st, r)
  if (out_dt == PA_F32) return D == 64 ? PA_RED(64, float) : PA_RED(128, float);
  if (out_dt == PA_BF16) return D == 64 ? PA_RED(64, __nv_bfloat16) : PA_RED(128, __nv_bfloat16);
  return D == 64 ? PA_RED(64, __half) : PA_RED(128, __half);
#undef PA_RED
}

}  // namespace pa
