// Device-side helpers shared by the sm_100a kernels: mbarriers with bounded
// waits, TMA (bulk tensor) loads, warp-level matrix instructions, and the
// 128-byte / 64-byte shared-memory swizzles the TMA unit writes.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/pa.h"
#include "pa_internal.h"

namespace pa {

// kWaitLimitNs (pa_internal.h): how long a bounded wait lasts before it gives
// up; the caller then records PA_DEVERR_TIMEOUT and winds down.
constexpr uint32_t kWaitLimitIters = 1u << 26;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void flag_error(int32_t* dev_err, int bits) {
  if (dev_err) atomicOr(dev_err, bits);
}

// ---------------------------------------------------------------- mbarrier --

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false if the
// wait gave up (after limit_ns, or the iteration limit); it never spins
// forever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t i = 1; i < kWaitLimitIters; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0 && globaltimer_ns() - t0 > limit_ns) return false;
  }
  return false;
}

// --------------------------------------------------------------------- TMA --

// 2-D tiled bulk-tensor load global -> shared, completion counted on `bar`.
// No multicast: each CTA loads its own tiles.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Same, with an L2 cache policy (e.g. evict-first for data read once).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map,
                                                 uint64_t* bar, int x, int y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Byte offset inside a tile written by TMA with 128-byte swizzle: the 16-byte
// chunk index (bits 4-6) is XOR-ed with the 128-byte row index (bits 7-9).
// Tiles must start on a 1024-byte boundary.
__device__ __forceinline__ uint32_t swz128(uint32_t off) { return off ^ (((off >> 7) & 7u) << 4); }
// 64-byte swizzle: chunk bits 4-5 XOR-ed with bits 7-8 (512-byte aligned tiles).
__device__ __forceinline__ uint32_t swz64(uint32_t off) { return off ^ (((off >> 7) & 3u) << 4); }

// ------------------------------------------------------- warp matrix ops --

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start before the previous kernel in its stream has
// finished; pdl_wait() blocks the calling thread until that kernel has
// completed and its memory operations are visible.  pdl_launch_dependents()
// lets the next such kernel start once every CTA of this grid has issued it
// (or exited).  Without a preceding programmatic launch both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D(16x8, f32) += A(16x16) * B(16x8), A row-major, B column-major.
template <bool BF16>
__device__ __forceinline__ void mma_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// --------------------------------------------------------- conversions --

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  if constexpr (BF16) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
  } else {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
  }
}

// two E4M3 codes (low byte = first element) -> f16x2, exact
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t two) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// Two E4M3 codes, picked out of w by the byte selector (result bytes 0 and 2),
// as an f16x2 holding code x 2^-8, exactly, using integer ops only: with the
// code s.eeee.mmm in the low byte of a 16-bit lane, (b + (b & 0x80)) << 7
// puts eeee.mmm into f16's exponent/mantissa fields (bias 15 instead of 7,
// hence 2^-8; subnormal codes land on f16 subnormals) and the add carries the
// sign from bit 14 into bit 15.  E4M3's NaN code maps to a finite value.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_div256(uint32_t w, uint32_t sel) {
  const uint32_t y = __byte_perm(w, 0u, sel);  // [b_i, 0, b_j, 0]
  return (y + (y & 0x00800080u)) << 7;
}

// Rows of bf16 queries meet f16 operands (fp8 caches widen to f16 exactly):
// a row is multiplied by 2^e before its f16 rounding, e chosen so that its
// largest magnitude lands in [2^14, 2^15), and the row's scores by 2^-e after
// the product.  Both steps are exact (powers of two, no overflow: E4M3 values
// are below 2^9, so a product stays below 2^24 and a 128-term sum below 2^31);
// an element keeps all its bits unless it is below 2^-28 of the row's largest,
// and then its error is at most 2^-39 of that largest -- far under the
// rounding of the fp32 sum itself.

// The larger magnitude of the two bf16 values in w, as bf16 bits (for values
// that are not NaN the bits order like the magnitudes).
__device__ __forceinline__ uint32_t bf16x2_max_mag(uint32_t w) {
  return max(w & 0x7fffu, (w >> 16) & 0x7fffu);
}
// e for a row whose largest magnitude has the bf16 bits `mag` (0 for a zero,
// infinite or NaN row), clamped to [-110, 110] so that 2^e and a score scale
// times 2^-e stay normal floats.
__device__ __forceinline__ int f16_row_shift(uint32_t mag) {
  if (mag == 0u || mag >= 0x7f80u) return 0;
  const int ex = mag >= 0x80u ? (int)(mag >> 7) - 127 : -127;  // floor(log2 |x|)
  return min(max(14 - ex, -110), 110);
}
// 2^e as a float, for e in [-126, 127]
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }
// two bf16 values times `up` (a power of two), rounded to f16
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t w, float up) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
  return pack2<false>(f.x * up, f.y * up);
}

__device__ __forceinline__ float warp_max_xor(float v, int lo_mask) {
  for (int m = 16; m >= lo_mask; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

}  // namespace pa
