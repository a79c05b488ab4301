// Device helpers shared by the attention kernels: mbarriers with bounded
// waits, TMA loads, tcgen05 fences, shared-memory matrix descriptors, the
// exponential of the softmax, and the walk over a block's key tiles.
#pragma once

#include <cuda_bf16.h>

#include "nomas_internal.h"
#include "f32x2.cuh"

namespace nomas {
namespace {

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct WaitCtl {
  volatile int *abort;              // CTA-wide abort flag in shared memory
  int32_t *dev_err;
  unsigned long long limit_ns;
};

// Slow path of wait_phase: spins until the phase completes, the CTA aborts,
// or the time limit passes (then it raises the abort flag and reports).
__device__ __forceinline__ bool wait_phase_slow(uint32_t bar, uint32_t parity, volatile int *abort,
                                             int32_t *dev_err, unsigned long long limit_ns) {
  const unsigned long long start = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - start > limit_ns) {
        *abort = 1;
        if (dev_err != nullptr) atomicOr(dev_err, NOMAS_DEVERR_WAIT_TIMEOUT);
        return false;
      }
    }
  }
}

// Waits for the phase of `bar` with the given parity.  Returns false when the
// CTA is aborting (this wait ran out of time, or another role's did).
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, const WaitCtl &c) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_phase_slow(bar, parity, c.abort, c.dev_err, c.limit_ns);
}

// Teardown wait for operations this thread started itself: ignores the abort
// flag, still bounded.
__device__ __forceinline__ void drain_phase(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const unsigned long long start = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - start > limit_ns) return;
  }
}

// --------------------------------------------------------------------- TMA --
// 2-D tiled TMA load into shared memory, completing on `bar`, with an L2
// eviction-priority policy (K/V tiles are re-read by every query block of the
// head and should stay in L2; Q is read once).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ----------------------------------------------------------------- tcgen05 --
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^x for a pair of values on the FMA pipe, to share the exponential work of
// the softmax between the MUFU unit and the FMA units.  Cody-Waite style
// reduction: adding 1.5 * 2^23 rounds x to the nearest integer j (kept in the
// low mantissa bits of the sum), f = x - j lies in [-1/2, 1/2] exactly, 2^f
// comes from a degree-3 polynomial whose coefficients were fitted by the
// Remez exchange algorithm (fit_exp2_poly.py in this package) to minimise the
// relative error on [-1/2, 1/2]
// (max 7.5e-5, far below the 2^-9 rounding step of the bf16 P it feeds), and
// j is added to the exponent field.  x is clamped at -125 so the exponent
// cannot underflow; 2^-125 stands in for 0.
constexpr float kShifter = 12582912.0f;  // 1.5 * 2^23
constexpr float kPc0 = 0.9999280571937561f;
constexpr float kPc1 = 0.6932609677314758f;
constexpr float kPc2 = 0.2426111251115799f;
constexpr float kPc3 = 0.0551716685295105f;
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x) {
  float2 v = unf2(x);
  v.x = fmaxf(v.x, -125.f);
  v.y = fmaxf(v.y, -125.f);
  const uint64_t xc = f2(v.x, v.y);
  const uint64_t t = add2(xc, f2(kShifter, kShifter));
  const uint64_t jf = add2(t, f2(-kShifter, -kShifter));
  const uint64_t fr = fma2(jf, f2(-1.f, -1.f), xc);
  uint64_t pp = fma2(f2(kPc3, kPc3), fr, f2(kPc2, kPc2));
  pp = fma2(pp, fr, f2(kPc1, kPc1));
  pp = fma2(pp, fr, f2(kPc0, kPc0));
  const float2 pv = unf2(pp), tv = unf2(t);
  return f2(__uint_as_float(__float_as_uint(pv.x) + (__float_as_uint(tv.x) << 23)),
            __uint_as_float(__float_as_uint(pv.y) + (__float_as_uint(tv.y) << 23)));
}

// The MMA lane must issue an instruction every 64 cycles to keep the tensor
// core busy (M=128, N=128, K=16 takes 64 cycles), so descriptors are built
// once and each K step only adds a compile-time offset to the start-address
// field (bits 0-13, in 16-byte units; addresses stay below 256 KiB, so the
// add never carries into the other fields).
__device__ __forceinline__ uint64_t desc_plus(uint64_t d, uint32_t bytes) {
  return d + (uint64_t)(bytes >> 4);
}

// Walks this block's key tiles as (span, tile within the span).  Dense mode
// visits the global tiles [g0, g1) in order (all of them without a key
// split); sparse mode
// reads the block's list of global tile ids (tiles numbered across the
// concatenated spans) and skips ids outside the spans -- every role walks the
// same list the same way, so they agree on the sequence.
template <bool kSparse>
struct TileWalk {
  const AttnArgs &p;
  const int32_t *list;
  int n_list;
  int idx = 0, s = 0, kt = 0, g = 0, g_end = 0;
  __device__ TileWalk(const AttnArgs &a, const int32_t *l, int n, int g0, int g1)
      : p(a), list(l), n_list(n) {
    if constexpr (!kSparse) {
      g = g0;
      g_end = g1;
      while (s + 1 < p.n_spans && g0 >= p.tile_base[s + 1]) ++s;
      kt = g0 - p.tile_base[s];
    }
  }
  // Next tile; false at the end.  `bad` is set when an invalid id was skipped.
  __device__ __forceinline__ bool next(int *span, int *ktile, bool *bad) {
    if constexpr (kSparse) {
      while (idx < n_list) {
        const int g = list[idx++];
        if (g < 0 || g >= p.tile_base[p.n_spans]) {
          *bad = true;
          continue;
        }
        int t = 0;
        while (t + 1 < p.n_spans && g >= p.tile_base[t + 1]) ++t;
        *span = t;
        *ktile = g - p.tile_base[t];
        return true;
      }
      return false;
    } else {
      if (g >= g_end) return false;
      *span = s;
      *ktile = kt;
      ++g;
      if (++kt >= p.tile_base[s + 1] - p.tile_base[s]) {
        ++s;
        kt = 0;
      }
      return true;
    }
  }
};

}  // namespace
}  // namespace nomas
