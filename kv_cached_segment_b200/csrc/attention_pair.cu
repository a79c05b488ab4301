// Segment-over-cache attention with the score tile triple-buffered in TMEM,
// so that the tensor core computes the scores of the next key tiles while
// the softmax is still working on the current one.
//
// "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
// (ai.thesatyajit.com), section "How one segment is made" (joint attention of
// text and video tokens, 16 heads of 128; the current segment reads earlier
// ones from the KV cache and sees itself and the text in full) and section
// "What 'world memory' stores" (the segment's queries attend over the cached
// keys and values).  Same operation, arguments and outputs as the two-tile
// kernel in attention.cu; only the schedule differs.
//
// Work unit: one CTA = one head x 128 query rows.  In the pair form, two CTAs
// of a cluster run as one 256-row unit on two SMs: every tcgen05.mma is
// cta_group::2 with M = 256, issued by the even CTA, and each CTA holds half
// of every key tile (keys 0-63 or 64-127 of K, dims 0-63 or 64-127 of V), so
// each SM reads half of the K/V bytes from L2 and half of the B operand from
// its own shared memory.
//
// TMEM (512 columns): S buffers at [0,128), [128,256), [256,384); O at
// [384,512).  The MMA lane issues, for K/V tiles j = 0, 1, ...:
//   S_0 S_1 S_2 | O += P_0 V_0, S_3 | O += P_1 V_1, S_4 | ...
// (S_j = Q K_j^T into buffer j mod 3; P_j, bf16, overwrites columns
// [0,32) and [64,96) of that buffer), so S_{j+1} and S_{j+2} are already in
// TMEM while the softmax works on S_j, and the softmax never waits for an
// O += P V to finish except to rescale O.
//
// Softmax: 8 warps.  Warps w and w + 4 share TMEM lanes 32 (w mod 4) ..
// 32 (w mod 4) + 31, one query row per lane; warp w takes keys 0-63 of each
// tile, warp w + 4 keys 64-127.  Both use the same running max m, which may
// be stale (P is formed against it, values up to 2^16, and the final division
// by the row sum formed with the same m makes the result exact).  After each
// tile the two warps of a row pair take a single named-barrier reduction:
// when either half saw a P sum above 2^16 (or overflow), or a wait ran out,
// they exchange their half-row maxima through shared memory, raise m, rescale
// their halves of O and the row sums, and redo the tile.
//
// Every wait is bounded (a globaltimer limit); on expiry the kernel records
// NOMAS_DEVERR_WAIT_TIMEOUT, drains its own TMA loads and MMAs, sets the
// block's rows of O and LSE to NaN, frees TMEM and returns.
//
// Both forms are selectable schedules, not the default: with one 128-row
// tile per CTA the MMA lane's per-tile waits and commits are comparable to
// the tile's 1,024 cycles of tensor work, and the pair's cross-CTA P
// signalling at cluster scope is costly, so the two-tile kernel is faster on
// every shape but the smallest.
#include <atomic>

#include <cuda_bf16.h>

#include "nomas_internal.h"
#include "f32x2.cuh"
#include "attn_device.cuh"
#include "tmem_ops.cuh"

namespace nomas {
namespace {

constexpr int kRows = 128;                            // query rows per CTA (MMA M per SM)
constexpr int kKeys = 128;                            // keys per K/V tile
constexpr int kSBufs = 3;                             // S buffers in TMEM
constexpr uint32_t kQBytes = kRows * kHeadDim * 2;    // 32 KiB
constexpr uint32_t kQHalf = kQBytes / 2;              // dims 0-63 / 64-127 of Q
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 384;

#ifndef NOMAS_PAIR_EXP2_FMA
#define NOMAS_PAIR_EXP2_FMA 2
#endif
// Pairs of P (out of every 8) whose exponentials run on the FMA pipe.
__device__ __forceinline__ constexpr bool fma_pair(int c) { return (c & 7) < NOMAS_PAIR_EXP2_FMA; }

// Shared-memory map.  A ring item is one K or one V tile (in the pair form,
// this CTA's half of it: 64 keys x 128 dims of K, or 128 keys x 64 dims of
// V, 16 KiB either way).
template <bool kPair>
struct PCfg {
  static constexpr uint32_t kItemBytes = kPair ? 16384u : 32768u;
  static constexpr int kStages = kPair ? 10 : 5;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = kQBytes;
  static constexpr uint32_t kOffBar = kOffKV + kStages * kItemBytes;
  static constexpr int kBarQFull = 0;                       // Q landed (both CTAs)
  static constexpr int kBarKVFull = 1;                      // + slot: item landed (both CTAs)
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;  // + slot: item consumed
  static constexpr int kBarSFull = kBarKVEmpty + kStages;   // + buffer: S ready
  static constexpr int kBarP = kBarSFull + kSBufs;          // + 2 buffer + half: P half ready
  // + buffer: O += P_j V_j done, j = buffer mod 3 (one barrier per S buffer,
  // so that a waiter never lags its barrier by two phases)
  static constexpr int kBarOReady = kBarP + 2 * kSBufs;
  static constexpr int kBarDrain = kBarOReady + kSBufs;
  // Pair form, odd CTA: its own loads land on these local barriers and a
  // forwarding lane passes each completion to the even CTA's barrier.
  static constexpr int kBarLocalQ = kBarDrain + 1;
  static constexpr int kBarLocalKV = kBarLocalQ + 1;        // + slot
  static constexpr int kNumBars = kBarLocalKV + kStages;
  static constexpr uint32_t kOffXchMax = (kOffBar + kNumBars * 8 + 15) & ~15u;  // [2][128] float2
  static constexpr uint32_t kOffXchL = kOffXchMax + 2 * kRows * 8;             // [2][128] float2
  static constexpr uint32_t kOffTmemSlot = kOffXchL + 2 * kRows * 8;
  static constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
  static constexpr uint32_t kSmemUsed = kOffAbort + 4;
  static constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;  // room to align the base
};
static_assert(PCfg<false>::kSmemAlloc <= 232448 && PCfg<true>::kSmemAlloc <= 232448,
              "shared memory per block");

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D,
// N = 128, M = 128 (one CTA) or 256 (CTA pair); A K-major; B K-major (K
// tiles) or MN-major (V tiles).
constexpr uint32_t pair_idesc(uint32_t m, uint32_t b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major << 16) | ((128u >> 3) << 17) |
         ((m >> 4) << 24);
}

// ------------------------------------------------------------------ cluster --
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Wait with cluster-scope acquire, for barriers that CTAs of the pair arrive on.
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __noinline__ bool wait_cl_slow(uint32_t bar, uint32_t parity, volatile int *abort,
                                         int32_t *dev_err, unsigned long long limit_ns) {
  const unsigned long long start = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cl(bar, parity)) return true;
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
template <bool kCl>
__device__ __forceinline__ bool wait_ph(uint32_t bar, uint32_t parity, const WaitCtl &c) {
  if constexpr (kCl) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    return wait_cl_slow(bar, parity, c.abort, c.dev_err, c.limit_ns);
  } else {
    return wait_phase(bar, parity, c);
  }
}

// ---------------------------------------------------------- tcgen05 forms --
// Every tcgen05 instruction of one kernel uses the same CTA group: ::1 for
// the single-CTA form, ::2 for the pair.
template <bool kPair>
__device__ __forceinline__ void tmem_alloc_all(uint32_t slot_addr) {
  if constexpr (kPair) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_addr),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  } else {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_addr),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
}
template <bool kPair>
__device__ __forceinline__ void tmem_free_all(uint32_t base) {
  if constexpr (kPair)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(kTmemCols)
                 : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(kTmemCols)
                 : "memory");
}
// D (+)= A B with A and B in shared memory; ACC = 0 overwrites D.
template <bool kPair, int ACC>
__device__ __forceinline__ void mma_ss2(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
  if constexpr (kPair)
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "n"(ACC)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "n"(ACC)
        : "memory");
}
// D (+)= A B with A (P) in tensor memory.
template <bool kPair>
__device__ __forceinline__ void mma_ts2(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
  if constexpr (kPair)
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrive on `bar` once the MMAs issued so far complete: in the pair form on
// the barrier at the same offset in both CTAs, else on this CTA's.
template <bool kPair>
__device__ __forceinline__ void commit_all(uint32_t bar) {
  if constexpr (kPair)
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}\n" ::"r"(bar)
        : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
// Arrive on this CTA's `bar` once the MMAs issued so far complete.
template <bool kPair>
__device__ __forceinline__ void commit_local(uint32_t bar) {
  if constexpr (kPair)
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// Named barrier of the two softmax warps that share a row quarter (ids 1-4,
// 64 threads): the OR of every thread's flag, the same in all of them.
__device__ __forceinline__ bool rows_any(int quarter, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %2, 0;\n\t"
      "bar.red.or.pred p, %1, 64, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(quarter + 1), "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void rows_sync(int quarter) {
  asm volatile("bar.sync %0, 64;" ::"r"(quarter + 1) : "memory");
}

template <bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
attention_pair_kernel(const __grid_constant__ AttnArgs p) {
  using C = PCfg<kPair>;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kItem = C::kItemBytes;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *const gbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  // Pair form: CTA rank 0 of the cluster issues the MMAs of both.
  const uint32_t rank = kPair ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int q_row0 = kPair ? (int)(blockIdx.x >> 1) * (2 * kRows) + (int)rank * kRows
                           : (int)blockIdx.x * kRows;

  const uint32_t sQ = base + C::kOffQ;
  const uint32_t sKV = base + C::kOffKV;
  auto bar = [&](int i) { return base + C::kOffBar + (uint32_t)i * 8u; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::kOffTmemSlot);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + C::kOffAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarQFull), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(C::kBarKVFull + s), 1);
      mbar_init(bar(C::kBarKVEmpty + s), 1);
      mbar_init(bar(C::kBarLocalKV + s), 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(bar(C::kBarSFull + b), 1);
      mbar_init(bar(C::kBarP + 2 * b), kPair ? 8 : 4);
      mbar_init(bar(C::kBarP + 2 * b + 1), kPair ? 8 : 4);
      mbar_init(bar(C::kBarOReady + b), 1);
    }
    mbar_init(bar(C::kBarDrain), 1);
    mbar_init(bar(C::kBarLocalQ), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc_all<kPair>(smem_u32(tmem_slot));
  tc_fence_before();
  __syncthreads();
  // Pair form: the peer's barriers are initialised before anything arrives
  // on them.
  if constexpr (kPair) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const WaitCtl ctl{abort_flag, p.dev_err, p.wait_limit_ns};
  // This block's share [g0, g1) of the key tiles (all of them unless the
  // keys are split across the grid's third dimension).
  const int total_tiles = p.tile_base[p.n_spans];
  const int g0 = (int)((int64_t)total_tiles * blockIdx.z / p.kv_splits);
  const int g1 = (int)((int64_t)total_tiles * (blockIdx.z + 1) / p.kv_splits);
  const int n_kv = g1 - g0;
  // Ring items in load order: K_0, K_1, K_2, then V_j, K_{j+3} for
  // j = 0, 1, ... (the order the MMA lane consumes them).
  const int n_items = 2 * n_kv;
  // Barrier on which this CTA's own loads of ring item slots complete.
  const int own_kv = kPair ? C::kBarLocalKV : C::kBarKVFull;
  const int own_q = kPair ? C::kBarLocalQ : C::kBarQFull;

  auto role_producer = [&]() {
    if (lane == 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      mbar_expect_tx(bar(own_q), kQBytes);
      for (int c = 0; c < 2; ++c)
        tma_load_2d(sQ + c * kQHalf, &p.tmap_q, bar(own_q), head * kHeadDim + c * 64, q_row0, pol_q);
      int t = 0;
      auto load_item = [&](int which, int s, int kt) -> bool {
        if (t == p.testing_skip_load) {  // testing hook: leave this load out
          ++t;
          return true;
        }
        const int slot = t % kStages;
        if (!wait_phase(bar(C::kBarKVEmpty + slot), ((uint32_t)(t / kStages) & 1u) ^ 1u, ctl))
          return false;
        const uint32_t fb = bar(own_kv + slot);
        const uint32_t dst = sKV + (uint32_t)slot * kItem;
        mbar_expect_tx(fb, kItem);
        const CUtensorMap *m = which == 0 ? &p.tmap_k[s] : &p.tmap_v[s];
        if constexpr (!kPair) {
          // whole tile: two boxes of 64 dims x 128 keys
          for (int c = 0; c < 2; ++c)
            tma_load_2d(dst + c * 16384u, m, fb, head * kHeadDim + c * 64, kt * kKeys, pol_kv);
        } else if (which == 0) {
          // K half: keys 64 rank .. + 63, two boxes of 64 dims x 64 keys
          for (int c = 0; c < 2; ++c)
            tma_load_2d(dst + c * 8192u, m, fb, head * kHeadDim + c * 64,
                        kt * kKeys + 64 * (int)rank, pol_kv);
        } else {
          // V half: dims 64 rank .. + 63 of all 128 keys, two boxes of 64 keys
          for (int r2 = 0; r2 < 2; ++r2)
            tma_load_2d(dst + r2 * 8192u, m, fb, head * kHeadDim + 64 * (int)rank,
                        kt * kKeys + 64 * r2, pol_kv);
        }
        ++t;
        return true;
      };
      TileWalk<false> wk(p, nullptr, 0, g0, g1), wv(p, nullptr, 0, g0, g1);
      int s, kt;
      bool bad = false, ok = true;
      for (int i = 0; i < 3 && ok; ++i)
        if (wk.next(&s, &kt, &bad)) ok = load_item(0, s, kt);
      while (ok && wv.next(&s, &kt, &bad)) {
        ok = load_item(1, s, kt);
        if (ok && wk.next(&s, &kt, &bad)) ok = load_item(0, s, kt);
      }
      // Teardown: every load this lane issued has landed.
      drain_phase(bar(own_q), 0, p.wait_limit_ns);
      for (int v = max(t - kStages, 0); v < t; ++v)
        if (v != p.testing_skip_load)
          drain_phase(bar(own_kv + v % kStages), (uint32_t)(v / kStages) & 1u, p.wait_limit_ns);
    }
    __syncwarp();
  };
  auto role_mma = [&]() {
    if (lane != 0) {
      // lanes 1-31 have no work
    } else if (kPair && !leader) {
      // ---------------------------------------------------- forwarder (odd CTA)
      // Passes the completion of each of this CTA's loads to the even CTA,
      // whose MMA lane reads both halves.
      if (n_kv > 0) {
        if (wait_phase(bar(own_q), 0, ctl)) {
          mbar_arrive_remote(mapa_rank(bar(C::kBarQFull), 0));
          for (int t = 0; t < n_items; ++t) {
            if (t == p.testing_skip_load) continue;
            const int slot = t % kStages;
            if (!wait_phase(bar(own_kv + slot), (uint32_t)(t / kStages) & 1u, ctl)) break;
            mbar_arrive_remote(mapa_rank(bar(C::kBarKVFull + slot), 0));
          }
        }
      }
    } else if (n_kv > 0) {
      // ------------------------------------------------------------------ MMA
      constexpr uint32_t kIdescQK = pair_idesc(kPair ? 256 : 128, 0);
      constexpr uint32_t kIdescPV = pair_idesc(kPair ? 256 : 128, 1);
      // K-major Q and K; MN-major V (16-key groups 2 KiB apart; single CTA:
      // the two 64-dim halves of V 16 KiB apart).
      constexpr uint32_t kKHalf = kPair ? 8192u : 16384u;  // K: dims 64-127 after dims 0-63
      const uint64_t dq = sw128_desc(sQ, 16, 1024);
      const uint64_t dk = sw128_desc(sKV, 16, 1024);
      const uint64_t dv = sw128_desc(sKV, 16384, 1024);
      const uint32_t tO = tmem_base + kTmemO;
      auto item_ready = [&](int t) -> bool {
        const int slot = t % kStages;
        const uint32_t ph = (uint32_t)(t / kStages) & 1u;
        if (!wait_phase(bar(own_kv + slot), ph, ctl)) return false;
        if constexpr (kPair)
          if (!wait_ph<true>(bar(C::kBarKVFull + slot), ph, ctl)) return false;
        tc_fence_after();
        return true;
      };
      // S_b = Q K^T over D = 128: 8 MMAs of K = 16.
      auto issue_qk = [&](int b, int t) {
        const uint64_t kd = desc_plus(dk, (uint32_t)(t % kStages) * kItem);
        const uint32_t d = tmem_base + 128u * (uint32_t)b;
        mma_ss2<kPair, 0>(d, dq, kd, kIdescQK);
#pragma unroll
        for (int k = 1; k < 8; ++k)
          mma_ss2<kPair, 1>(d, desc_plus(dq, (uint32_t)(k >> 2) * kQHalf + (uint32_t)(k & 3) * 32u),
                            desc_plus(kd, (uint32_t)(k >> 2) * kKHalf + (uint32_t)(k & 3) * 32u),
                            kIdescQK);
      };
      int t = 0;
      do {
        if (!wait_phase(bar(own_q), 0, ctl)) break;
        if constexpr (kPair)
          if (!wait_ph<true>(bar(C::kBarQFull), 0, ctl)) break;
        bool ok = true;
        for (int i = 0; i < 3 && i < n_kv; ++i, ++t) {
          if (!item_ready(t)) {
            ok = false;
            break;
          }
          issue_qk(i, t);
          commit_all<kPair>(bar(C::kBarSFull + i));
          commit_all<kPair>(bar(C::kBarKVEmpty + t % kStages));
        }
        if (!ok) break;
        for (int j = 0; j < n_kv; ++j) {
          const int b = j % kSBufs;
          const uint32_t par = (uint32_t)(j / kSBufs) & 1u;
          const uint32_t tS = tmem_base + 128u * (uint32_t)b;
          if (!item_ready(t)) break;
          const uint64_t vd = desc_plus(dv, (uint32_t)(t % kStages) * kItem);
          // O += P_j V_j: keys 0-63 (P columns 0-31), then keys 64-127 (P
          // columns 64-95), 16 keys = 8 P columns = 2 KiB of V per MMA.
          if (!wait_ph<kPair>(bar(C::kBarP + 2 * b), par, ctl)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts2<kPair>(tO, tS + 8u * (uint32_t)k, desc_plus(vd, 2048u * (uint32_t)k), kIdescPV,
                           (j > 0 || k > 0) ? 1u : 0u);
          if (!wait_ph<kPair>(bar(C::kBarP + 2 * b + 1), par, ctl)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 4; k < 8; ++k)
            mma_ts2<kPair>(tO, tS + 64u + 8u * (uint32_t)(k - 4), desc_plus(vd, 2048u * (uint32_t)k),
                           kIdescPV, 1u);
          commit_all<kPair>(bar(C::kBarKVEmpty + t % kStages));
          commit_all<kPair>(bar(C::kBarOReady + b));
          ++t;
          if (j + kSBufs < n_kv) {
            if (!item_ready(t)) break;
            issue_qk(b, t);
            commit_all<kPair>(bar(C::kBarSFull + b));
            commit_all<kPair>(bar(C::kBarKVEmpty + t % kStages));
            ++t;
          }
        }
      } while (false);
      // Teardown: every MMA issued above completes before TMEM is freed.
      commit_local<kPair>(bar(C::kBarDrain));
      drain_phase(bar(C::kBarDrain), 0, p.wait_limit_ns);
    }
    __syncwarp();
  };
  auto role_softmax = [&]() {
    const int quarter = warp & 3;
    const int h = warp >> 2;  // 0: keys 0-63 of each tile, 1: keys 64-127
    const int row = quarter * 32 + lane;
    const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
    const uint32_t tOh = tmem_base + lane_bits + kTmemO + 64u * (uint32_t)h;
    float2 *xmax = reinterpret_cast<float2 *>(gbase + C::kOffXchMax);
    float2 *xl = reinterpret_cast<float2 *>(gbase + C::kOffXchL);
    const float sl2 = p.scale_log2;
    float m = -INFINITY;  // running max of scale*log2(e)*s, the same in both halves
    float l = 0.f;        // this half's running sum of P
    bool ok = true;
    int j = 0;
    TileWalk<false> walk(p, nullptr, 0, g0, g1);
    int s, kt;
    bool bad = false;
    uint32_t sr[64];
    float *sv = reinterpret_cast<float *>(sr);
    uint32_t pk[32];
    float lsum = 0.f, xp = -INFINITY;
    // P = 2^(s * scale * log2 e - m) of this half as bf16 pairs, its fp32
    // sum, and the largest argument given to the FMA-pipe exponential.
    auto form_p = [&]() {
      const uint64_t sl2x2 = f2(sl2, sl2), negm2 = f2(-m, -m);
      uint64_t a0 = f2(0.f, 0.f), a1 = f2(0.f, 0.f);
      xp = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const uint64_t x = fma2(f2(sv[2 * c], sv[2 * c + 1]), sl2x2, negm2);
        const float2 xv = unf2(x);
        uint64_t e;
        if (fma_pair(c)) {
          xp = fmax3(xp, xv.x, xv.y);
          e = exp2_poly_x2(x);
        } else {
          e = f2(ex2(xv.x), ex2(xv.y));
        }
        if (c & 1)
          a1 = add2(a1, e);
        else
          a0 = add2(a0, e);
        const float2 ev = unf2(e);
        pk[c] = pack_bf16x2(ev.x, ev.y);
      }
      const float2 u = unf2(a0), w = unf2(a1);
      lsum = (u.x + u.y) + (w.x + w.y);
    };
    // S_j comes out of TMEM one tile ahead: the load of S_{j+1} is issued
    // before waiting for the stores of P_j to drain.
    auto load_s = [&](int jj) -> bool {
      const int b = jj % kSBufs;
      const bool got =
          __all_sync(0xffffffffu, wait_phase(bar(C::kBarSFull + b), (uint32_t)(jj / kSBufs) & 1u, ctl));
      tc_fence_after();
      const uint32_t tS = tmem_base + lane_bits + 128u * (uint32_t)b + 64u * (uint32_t)h;
      tmem::ld32(tS, sr);
      tmem::ld32(tS + 32, sr + 32);
      return got;
    };
    bool have = walk.next(&s, &kt, &bad);
    bool got = have ? load_s(0) : true;
    if (have) tmem::wait_ld64(sr);
    while (ok && have) {
      const int b = j % kSBufs;
      const uint32_t tS = tmem_base + lane_bits + 128u * (uint32_t)b + 64u * (uint32_t)h;
      const int64_t rem = p.span_len[s] - (int64_t)kt * kKeys - 64 * h;
      if (rem < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= rem) sv[c] = -INFINITY;
      }
      // Stale max: after the first tile P is formed against m without this
      // tile's max.  It stands if every P of the row is at most 2^16: the
      // fp32 half sums are at most 2^16 (an overflow to +inf fails this
      // too), and the FMA-pipe exponential, valid for arguments below 128,
      // saw none above 16.  Otherwise the two halves take the exact max.
      bool need = j == 0 || !got;
      if (j > 0) {
        form_p();
        need = need || !(lsum <= 65536.f) || xp > 16.f;
      }
      if (rows_any(quarter, need)) {
        bool g = got;
        // O must be quiescent before it is rescaled: the last O += P V done.
        if (j > 0) {
          const int jb = (j - 1) % kSBufs;
          g = g && __all_sync(0xffffffffu, wait_phase(bar(C::kBarOReady + jb),
                                                      (uint32_t)((j - 1) / kSBufs) & 1u, ctl));
          tc_fence_after();
        }
        float mh = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; c += 2) mh = fmax3(mh, sv[c], sv[c + 1]);
        mh *= sl2;
        xmax[h * kRows + row] = make_float2(mh, g ? 1.f : 0.f);
        rows_sync(quarter);
        const float2 other = xmax[(1 - h) * kRows + row];
        // The same decision in both warps of the row pair.
        if (!(g && other.y != 0.f)) {
          ok = false;
          break;
        }
        const float m_new = fmaxf(m, fmaxf(mh, other.x));
        if (j > 0) {
          const float alpha = ex2(m - m_new);
          l *= alpha;
#pragma unroll
          for (int cc = 0; cc < 64; cc += 32) {
            uint32_t orow[32];
            tmem::ld32(tOh + cc, orow);
            tmem::wait_ld32(orow);
#pragma unroll
            for (int c = 0; c < 32; ++c) orow[c] = __float_as_uint(__uint_as_float(orow[c]) * alpha);
            tmem::st32(tOh + cc, orow);
          }
        }
        m = m_new;
        form_p();
      }
      // P of this half over the first 32 columns of its S columns; the MMA
      // lane starts O += P V on a half once its 4 (pair: 8) warps arrived.
      tmem::st32(tS, pk);
      l += lsum;
      have = walk.next(&s, &kt, &bad);
      if (have) got = load_s(j + 1);
      tmem::wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair)
          mbar_arrive_remote(mapa_rank(bar(C::kBarP + 2 * b + h), 0));
        else
          mbar_arrive(bar(C::kBarP + 2 * b + h));
      }
      if (have) tmem::wait_ld64(sr);
      ++j;
    }
    // Epilogue.  Both halves of a row agree on whether O is complete (the
    // last O += P V done in both), and share their row sums.
    bool g = ok && n_kv > 0;
    if (g)
      g = __all_sync(0xffffffffu, wait_phase(bar(C::kBarOReady + (n_kv - 1) % kSBufs),
                                             (uint32_t)((n_kv - 1) / kSBufs) & 1u, ctl));
    xl[h * kRows + row] = make_float2(l, g ? 1.f : 0.f);
    rows_sync(quarter);
    const float2 other = xl[(1 - h) * kRows + row];
    const bool have_o = g && other.y != 0.f;
    const float l_row = l + other.x;  // the same sum in both halves
    // Outputs: O / l -> bf16 and LSE = ln(2) * (m + log2 l), into part
    // blockIdx.z of the outputs when the keys are split, or into part
    // owner_slot of the buffers of the row's owner when the outputs are
    // routed (plain stores, possibly to another GPU's memory over NVLink).
    const int64_t my_row = (int64_t)q_row0 + row;
    uint16_t *o_base = p.o;
    float *lse_base = p.lse;
    int64_t part = blockIdx.z;
    if (p.n_owners > 0) {
      int so = 0;
      while (so + 1 < p.n_owners && my_row >= p.owner_row0[so + 1]) ++so;
      o_base = p.owner_o[so];
      lse_base = p.owner_lse[so];
      part = p.owner_slot;
    }
    const int64_t row_elems = (int64_t)p.heads * kHeadDim;
    uint16_t *const o_out = o_base + part * p.n_q * row_elems;
    float *const lse_out = lse_base == nullptr ? nullptr : lse_base + part * p.heads * p.n_q;
    uint4 *const dst =
        reinterpret_cast<uint4 *>(o_out + my_row * row_elems + head * kHeadDim + 64 * h);
    if (have_o) {
      tc_fence_after();
      const float inv_l = 1.0f / l_row;
#pragma unroll
      for (int cc = 0; cc < 64; cc += 32) {
        uint32_t orow[32];
        tmem::ld32(tOh + cc, orow);
        tmem::wait_ld32(orow);
        if (my_row < p.n_q) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            const uint32_t *o8 = orow + 8 * v;
            w.x = pack_bf16x2(__uint_as_float(o8[0]) * inv_l, __uint_as_float(o8[1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o8[2]) * inv_l, __uint_as_float(o8[3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o8[4]) * inv_l, __uint_as_float(o8[5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o8[6]) * inv_l, __uint_as_float(o8[7]) * inv_l);
            dst[cc / 8 + v] = w;
          }
        }
      }
      if (h == 0 && lse_out != nullptr && my_row < p.n_q)
        lse_out[(int64_t)head * p.n_q + my_row] = (m + log2f(l_row)) * 0.69314718055994531f;
    } else if (my_row < p.n_q) {
      // No key tile for this block (a key split with an empty share): O = 0,
      // LSE = -inf.  A block that aborted (a wait ran out) marks its rows NaN
      // so that nothing downstream takes stale buffer contents for them.
      const bool empty = ok && n_kv == 0;
      const uint32_t fill = empty ? 0u : 0x7FC07FC0u;  // bf16 0 or quiet NaN pairs
#pragma unroll
      for (int v = 0; v < 8; ++v) dst[v] = make_uint4(fill, fill, fill, fill);
      if (h == 0 && lse_out != nullptr)
        lse_out[(int64_t)head * p.n_q + my_row] = empty ? -INFINITY : NAN;
    }
  };

  if (warp == kProducerWarp)
    role_producer();
  else if (warp == kMmaWarp)
    role_mma();
  else
    role_softmax();

  tc_fence_before();
  __syncthreads();
  // Pair form: the even CTA's MMAs (drained above) read this CTA's shared
  // memory and write its TMEM, and the odd CTA's arrivals land in the even
  // CTA's barriers: neither frees anything before both are here.
  if constexpr (kPair) cluster_sync_all();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_free_all<kPair>(tmem_base);
  }
}

}  // namespace

bool attention_pair_supported(const AttnArgs &a) {
  return a.i8 == 0 && a.tile_list == nullptr;
}

cudaError_t launch_attention_pair(const AttnArgs &a, bool pair, cudaStream_t stream) {
  // Per-device, idempotent shared-memory opt-in (see launch_attention).
  static std::atomic<int> attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (attr_set[dev].load(std::memory_order_acquire) == 0) {
    e = cudaFuncSetAttribute(attention_pair_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, PCfg<false>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attention_pair_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, PCfg<true>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(1, std::memory_order_release);
  }
  if (!attention_pair_supported(a) || a.heads < 1 || a.heads > kHeads) return cudaErrorInvalidValue;
  if (a.kv_splits < 1 || a.kv_splits > NOMAS_MAX_MERGE_PARTS || (a.kv_splits > 1 && a.lse == nullptr))
    return cudaErrorInvalidValue;
  const int64_t units = ((int64_t)a.n_q + 2 * kRows - 1) / (2 * kRows);  // 256-row units
  if (units <= 0) return cudaSuccess;
  if (units > 0x3fffffff) return cudaErrorInvalidValue;
  if (!pair) {
    const int64_t blocks = ((int64_t)a.n_q + kRows - 1) / kRows;
    dim3 grid((unsigned)blocks, (unsigned)a.heads, (unsigned)a.kv_splits);
    attention_pair_kernel<false><<<grid, kThreads, PCfg<false>::kSmemAlloc, stream>>>(a);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(2 * units), (unsigned)a.heads, (unsigned)a.kv_splits);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PCfg<true>::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, attention_pair_kernel<true>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace nomas
