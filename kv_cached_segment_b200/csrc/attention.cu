// Segment-over-cache attention for sm_100a: TMA -> shared memory ->
// tcgen05.mma with TMEM accumulators, fp32 online softmax, no mask.
//
// "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
// (ai.thesatyajit.com), section "How one segment is made" (joint attention of
// text and video tokens, 16 heads of 128, causal across segments: the current
// segment reads earlier ones from the KV cache and sees itself and the text
// in full) and section "What 'world memory' stores" (the queries of segment k
// attend over the cached keys and values).
//
// Work unit: one CTA = one head x 256 query rows, as two 128-row Q tiles that
// share every K/V tile.  Keys stream through a ring of 32-KiB shared-memory
// slots, K and V tiles alternating, 128 keys per tile, across up to four
// spans (cache or window, text, segment), each with its own tensor map; TMA
// zero-fills rows past a span's end and the softmax masks them.
//
// Warp roles (320 threads):
//   warps 0-3  softmax for Q tile 0 (TMEM lanes 0-127, one query row per thread)
//   warps 4-7  softmax for Q tile 1
//   warp 8     TMA producer (one elected lane)
//   warp 9     MMA issuer (one elected lane); owns the TMEM allocation
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512);
// P_i (bf16, 64 columns) overwrites the first half of S_i once the softmax has
// read S_i into registers, and is the TMEM A operand of O_i += P_i V.
//
// Issue order of the MMA lane, per K/V tile j:
//   O0 += P0(j) V_j ; S0 = Q0 K_{j+1}^T ; O1 += P1(j) V_j ; S1 = Q1 K_{j+1}^T
// so each softmax group works on one tile while the tensor core runs the
// other tile's two GEMMs.  P is published in two halves of 64 keys, so the
// first half of O += P V runs while the softmax computes the second half.
// tcgen05 operations of one thread complete in issue order, so the commit
// that announces S_i(j+1) also covers O_i += P_i(j) V_j: when a softmax
// thread sees S_i ready, O_i is quiescent and the thread may rescale it in
// place.  The running max is allowed to be stale: P is formed against it
// (values up to 2^16) and the final division by the row sum, formed with the
// same max, makes the result exact; it is raised, with O and the row sum
// rescaled, only when a bound check shows that some P of the tile would
// exceed 2^16.
//
// Every wait is bounded (a globaltimer limit); on expiry the kernel records
// NOMAS_DEVERR_WAIT_TIMEOUT, drains its own TMA loads and MMAs, sets the
// block's rows of O and LSE to NaN, frees TMEM and returns.
//
// INT8-history variant ("The 4090 preset": the resident frames stay on the
// GPU in INT8; "Hy-Nomas en una RTX 4090", section "El preset de una GPU":
// stored in INT8, computed in BF16): the first span holds INT8 codes and
// per-(token, head) fp32 scales.  512 threads: warps 12-15 are a converter
// warpgroup (warps 10-11 idle).  The producer TMA-loads each INT8 tile's
// codes into one of two 16-KiB staging slots; converter thread r writes key
// row r as bf16(code * scale) into the ring slot, in the layout a TMA load of
// a bf16 tile gives, and one thread then arrives on the slot's full barrier,
// so the MMA lane and the softmax run unchanged.  The ring has 4 slots here,
// and setmaxnreg moves registers from the producer/MMA and converter
// warpgroups to the softmax warpgroups.
#include <atomic>

#include <cuda_bf16.h>

#include "nomas_internal.h"
#include "f32x2.cuh"
#include "attn_device.cuh"
#include "tmem_ops.cuh"

namespace nomas {
namespace {

constexpr int kBM = 128;              // query rows per Q tile (MMA M)
constexpr int kBN = 128;              // keys per K/V tile (MMA N of QK^T)
constexpr int kQTiles = 2;
#ifndef NOMAS_ATTN_STAGES
#define NOMAS_ATTN_STAGES 5
#endif
constexpr uint32_t kTileBytes = kBN * kHeadDim * 2;   // 32 KiB
constexpr uint32_t kHalfBytes = kTileBytes / 2;       // 64 dims x 128 rows
constexpr uint32_t kCodeTileBytes = kBN * kHeadDim;   // 16 KiB of INT8 codes
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvWarp0 = 12;        // INT8 variant: warps 12-15 dequantise
constexpr uint32_t kTmemCols = 512;

// Shared-memory map (offsets from a 1024-B aligned base) and thread count of
// the two variants: bf16 spans only (10 warps, 5 ring slots), or a first span
// held as INT8 codes + scales (16 warps: a converter warpgroup is added; 4
// ring slots, 2 staging slots for code tiles).
template <bool kI8>
struct Cfg {
  static constexpr int kStages = kI8 ? 4 : NOMAS_ATTN_STAGES;  // K/V ring slots
  static constexpr int kThreads = kI8 ? 512 : 320;
  static constexpr int kStaging = kI8 ? 2 : 0;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = kOffQ + kQTiles * kTileBytes;
  static constexpr uint32_t kOffStage = kOffKV + kStages * kTileBytes;
  static constexpr uint32_t kOffBar = kOffStage + kStaging * kCodeTileBytes;
  // barrier indices (8 B each)
  static constexpr int kBarQFull = 0;
  static constexpr int kBarKVFull = 1;                      // + slot
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;  // + slot
  static constexpr int kBarSFull = kBarKVEmpty + kStages;   // + tile
  static constexpr int kBarPFull = kBarSFull + 2;           // + tile
  static constexpr int kBarPHalf = kBarPFull + 2;           // + tile: first 64 keys of P
  static constexpr int kBarOFull = kBarPHalf + 2;           // + tile
  static constexpr int kBarDrain = kBarOFull + 2;
  static constexpr int kBarStFull = kBarDrain + 1;          // + staging slot
  static constexpr int kBarStEmpty = kBarStFull + kStaging; // + staging slot
  static constexpr int kNumBars = kBarStEmpty + kStaging;
  static constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
  static constexpr uint32_t kSmemUsed = kOffAbort + 4;
  static constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;  // room to align the base
};
static_assert(Cfg<true>::kSmemAlloc <= 232448 && Cfg<false>::kSmemAlloc <= 232448,
              "shared memory per block");

// Register split of the INT8 variant (setmaxnreg, per warpgroup): the block
// is launched with 512 threads x 128 registers = 65,536; the two softmax
// warpgroups raise theirs to 168 and the producer/MMA and converter
// warpgroups lower theirs to 88: 2 x 128 x 168 + 2 x 128 x 88 = 65,536.
constexpr int kI8LaunchRegs = 128;
constexpr int kI8SoftmaxRegs = 168;
constexpr int kI8OtherRegs = 88;
static_assert(2 * 128 * kI8SoftmaxRegs + 2 * 128 * kI8OtherRegs <= 512 * kI8LaunchRegs,
              "register split exceeds the block's launch allocation");

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D,
// M = 128, N = 128; A K-major; B K-major (QK^T: K rows are key-major with
// dims contiguous) or MN-major (PV: V rows have dims, i.e. N, contiguous).
constexpr uint32_t make_idesc(uint32_t b_mn_major) {
  return (1u << 4)            // D format f32
       | (1u << 7)            // A format bf16
       | (1u << 10)           // B format bf16
       | (b_mn_major << 16)   // B major
       | ((128u >> 3) << 17)  // N
       | ((128u >> 4) << 24); // M
}
constexpr uint32_t kIdescQK = make_idesc(0);
constexpr uint32_t kIdescPV = make_idesc(1);

// One tcgen05.mma kind::f16 with both operands in shared memory (SS) or A in
// tensor memory (TS).  ACC = 0 overwrites D, 1 accumulates into it; the
// predicate comes from an immediate so the issue costs one instruction.
template <int ACC>
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "n"(ACC)
      : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}


// Pairs of P (out of every 8) whose exponentials run on the FMA pipe.
#ifndef NOMAS_EXP2_FMA_PAIRS
#define NOMAS_EXP2_FMA_PAIRS 1
#endif
#ifndef NOMAS_EXP2_FMA_PAIRS_H1
#define NOMAS_EXP2_FMA_PAIRS_H1 NOMAS_EXP2_FMA_PAIRS
#endif
// c < 32: first half of the tile (on the critical path to the MMA lane).
__device__ __forceinline__ constexpr bool pair_on_fma(int c) {
  return c < 32 ? (c & 7) < NOMAS_EXP2_FMA_PAIRS : (c & 7) < NOMAS_EXP2_FMA_PAIRS_H1;
}


// S = Q_i K^T over D = 128: 8 MMAs of K = 16.  Both operands K-major, 128-B
// swizzled, two 16-KiB halves (dims 0-63, 64-127); a K step of 16 elements
// advances the start address by 32 B inside a swizzle atom.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
  mma_ss<0>(d_tmem, q_desc, k_desc, kIdescQK);
#pragma unroll
  for (int k = 1; k < 8; ++k) {
    const uint32_t off = (uint32_t)(k >> 2) * kHalfBytes + (uint32_t)(k & 3) * 32u;
    mma_ss<1>(d_tmem, desc_plus(q_desc, off), desc_plus(k_desc, off), kIdescQK);
  }
}

// O_i (+)= P_i V over 64 of the 128 keys of a tile (half 0: keys 0-63, half
// 1: keys 64-127): 4 MMAs of K = 16 keys.  P comes from TMEM (8 columns of
// packed bf16 pairs per step); V is MN-major: 8-key groups are 1024 B apart
// (SBO), the two 64-dim halves 16 KiB apart (LBO); a K step of 16 keys
// advances the start address by 2 KiB.
template <int HALF>
__device__ __forceinline__ void issue_pv_half(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc,
                                              uint32_t accumulate) {
#pragma unroll
  for (int k = 4 * HALF; k < 4 * HALF + 4; ++k)
    mma_ts(d_tmem, p_tmem + (uint32_t)k * 8u, desc_plus(v_desc, (uint32_t)k * 2048u), kIdescPV,
           (k > 0) ? 1u : accumulate);
}

// ------------------------------------------------- INT8 tile dequantisation --
__device__ __forceinline__ void lds128(uint32_t addr, uint32_t (&w)[4]) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
               : "r"(addr));
}
__device__ __forceinline__ void sts128(uint32_t addr, const uint32_t *w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3])
               : "memory");
}
// Makes this thread's shared-memory stores visible to the tensor core (the
// async proxy), before the barrier that hands the tile over.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// The converter warpgroup's own named barrier (id 1, 128 threads); the
// reduction form returns the AND of every thread's flag, so that all of them
// take the same branch after a bounded wait.
__device__ __forceinline__ bool converters_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void converters_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Dequantises one key row of an INT8 code tile into a bf16 ring slot:
// 128 codes become bf16(code * scale) (product rounded to float32, then to
// bf16 nearest-even), written in the layout TMA gives a bf16 tile: two
// 64-dim halves of 128 rows x 128 B, the 16-byte chunk j of row r at
// position j ^ (r & 7) (128-byte swizzle).  The code tile arrived with the
// same swizzle on its single 128-byte row, so neither side has bank
// conflicts.  A code becomes a float exactly: biased by 128 it is the low
// mantissa byte of 2^23 (one byte permute), and subtracting 2^23 + 128 is
// exact.
__device__ __forceinline__ void convert_row(uint32_t src_row, uint32_t dst_row, uint32_t sw,
                                            float scale) {
  const uint64_t sc2 = f2(scale, scale);
  const uint64_t off2 = f2(-8388736.f, -8388736.f);  // -(2^23 + 128)
  // All eight 16-byte loads of the row first: the shared-memory stores below
  // would otherwise order each load after the previous chunk's stores and
  // expose the load latency eight times.
  uint32_t wq[8][4];
#pragma unroll
  for (int q = 0; q < 8; ++q) lds128(src_row + (((uint32_t)q ^ sw) << 4), wq[q]);
#pragma unroll
  for (int q = 0; q < 8; ++q) {  // 16 codes: dims 16q .. 16q + 15
    const uint32_t(&w)[4] = wq[q];
    uint32_t out[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t b = w[i] ^ 0x80808080u;
      const float c0 = __uint_as_float(__byte_perm(b, 0x4B000000u, 0x7540));
      const float c1 = __uint_as_float(__byte_perm(b, 0x4B000000u, 0x7541));
      const float c2 = __uint_as_float(__byte_perm(b, 0x4B000000u, 0x7542));
      const float c3 = __uint_as_float(__byte_perm(b, 0x4B000000u, 0x7543));
      const float2 v01 = unf2(mul2(add2(f2(c0, c1), off2), sc2));
      const float2 v23 = unf2(mul2(add2(f2(c2, c3), off2), sc2));
      out[2 * i] = pack_bf16x2(v01.x, v01.y);
      out[2 * i + 1] = pack_bf16x2(v23.x, v23.y);
    }
    const uint32_t c0 = 2u * q, c1 = 2u * q + 1u;  // 8-dim chunks of the output row
    sts128(dst_row + (c0 >> 3) * kHalfBytes + (((c0 & 7u) ^ sw) << 4), out);
    sts128(dst_row + (c1 >> 3) * kHalfBytes + (((c1 & 7u) ^ sw) << 4), out + 4);
  }
}


template <bool kSparse, bool kI8>
__global__ void __launch_bounds__(Cfg<kI8>::kThreads, 1)
attention_kernel(const __grid_constant__ AttnArgs p) {
  using C = Cfg<kI8>;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kOffQ = C::kOffQ, kOffKV = C::kOffKV, kOffStage = C::kOffStage,
                     kOffBar = C::kOffBar, kOffTmemSlot = C::kOffTmemSlot, kOffAbort = C::kOffAbort;
  constexpr int kBarQFull = C::kBarQFull, kBarKVFull = C::kBarKVFull,
                kBarKVEmpty = C::kBarKVEmpty, kBarSFull = C::kBarSFull, kBarPFull = C::kBarPFull,
                kBarPHalf = C::kBarPHalf, kBarOFull = C::kBarOFull, kBarDrain = C::kBarDrain,
                kBarStFull = C::kBarStFull, kBarStEmpty = C::kBarStEmpty;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *const gbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int q_row0 = blockIdx.x * (kQTiles * kBM);

  const uint32_t sQ = base + kOffQ;
  const uint32_t sKV = base + kOffKV;
  const uint32_t sStage = base + kOffStage;  // INT8 variant: code tiles from TMA
  auto bar = [&](int i) { return base + kOffBar + (uint32_t)i * 8u; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + kOffTmemSlot);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + kOffAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQFull), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKVFull + s), 1);
      mbar_init(bar(kBarKVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(kBarSFull + t), 1);
      mbar_init(bar(kBarPFull + t), 128);
      mbar_init(bar(kBarPHalf + t), 128);
      mbar_init(bar(kBarOFull + t), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    for (int st = 0; st < C::kStaging; ++st) {
      mbar_init(bar(kBarStFull + st), 1);
      mbar_init(bar(kBarStEmpty + st), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const WaitCtl ctl{abort_flag, p.dev_err, p.wait_limit_ns};
  // This block's key tiles: the whole key sequence, or its sparse list.
  const int32_t *list = nullptr;
  int n_list = 0;
  // Dense: this block's share [g0, g1) of the key tiles (all of them unless
  // the keys are split across the grid's third dimension).
  const int total_tiles = p.tile_base[p.n_spans];
  const int g0 = (int)((int64_t)total_tiles * blockIdx.z / p.kv_splits);
  const int g1 = (int)((int64_t)total_tiles * (blockIdx.z + 1) / p.kv_splits);
  int n_kv = g1 - g0;  // K/V tiles this block streams
  if constexpr (kSparse) {
    const int64_t row = (int64_t)blockIdx.x * p.heads + head;
    list = p.tile_list + row * p.max_tiles;
    n_list = min(max(p.tile_count[row], 0), p.max_tiles);
    n_kv = 0;
    TileWalk<true> w(p, list, n_list, 0, 0);
    int s_, kt_;
    bool bad_ = false;
    while (w.next(&s_, &kt_, &bad_)) ++n_kv;
  }

  auto role_producer = [&]() {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      mbar_expect_tx(bar(kBarQFull), kQTiles * kTileBytes);
      for (int i = 0; i < kQTiles; ++i)
        for (int c = 0; c < 2; ++c)
          tma_load_2d(sQ + i * kTileBytes + c * kHalfBytes, &p.tmap_q, bar(kBarQFull),
                      head * kHeadDim + c * 64, q_row0 + i * kBM, pol_q);
      int t = 0;
      // INT8 variant: code tiles issued to the staging slots, the one left
      // out by the testing hook, and the end of the ring indices that the
      // converters fill (the INT8 span comes first).
      int u = 0, u_skip = -1, t_i8_end = 0;
      bool ok = true;
      TileWalk<kSparse> walk(p, list, n_list, g0, g1);
      int s, kt;
      bool bad = false;
      while (ok && walk.next(&s, &kt, &bad)) {
        {
          for (int which = 0; which < 2; ++which, ++t) {
            if (kI8 && s == 0) {
              // INT8 tile: its codes go to a staging slot; the converter
              // warpgroup fills ring slot t from there.
              const int st = u & 1;
              const uint32_t sph = (uint32_t)(u >> 1) & 1u;
              t_i8_end = t + 1;
              if (t == p.testing_skip_load) {
                u_skip = u++;
                continue;
              }
              if (!wait_phase(bar(kBarStEmpty + st), sph ^ 1u, ctl)) {
                ok = false;
                break;
              }
              mbar_expect_tx(bar(kBarStFull + st), kCodeTileBytes);
              tma_load_2d(sStage + st * kCodeTileBytes, which == 0 ? &p.tmap_k[0] : &p.tmap_v[0],
                          bar(kBarStFull + st), head * kHeadDim, kt * kBN, pol_kv);
              ++u;
              continue;
            }
            // Testing hook: leave one load out so that a consumer wait runs
            // out of time (exercises the bounded-wait abort path).
            if (t == p.testing_skip_load) continue;
            const int slot = t % kStages;
            const uint32_t ph = (uint32_t)(t / kStages) & 1u;
            if (!wait_phase(bar(kBarKVEmpty + slot), ph ^ 1u, ctl)) {
              ok = false;
              break;
            }
            mbar_expect_tx(bar(kBarKVFull + slot), kTileBytes);
            const CUtensorMap *m = which == 0 ? &p.tmap_k[s] : &p.tmap_v[s];
            for (int c = 0; c < 2; ++c)
              tma_load_2d(sKV + slot * kTileBytes + c * kHalfBytes, m, bar(kBarKVFull + slot),
                          head * kHeadDim + c * 64, kt * kBN, pol_kv);
          }
        }
      }
      if (bad && p.dev_err != nullptr) atomicOr(p.dev_err, NOMAS_DEVERR_BAD_TILE_INDEX);
      // Teardown: wait until every load this lane issued has landed (ring
      // slots the converters fill are theirs, not this lane's).
      drain_phase(bar(kBarQFull), 0, p.wait_limit_ns);
      for (int v = max(t - kStages, t_i8_end); v < t; ++v)
        if (v != p.testing_skip_load)
          drain_phase(bar(kBarKVFull + v % kStages), (uint32_t)(v / kStages) & 1u, p.wait_limit_ns);
      for (int v = max(u - 2, 0); v < u; ++v)
        if (v != u_skip)
          drain_phase(bar(kBarStFull + (v & 1)), (uint32_t)(v >> 1) & 1u, p.wait_limit_ns);
    }
    __syncwarp();
  };
  auto role_mma = [&]() {
    // ------------------------------------------------------------------ MMA
    if (lane == 0 && n_kv > 0) {
      const uint32_t tS[2] = {tmem_base + 0u, tmem_base + 128u};
      const uint32_t tO[2] = {tmem_base + 256u, tmem_base + 384u};
      auto slot_of = [](int t) { return t % kStages; };
      auto ph_of = [](int t) { return (uint32_t)(t / kStages) & 1u; };
      const uint64_t dq0 = sw128_desc(sQ, 16, 1024);
      const uint64_t dq1 = desc_plus(dq0, kTileBytes);
      const uint64_t dk = sw128_desc(sKV, 16, 1024);           // slot 0, K-major
      const uint64_t dv = sw128_desc(sKV, kHalfBytes, 1024);   // slot 0, MN-major
      do {
        if (!wait_phase(bar(kBarQFull), 0, ctl)) break;
        if (!wait_phase(bar(kBarKVFull + slot_of(0)), ph_of(0), ctl)) break;
        tc_fence_after();
        issue_qk(tS[0], dq0, dk);
        mma_commit(bar(kBarSFull + 0));
        issue_qk(tS[1], dq1, dk);
        mma_commit(bar(kBarSFull + 1));
        mma_commit(bar(kBarKVEmpty + slot_of(0)));
        for (int j = 0; j < n_kv; ++j) {
          const int tv = 2 * j + 1, tk = 2 * j + 2;
          const uint64_t vd = desc_plus(dv, (uint32_t)slot_of(tv) * kTileBytes);
          const uint64_t kd = desc_plus(dk, (uint32_t)slot_of(tk) * kTileBytes);
          const uint32_t par = (uint32_t)j & 1u;
          const uint32_t acc = j > 0 ? 1u : 0u;
          const bool more = j + 1 < n_kv;
          if (!wait_phase(bar(kBarKVFull + slot_of(tv)), ph_of(tv), ctl)) break;
          // The next K tile is waited for here, off the path from the P
          // handoff to the next S (each wait costs ~100 cycles even when the
          // phase is complete).  Its slot was freed by items consumed before
          // this point, so the wait cannot hold up the ring.
          if (more && !wait_phase(bar(kBarKVFull + slot_of(tk)), ph_of(tk), ctl)) break;
          if (!wait_phase(bar(kBarPHalf + 0), par, ctl)) break;
          tc_fence_after();
          issue_pv_half<0>(tO[0], tS[0], vd, acc);
          if (!wait_phase(bar(kBarPFull + 0), par, ctl)) break;
          tc_fence_after();
          issue_pv_half<1>(tO[0], tS[0], vd, acc);
          if (more) {
            issue_qk(tS[0], dq0, kd);
            mma_commit(bar(kBarSFull + 0));
          } else {
            mma_commit(bar(kBarOFull + 0));
          }
          if (!wait_phase(bar(kBarPHalf + 1), par, ctl)) break;
          tc_fence_after();
          issue_pv_half<0>(tO[1], tS[1], vd, acc);
          if (!wait_phase(bar(kBarPFull + 1), par, ctl)) break;
          tc_fence_after();
          issue_pv_half<1>(tO[1], tS[1], vd, acc);
          mma_commit(bar(kBarKVEmpty + slot_of(tv)));
          if (more) {
            issue_qk(tS[1], dq1, kd);
            mma_commit(bar(kBarSFull + 1));
            mma_commit(bar(kBarKVEmpty + slot_of(tk)));
          } else {
            mma_commit(bar(kBarOFull + 1));
          }
        }
      } while (false);
      // Teardown: every MMA issued above completes before TMEM is freed.
      mma_commit(bar(kBarDrain));
      drain_phase(bar(kBarDrain), 0, p.wait_limit_ns);
    }
    __syncwarp();
  };
  auto role_convert = [&]() {
    // ---------------------------------------------------------- converters
    // INT8 variant only: warps 10-11 have no role; warps 12-15 (one per
    // sub-partition) dequantise the INT8 span's code tiles into the ring,
    // thread r handling key row r of every tile.
    if constexpr (kI8) {
      if (warp >= kConvWarp0) {
        const int r = (int)threadIdx.x - kConvWarp0 * 32;
        const uint32_t sw = (uint32_t)(r & 7);
        int t = 0, u = 0;
        bool ok = true;
        TileWalk<kSparse> walk(p, list, n_list, g0, g1);
        int s, kt;
        bool bad = false;
        while (ok && walk.next(&s, &kt, &bad)) {
          if (s != 0) break;  // the INT8 span comes first; the producer loads the rest
          const int64_t key = (int64_t)kt * kBN + r;
          const bool in_span = key < p.span_len[0];
          for (int which = 0; which < 2; ++which, ++t, ++u) {
            const float scale = in_span ? __ldg(p.i8_scale[which] + key * p.heads + head) : 0.f;
            const int st = u & 1;
            const int slot = t % kStages;
            const bool got =
                wait_phase(bar(kBarStFull + st), (uint32_t)(u >> 1) & 1u, ctl) &&
                wait_phase(bar(kBarKVEmpty + slot), ((uint32_t)(t / kStages) & 1u) ^ 1u, ctl);
            if (!converters_all(got)) {
              ok = false;
              break;
            }
            convert_row(sStage + st * kCodeTileBytes + r * 128, sKV + slot * kTileBytes + r * 128,
                        sw, scale);
            fence_proxy_async_smem();
            converters_sync();
            if (r == 0) {
              mbar_arrive(bar(kBarKVFull + slot));
              mbar_arrive(bar(kBarStEmpty + st));
            }
          }
        }
      }
    }
  };
  auto role_softmax = [&]() {
    // -------------------------------------------------------------- softmax
    const int tile = warp >> 2;
    const int quarter = warp & 3;
    const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem_base + lane_bits + (uint32_t)tile * 128u;
    const uint32_t tO = tmem_base + lane_bits + 256u + (uint32_t)tile * 128u;
    const float sl2 = p.scale_log2;
    float m = -INFINITY;  // running max of scale*log2(e)*s (possibly stale)
    float l = 0.f;        // running row sum of exp2(...)
    bool ok = true;
    int j = 0;
    TileWalk<kSparse> walk(p, list, n_list, g0, g1);
    int s, kt;
    bool bad = false;
    while (ok && walk.next(&s, &kt, &bad)) {
      const int64_t len = p.span_len[s];
      {
        // Warp-uniform outcome: the tcgen05 loads and stores below are
        // warp-collective, so a lane that saw the abort flag takes the whole
        // warp with it.
        if (!__all_sync(0xffffffffu, wait_phase(bar(kBarSFull + tile), (uint32_t)j & 1u, ctl))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // The whole S row (128 keys) comes out of TMEM in one go.
        uint32_t sr[128];
        tmem::ld32(tS + 0, sr + 0);
        tmem::ld32(tS + 32, sr + 32);
        tmem::ld32(tS + 64, sr + 64);
        tmem::ld32(tS + 96, sr + 96);
        tmem::wait_ld128(sr);
        float *sv = reinterpret_cast<float *>(sr);
        const int64_t rem = len - (int64_t)kt * kBN;
        const int valid = rem < kBN ? (int)rem : kBN;
        if (valid < kBN) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) sv[c] = -INFINITY;
        }
        auto row_max = [&](int c0, int c1) {
          float mA = -INFINITY, mB = -INFINITY, mC = -INFINITY, mD = -INFINITY;
#pragma unroll
          for (int c = c0; c < c1; c += 8) {
            mA = fmax3(mA, sv[c], sv[c + 1]);
            mB = fmax3(mB, sv[c + 2], sv[c + 3]);
            mC = fmax3(mC, sv[c + 4], sv[c + 5]);
            mD = fmax3(mD, sv[c + 6], sv[c + 7]);
          }
          return fmaxf(fmax3(mA, mB, mC), mD) * sl2;
        };
        bool rescale = false;
        float alpha = 1.f;
        if (j == 0) m = row_max(0, 128);
        // P = 2^(s * scale * log2 e - m) as bf16 pairs, published to the MMA
        // lane in two halves of 64 keys so that O += P V on the first half
        // overlaps the exponentials of the second.  The row sum accumulates
        // the fp32 values.
        uint64_t lacc0, lacc1;
        uint32_t pk0[32], pk1[32];
        float xp;  // max exponent fed to the FMA-pipe exp2 in half 0
        auto half0 = [&]() {
          const uint64_t sl2x2 = f2(sl2, sl2), negm2 = f2(-m, -m);
          lacc0 = f2(0.f, 0.f);
          lacc1 = f2(0.f, 0.f);
          xp = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const uint64_t x = fma2(f2(sv[2 * c], sv[2 * c + 1]), sl2x2, negm2);
            uint64_t e;
            if (pair_on_fma(c)) {
              const float2 xv = unf2(x);
              xp = fmax3(xp, xv.x, xv.y);
              e = exp2_poly_x2(x);
            } else {
              const float2 xv = unf2(x);
              e = f2(ex2(xv.x), ex2(xv.y));
            }
            if (c & 1)
              lacc1 = add2(lacc1, e);
            else
              lacc0 = add2(lacc0, e);
            const float2 ev = unf2(e);
            pk0[c] = pack_bf16x2(ev.x, ev.y);
          }
        };
        // Stale max: after the first tile, half 0 is exponentiated against
        // the running max m without first taking this tile's max.  The
        // result is exact for any m (the factor 2^-m cancels in O / l); m
        // only has to keep every P far from overflow.  Three bounds, each
        // P <= 2^16, are checked afterwards:
        //   - the fp32 sum of half 0 (the hardware exp2 returns +inf on
        //     overflow, which fails the test too);
        //   - the max of the half-0 columns whose exp2 runs on the FMA pipe,
        //     since that emulation is only valid for arguments below 128;
        //   - the max of half 1, before it is exponentiated.
        // If any row of the warp fails, the exact max is taken, O and l are
        // rescaled and half 0 is redone; S is still intact in TMEM then.
        half0();
        if (j > 0) {
          const float mx1 = row_max(64, 128);
          const float2 a0 = unf2(lacc0), a1 = unf2(lacc1);
          const float lh0 = (a0.x + a0.y) + (a1.x + a1.y);
          const bool bad = !(lh0 <= 65536.f) || xp > 16.f || mx1 > m + 16.f;
          if (__any_sync(0xffffffffu, bad)) {
            tmem::ld32(tS + 0, sr + 0);
            tmem::ld32(tS + 32, sr + 32);
            tmem::wait_ld64(sr);
            if (valid < 64) {
#pragma unroll
              for (int c = 0; c < 64; ++c)
                if (c >= valid) sv[c] = -INFINITY;
            }
            const float m_new = fmaxf(m, row_max(0, 128));
            alpha = ex2(m - m_new);
            m = m_new;
            l *= alpha;
            rescale = true;
            half0();
          }
        }
        // A pending O rescale happens before the first half is published
        // (the MMA lane may then start updating O).
        tmem::st32(tS + 0, pk0);
        if (rescale) {
#pragma unroll
          for (int cc = 0; cc < 128; cc += 32) {
            uint32_t orow[32];
            tmem::ld32(tO + cc, orow);
            tmem::wait_ld32(orow);
#pragma unroll
            for (int c = 0; c < 32; ++c)
              orow[c] = __float_as_uint(__uint_as_float(orow[c]) * alpha);
            tmem::st32(tO + cc, orow);
          }
        }
        tmem::wait_st();
        tc_fence_before();
        const uint64_t sl2x2 = f2(sl2, sl2), negm2 = f2(-m, -m);
        mbar_arrive(bar(kBarPHalf + tile));
#pragma unroll
        for (int c = 32; c < 64; ++c) {
          const uint64_t x = fma2(f2(sv[2 * c], sv[2 * c + 1]), sl2x2, negm2);
          uint64_t e;
          if (pair_on_fma(c)) {
            e = exp2_poly_x2(x);
          } else {
            const float2 xv = unf2(x);
            e = f2(ex2(xv.x), ex2(xv.y));
          }
          if (c & 1)
            lacc1 = add2(lacc1, e);
          else
            lacc0 = add2(lacc0, e);
          const float2 ev = unf2(e);
          pk1[c - 32] = pack_bf16x2(ev.x, ev.y);
        }
        tmem::st32(tS + 32, pk1);
        {
          const float2 a = unf2(lacc0), b = unf2(lacc1);
          l += (a.x + a.y) + (b.x + b.y);
        }
        tmem::wait_st();
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + tile));
        ++j;
      }
    }
    // Epilogue: O / l -> bf16, LSE = ln(2) * (m + log2 l), into part
    // blockIdx.z of the outputs when the keys are split, or into part
    // owner_slot of the buffers of the row's owner when the outputs are
    // routed (those may be other GPUs' memory: plain stores over NVLink).
    const int64_t my_row = (int64_t)q_row0 + tile * kBM + quarter * 32 + lane;
    uint16_t *o_base = p.o;
    float *lse_base = p.lse;
    int64_t part = blockIdx.z;
    if (p.n_owners > 0) {
      int s = 0;
      while (s + 1 < p.n_owners && my_row >= p.owner_row0[s + 1]) ++s;
      o_base = p.owner_o[s];
      lse_base = p.owner_lse[s];
      part = p.owner_slot;
    }
    const int64_t row_elems = (int64_t)p.heads * kHeadDim;
    uint16_t *const o_out = o_base + part * p.n_q * row_elems;
    float *const lse_out = lse_base == nullptr ? nullptr : lse_base + part * p.heads * p.n_q;
    bool have_o = ok && n_kv > 0;
    if (have_o) have_o = __all_sync(0xffffffffu, wait_phase(bar(kBarOFull + tile), 0, ctl));
    if (have_o) {
      tc_fence_after();
      const int64_t row = (int64_t)q_row0 + tile * kBM + quarter * 32 + lane;
      const float inv_l = 1.0f / l;
      uint16_t *orow_g = o_out + row * row_elems + head * kHeadDim;
#pragma unroll
      for (int cc = 0; cc < 128; cc += 32) {
        uint32_t orow[32];
        tmem::ld32(tO + cc, orow);
        tmem::wait_ld32(orow);
        if (row < p.n_q) {
          uint4 *dst = reinterpret_cast<uint4 *>(orow_g + cc);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(orow[8 * v + 0]) * inv_l, __uint_as_float(orow[8 * v + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(orow[8 * v + 2]) * inv_l, __uint_as_float(orow[8 * v + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(orow[8 * v + 4]) * inv_l, __uint_as_float(orow[8 * v + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(orow[8 * v + 6]) * inv_l, __uint_as_float(orow[8 * v + 7]) * inv_l);
            dst[v] = w;
          }
        }
      }
      if (lse_out != nullptr && row < p.n_q)
        lse_out[(int64_t)head * p.n_q + row] = (m + log2f(l)) * 0.69314718055994531f;
    } else {
      // No key selected for this block (a sparse list with no valid entry):
      // the empty sums give O = 0 and LSE = -inf.  A block that aborted (a
      // wait ran out) marks its rows NaN instead, so that nothing downstream
      // -- a merge of key-split or key-sharded partials in particular -- can
      // take earlier contents of the buffers for this block's result.
      const bool empty = ok && n_kv == 0;
      const uint32_t fill = empty ? 0u : 0x7FC07FC0u;  // bf16 0 or quiet NaN pairs
      const int64_t row = (int64_t)q_row0 + tile * kBM + quarter * 32 + lane;
      if (row < p.n_q) {
        uint4 *dst = reinterpret_cast<uint4 *>(o_out + row * row_elems + head * kHeadDim);
#pragma unroll
        for (int v = 0; v < 16; ++v) dst[v] = make_uint4(fill, fill, fill, fill);
        if (lse_out != nullptr) lse_out[(int64_t)head * p.n_q + row] = empty ? -INFINITY : NAN;
      }
    }
  };

  if constexpr (kI8) {
    // setmaxnreg is warpgroup-collective: the two softmax warpgroups (warps
    // 0-7) raise their registers at one instruction, the producer/MMA and
    // converter warpgroups (warps 8-15) lower theirs at another, before the
    // roles diverge.
    if (warp < 8) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kI8SoftmaxRegs) : "memory");
      role_softmax();
    } else {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kI8OtherRegs) : "memory");
      if (warp == kProducerWarp)
        role_producer();
      else if (warp == kMmaWarp)
        role_mma();
      else
        role_convert();
    }
  } else {
    if (warp == kProducerWarp)
      role_producer();
    else if (warp == kMmaWarp)
      role_mma();
    else
      role_softmax();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// Zero keys: O = 0, LSE = -inf.
__global__ void attention_empty_kernel(uint16_t *o, float *lse, int64_t n_q, int32_t heads) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n_vec = n_q * heads * (kHeadDim * 2 / 16);
  for (int64_t v = i; v < n_vec; v += (int64_t)gridDim.x * blockDim.x)
    reinterpret_cast<uint4 *>(o)[v] = make_uint4(0, 0, 0, 0);
  if (lse != nullptr)
    for (int64_t v = i; v < n_q * heads; v += (int64_t)gridDim.x * blockDim.x) lse[v] = -INFINITY;
}

}  // namespace

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t stream) {
  // The shared-memory opt-in is a per-device function attribute.  Several
  // host threads may make their first call on a device at once: the
  // attribute calls are idempotent, and the flag is atomic.  The INT8
  // variant's register split is only safe when the kernel was compiled to
  // exactly the launch allocation it assumes (otherwise a warpgroup's raise
  // could wait for registers that never come): checked here, before its
  // first launch on the device, and refused otherwise.
  static std::atomic<int> attr_state[64];  // 0 unset, 1 set, 2 set but INT8 refused
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int state = attr_state[dev].load(std::memory_order_acquire);
  if (state == 0) {
    e = cudaFuncSetAttribute(attention_kernel<false, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<false>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attention_kernel<true, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<false>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attention_kernel<false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<true>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, attention_kernel<false, true>);
    if (e != cudaSuccess) return e;
    state = (fa.numRegs == kI8LaunchRegs && fa.maxThreadsPerBlock >= Cfg<true>::kThreads) ? 1 : 2;
    attr_state[dev].store(state, std::memory_order_release);
  }
  const int64_t q_blocks = ((int64_t)a.n_q + kQTiles * kBM - 1) / (kQTiles * kBM);
  if (q_blocks <= 0) return cudaSuccess;
  if (q_blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (a.kv_splits < 1 || a.kv_splits > NOMAS_MAX_MERGE_PARTS ||
      (a.kv_splits > 1 && (a.tile_list != nullptr || a.lse == nullptr)))
    return cudaErrorInvalidValue;
  if (a.heads < 1 || a.heads > kHeads) return cudaErrorInvalidValue;
  dim3 grid((unsigned)q_blocks, (unsigned)a.heads, (unsigned)a.kv_splits);
  if (a.i8) {
    if (a.tile_list != nullptr) return cudaErrorInvalidValue;
    if (state != 1) return cudaErrorInvalidKernelImage;
    attention_kernel<false, true><<<grid, Cfg<true>::kThreads, Cfg<true>::kSmemAlloc, stream>>>(a);
  } else if (a.tile_list != nullptr) {
    attention_kernel<true, false><<<grid, Cfg<false>::kThreads, Cfg<false>::kSmemAlloc, stream>>>(a);
  } else {
    attention_kernel<false, false><<<grid, Cfg<false>::kThreads, Cfg<false>::kSmemAlloc, stream>>>(
        a);
  }
  return cudaGetLastError();
}

cudaError_t launch_attention_empty(uint16_t *o, float *lse, int64_t n_q, int32_t heads,
                                   cudaStream_t stream) {
  if (n_q <= 0) return cudaSuccess;
  attention_empty_kernel<<<1184, 256, 0, stream>>>(o, lse, n_q, heads);
  return cudaGetLastError();
}

}  // namespace nomas
