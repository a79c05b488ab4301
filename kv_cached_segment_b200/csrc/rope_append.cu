// Fused 3D RoPE + KV-cache append (memory-bound), into a bf16 cache or an
// INT8 cache (codes + per-(token, head) scales).
//
// "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
// (ai.thesatyajit.com): section "How one segment is made", item "The blocks"
// (3D RoPE over t/h/w with a per-axis split of the head dimension) and
// section "Writing the segment into memory" (the finished segment's keys and
// values are stored in the cache).
//
// One pass over the segment: Q rows are rotated into q_out, K rows are
// rotated straight into the cache at its write offset, V rows are copied into
// the cache bit for bit.  Every byte is read once and written once with
// 16-byte vector accesses: 24 KiB of traffic per video token (Q, K, V in;
// Q', K', V out).
//
// Thread mapping: a block of 256 threads covers 16 token rows; the 16 threads
// of a row each own one 16-byte column chunk (8 dims = 4 rotation pairs) and
// walk the 16 heads, so the 4 cos/sin pairs a thread needs are computed once
// per row and reused for 16 heads x (Q, K).  For a fixed head the 16 threads
// of a row touch 256 contiguous bytes.
#include <cuda_bf16.h>

#include "nomas_internal.h"
#include "f32x2.cuh"

namespace nomas {
namespace {

constexpr int kRowsPerBlock = 16;
constexpr int kThreads = kRowsPerBlock * 16;
constexpr int kHeadGroup = 4;  // heads loaded before the first store

__device__ __forceinline__ uint32_t rot_pair(uint32_t w, float c, float s) {
  // w holds the pair (x[2j] in the low half, x[2j+1] in the high half).
  const float a = __uint_as_float(w << 16);
  const float b = __uint_as_float(w & 0xffff0000u);
  const float ra = __fmaf_rn(a, c, -__fmul_rn(b, s));
  const float rb = __fmaf_rn(a, s, __fmul_rn(b, c));
  __nv_bfloat162 r = __floats2bfloat162_rn(ra, rb);
  return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint4 rot_chunk(uint4 v, const float (&c)[4], const float (&s)[4]) {
  v.x = rot_pair(v.x, c[0], s[0]);
  v.y = rot_pair(v.y, c[1], s[1]);
  v.z = rot_pair(v.z, c[2], s[2]);
  v.w = rot_pair(v.w, c[3], s[3]);
  return v;
}

// Symmetric INT8 quantisation per (token, head): with a = max |x| over the
// head's 128 values, the stored scale is a / 127 rounded to float32 and the
// code is the integer nearest to the exact quotient 127 x / a, ties to even;
// an all-zero head gets scale 0 and codes 0.
//
// A thread holds 8 values of each of 4 items (the keys, or the values, of 4
// heads) of its row.  The absmax of the 4 items over the row's 16 lanes is a
// transposed butterfly: at the first two xor steps a lane keeps half of its
// items and trades the other half with its partner, so 2 + 1 + 1 + 1
// shuffles leave lanes 4i..4i+3 holding item i reduced over the row.  Each
// lane then does the divisions for its own item only, and shuffles hand
// every lane the reciprocals of each item.
static_assert(kHeadGroup == 4, "the butterfly below reduces 4 items over 16 lanes");

__device__ __forceinline__ float chunk_absmax(uint4 v) {
  const float x0 = __uint_as_float(v.x << 16), x1 = __uint_as_float(v.x & 0xffff0000u);
  const float x2 = __uint_as_float(v.y << 16), x3 = __uint_as_float(v.y & 0xffff0000u);
  const float x4 = __uint_as_float(v.z << 16), x5 = __uint_as_float(v.z & 0xffff0000u);
  const float x6 = __uint_as_float(v.w << 16), x7 = __uint_as_float(v.w & 0xffff0000u);
  float m = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fabsf(x2));
  m = fmaxf(fmaxf(m, fabsf(x3)), fabsf(x4));
  m = fmaxf(fmaxf(m, fabsf(x5)), fabsf(x6));
  return fmaxf(m, fabsf(x7));
}

// Item (cc >> 2)'s absmax over the 16 lanes of the row.
__device__ __forceinline__ float row_absmax_transposed(const float (&am)[kHeadGroup], int cc,
                                                       unsigned row_mask) {
  const bool b8 = cc & 8, b4 = cc & 4;
  float a1[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float keep = b8 ? am[j + 2] : am[j];
    const float send = b8 ? am[j] : am[j + 2];
    a1[j] = fmaxf(keep, __shfl_xor_sync(row_mask, send, 8));
  }
  const float keep = b4 ? a1[1] : a1[0];
  const float send = b4 ? a1[0] : a1[1];
  float r = fmaxf(keep, __shfl_xor_sync(row_mask, send, 4));
  r = fmaxf(r, __shfl_xor_sync(row_mask, r, 2));
  return fmaxf(r, __shfl_xor_sync(row_mask, r, 1));
}

// 8 codes of one chunk.  Each value's quotient 127 x / a is formed in
// float32 with one correction step: p = x * fl(127 / a) (within two units in
// the last place), the residual r = 127 x - p a is exact in a fused
// multiply-add, and q = p + r * fl(1 / a) is then within half a unit (plus
// a negligible term) of the exact quotient: a faithful rounding of it.  A
// quotient that is not itself a tie lies more than 2^-17 from one (x and a
// carry 8 significant bits), more than a unit in the last place of any
// quotient below 128, so both float32 neighbours of the exact quotient are on
// its side of every half-integer, and an exact tie is representable and
// returned exactly.  Rounding q to an integer half to even therefore gives
// the code of the exact quotient.  That rounding is an add of 1.5 * 2^23,
// which leaves the integer, in two's complement, in the low byte of the sum
// (|q| < 127.5, so no clamp is needed).  When 127 / a overflows (a below
// about 3.7e-37), the values take a correctly rounded division instead.
__device__ __forceinline__ uint32_t round_magic(float x) {
  return __float_as_uint(__fadd_rn(x, 12582912.0f));  // 1.5 * 2^23
}
__device__ __forceinline__ uint2 quant_chunk(uint4 v, float inv, float inv1, float amax) {
  constexpr float kMagic = 12582912.0f;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t t[8];
  if (inv <= 3.0e38f) {  // 127 / a finite (then 1 / a is too)
    const uint64_t inv2 = f2(inv, inv), inv12 = f2(inv1, inv1), nega2 = f2(-amax, -amax);
    const uint64_t c127 = f2(127.f, 127.f), magic2 = f2(kMagic, kMagic);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t xx = f2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
      const uint64_t p = mul2(xx, inv2);
      const uint64_t x127 = mul2(xx, c127);     // exact
      const uint64_t r = fma2(p, nega2, x127);  // exact
      const uint64_t q = fma2(r, inv12, p);
      const float2 tv = unf2(add2(q, magic2));
      t[2 * i] = __float_as_uint(tv.x);
      t[2 * i + 1] = __float_as_uint(tv.y);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      t[2 * i] = round_magic(__fdiv_rn(__fmul_rn(__uint_as_float(w[i] << 16), 127.f), amax));
      t[2 * i + 1] =
          round_magic(__fdiv_rn(__fmul_rn(__uint_as_float(w[i] & 0xffff0000u), 127.f), amax));
    }
  }
  const uint32_t lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040),
                                  0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040),
                                  0x5410);
  return make_uint2(lo, hi);
}

template <bool kQuant>
__global__ void __launch_bounds__(kThreads)
rope_append_kernel(const __grid_constant__ RopeArgs a) {
  const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 4);
  const int cc = threadIdx.x & 15;  // 16-byte chunk inside a head: dims 8cc..8cc+7
  // The 16 lanes of this row (shuffle partners of the INT8 absmax).
  const unsigned row_mask = 0xffffu << (threadIdx.x & 16);

  const bool do_q = a.q_in != nullptr && row < a.n_q_rows;
  const bool do_k = a.k_in != nullptr && row < a.n_kv_rows;
  const bool do_v = a.v_in != nullptr && row < a.n_kv_rows;
  if (!do_q && !do_k && !do_v) return;  // uniform over the row's 16 lanes

  const bool rotate = row < a.n_video;
  float c[4] = {1.f, 1.f, 1.f, 1.f}, s[4] = {0.f, 0.f, 0.f, 0.f};
  if (rotate) {
    const int64_t hw = (int64_t)a.grid_h * a.grid_w;
    const double pos_t = (double)(a.t0 + row / hw);
    const double pos_h = (double)((row / a.grid_w) % a.grid_h);
    const double pos_w = (double)(row % a.grid_w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int p = cc * 4 + i;
      const int ax = a.axis[p];
      const double pos = ax == 0 ? pos_t : (ax == 1 ? pos_h : pos_w);
      double sd, cd;
      sincos(pos * a.omega[p], &sd, &cd);
      c[i] = (float)cd;
      s[i] = (float)sd;
    }
  }

  const int64_t base = row * kRowVecs + cc;
  const uint4 *q_in = reinterpret_cast<const uint4 *>(a.q_in);
  const uint4 *k_in = reinterpret_cast<const uint4 *>(a.k_in);
  const uint4 *v_in = reinterpret_cast<const uint4 *>(a.v_in);
  uint4 *q_out = reinterpret_cast<uint4 *>(a.q_out);
  uint4 *k_out = reinterpret_cast<uint4 *>(a.k_out);
  uint4 *v_out = reinterpret_cast<uint4 *>(a.v_out);

  if constexpr (!kQuant) {
#pragma unroll 1
    for (int h0 = 0; h0 < kHeads; h0 += kHeadGroup) {
      uint4 qv[kHeadGroup], kv[kHeadGroup], vv[kHeadGroup];
#pragma unroll
      for (int g = 0; g < kHeadGroup; ++g) {
        const int64_t off = base + (int64_t)(h0 + g) * 16;
        if (do_q) qv[g] = q_in[off];
        if (do_k) kv[g] = k_in[off];
        if (do_v) vv[g] = v_in[off];
      }
#pragma unroll
      for (int g = 0; g < kHeadGroup; ++g) {
        const int64_t off = base + (int64_t)(h0 + g) * 16;
        if (do_q) q_out[off] = rotate ? rot_chunk(qv[g], c, s) : qv[g];
        if (do_k) k_out[off] = rotate ? rot_chunk(kv[g], c, s) : kv[g];
        if (do_v) v_out[off] = vv[g];
      }
    }
  } else {
    // Q rows first (rotated, bf16), then K and V into the INT8 cache, so
    // that the quantiser's loop holds no Q registers.
    if (do_q) {
#pragma unroll 1
      for (int h0 = 0; h0 < kHeads; h0 += kHeadGroup) {
        uint4 qv[kHeadGroup];
#pragma unroll
        for (int g = 0; g < kHeadGroup; ++g) qv[g] = q_in[base + (int64_t)(h0 + g) * 16];
#pragma unroll
        for (int g = 0; g < kHeadGroup; ++g)
          q_out[base + (int64_t)(h0 + g) * 16] = rotate ? rot_chunk(qv[g], c, s) : qv[g];
      }
    }
    if (!do_k && !do_v) return;  // uniform over the row's 16 lanes
#pragma unroll 1
    for (int h0 = 0; h0 < kHeads; h0 += kHeadGroup) {
      uint4 kv[kHeadGroup], vv[kHeadGroup];
#pragma unroll
      for (int g = 0; g < kHeadGroup; ++g) {
        const int64_t off = base + (int64_t)(h0 + g) * 16;
        if (do_k) kv[g] = k_in[off];
        if (do_v) vv[g] = v_in[off];
      }
      // Keys (rotated and rounded to bf16 first), then values: per pass the
      // 4 heads of the group are the butterfly's 4 items.
      auto quant_pass = [&](const uint4 (&src)[kHeadGroup], int8_t *codes, float *scales) {
        float am[kHeadGroup];
#pragma unroll
        for (int g = 0; g < kHeadGroup; ++g) am[g] = chunk_absmax(src[g]);
        const float amax = row_absmax_transposed(am, cc, row_mask);
        const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
        const float inv1 = amax > 0.f ? __frcp_rn(amax) : 0.f;
        if ((cc & 3) == 0) scales[row * kHeads + h0 + (cc >> 2)] = __fdiv_rn(amax, 127.f);
#pragma unroll
        for (int g = 0; g < kHeadGroup; ++g) {
          // 8 codes per thread at [row][head][8cc..8cc+7]
          const int64_t coff = row * (kRowElems / 8) + (int64_t)(h0 + g) * 16 + cc;
          const int owner = (threadIdx.x & 16) + 4 * g;
          const float inv_g = __shfl_sync(row_mask, inv, owner);
          const float inv1_g = __shfl_sync(row_mask, inv1, owner);
          const float amax_g = __shfl_sync(row_mask, amax, owner);
          reinterpret_cast<uint2 *>(codes)[coff] = quant_chunk(src[g], inv_g, inv1_g, amax_g);
        }
      };
      if (do_k) {
#pragma unroll
        for (int g = 0; g < kHeadGroup; ++g)
          if (rotate) kv[g] = rot_chunk(kv[g], c, s);
        quant_pass(kv, a.k_codes, a.k_scales);
      }
      if (do_v) quant_pass(vv, a.v_codes, a.v_scales);
    }
  }
}

}  // namespace

cudaError_t launch_rope_append(const RopeArgs &a, cudaStream_t stream) {
  const int64_t rows = a.n_q_rows > a.n_kv_rows ? a.n_q_rows : a.n_kv_rows;
  if (rows <= 0) return cudaSuccess;
  const int64_t blocks = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  rope_append_kernel<false><<<(unsigned)blocks, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rope_append_i8(const RopeArgs &a, cudaStream_t stream) {
  const int64_t rows = a.n_q_rows > a.n_kv_rows ? a.n_q_rows : a.n_kv_rows;
  if (rows <= 0) return cudaSuccess;
  const int64_t blocks = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  rope_append_kernel<true><<<(unsigned)blocks, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace nomas
