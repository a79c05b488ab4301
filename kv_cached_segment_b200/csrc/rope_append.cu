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

// Symmetric INT8 quantisation of one (token, head): the 16 threads of the row
// each hold 8 of the 128 bf16 values; the absmax a is reduced with shuffles
// inside the row's 16 lanes.  The stored scale is a / 127 and code =
// rint(x * (127 / a)); the two divisions (one per token and head) and the
// product round to nearest in float32 and the conversion rounds half to even,
// so the codes are reproducible bit for bit; an all-zero head gets scale 0.
__device__ __forceinline__ uint2 quant_chunk(uint4 v, unsigned row_mask, float *scale_out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float x[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(row_mask, amax, off));
  const float scale = __fdiv_rn(amax, 127.f);
  uint32_t lo = 0, hi = 0;
  if (amax > 0.f) {
    const float inv = __fdiv_rn(127.f, amax);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = __float2int_rn(__fmul_rn(x[i], inv));
      q = max(-127, min(127, q));
      const uint32_t b = (uint32_t)(q & 0xff);
      if (i < 4)
        lo |= b << (8 * i);
      else
        hi |= b << (8 * (i - 4));
    }
  }
  *scale_out = scale;
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
      if constexpr (kQuant) {
        // codes: 8 bytes per thread at [row][head][8cc..8cc+7]; one scale per (row, head)
        const int64_t coff = row * (kRowElems / 8) + (int64_t)(h0 + g) * 16 + cc;
        const int64_t soff = row * kHeads + h0 + g;
        float sc;
        if (do_k) {
          const uint2 q8 = quant_chunk(rotate ? rot_chunk(kv[g], c, s) : kv[g], row_mask, &sc);
          reinterpret_cast<uint2 *>(a.k_codes)[coff] = q8;
          if (cc == 0) a.k_scales[soff] = sc;
        }
        if (do_v) {
          const uint2 q8 = quant_chunk(vv[g], row_mask, &sc);
          reinterpret_cast<uint2 *>(a.v_codes)[coff] = q8;
          if (cc == 0) a.v_scales[soff] = sc;
        }
      } else {
        if (do_k) k_out[off] = rotate ? rot_chunk(kv[g], c, s) : kv[g];
        if (do_v) v_out[off] = vv[g];
      }
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
