// Frame-list gather of the KV cache into a contiguous window (memory-bound,
// bit-exact).
//
// "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
// (ai.thesatyajit.com), section "The 4090 preset": before each segment only a
// chosen list of past latent frames is restored to the GPU.  A latent frame is
// a contiguous run of tokens_per_frame cache rows, so the gather is a list of
// large contiguous block copies: 8 KiB read + 8 KiB written per selected token
// (K and V).
//
// Grid: x = 32-KiB tiles of one frame, y = window frame, z = K or V.  Every
// thread issues its 8 independent 16-byte loads before its 8 stores.  A
// second kernel gathers from an INT8 cache and dequantizes into bf16.
#include <cuda_bf16.h>

#include "nomas_internal.h"

namespace nomas {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;
constexpr int kTileVecs = kThreads * kUnroll;  // 2048 x 16 B = 32 KiB

__global__ void __launch_bounds__(kThreads)
select_kernel(const __grid_constant__ SelectArgs a, const __grid_constant__ SelectHostList hl) {
  const int j = blockIdx.y;  // entry of this launch
  int32_t f;
  if (a.idx_dev != nullptr) {
    f = a.idx_dev[a.first_frame + j];
    if (f < 0 || (int64_t)f >= a.n_src_frames) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0 && a.dev_err != nullptr)
        atomicOr(a.dev_err, NOMAS_DEVERR_BAD_FRAME_INDEX);
      return;
    }
  } else {
    f = hl.idx[j];
  }
  const uint4 *src = reinterpret_cast<const uint4 *>(blockIdx.z == 0 ? a.src_k : a.src_v);
  uint4 *dst = reinterpret_cast<uint4 *>(blockIdx.z == 0 ? a.dst_k : a.dst_v);
  src += (int64_t)f * a.frame_vecs;
  dst += (int64_t)(a.first_frame + j) * a.frame_vecs;

  const int64_t t0 = (int64_t)blockIdx.x * kTileVecs + threadIdx.x;
  uint4 buf[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int64_t i = t0 + (int64_t)u * kThreads;
    if (i < a.frame_vecs) buf[u] = src[i];
  }
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int64_t i = t0 + (int64_t)u * kThreads;
    if (i < a.frame_vecs) dst[i] = buf[u];
  }
}

// Gather + dequantize: window rows of frame j receive code * scale of source
// frame idx[j], the exact product rounded once to the nearest bf16 (ties to
// even).  A
// thread handles 8 codes (one 16-byte bf16 output chunk) per step: 4,224 B
// read (codes + scales, K and V) and 8 KiB written per selected token.
constexpr int kDqUnroll = 4;
constexpr int kDqTile = kThreads * kDqUnroll;  // chunks of 8 codes per block

// code * scale rounded to float32 "to odd": truncated toward zero, with the
// last bit set when the truncation dropped anything.  The product of a 7-bit
// code and a 24-bit scale has at most 31 significant bits, so the fused
// multiply-add residual below is exact and is zero exactly when the product
// is.  bf16 keeps 8 significant bits, at least two fewer than float32's 24,
// so rounding the round-to-odd float32 to the nearest bf16 gives the nearest
// bf16 of the exact product: no double-rounding error.
__device__ __forceinline__ float product_round_to_odd(float code, float scale) {
  const float r = __fmul_rz(code, scale);
  const float e = __fmaf_rn(code, scale, -r);
  return __uint_as_float(__float_as_uint(r) | (e != 0.f ? 1u : 0u));
}

__global__ void __launch_bounds__(kThreads)
select_i8_kernel(const __grid_constant__ SelectI8Args a, const __grid_constant__ SelectHostList hl) {
  const int j = blockIdx.y;
  int32_t f;
  if (a.idx_dev != nullptr) {
    f = a.idx_dev[a.first_frame + j];
    if (f < 0 || (int64_t)f >= a.n_src_frames) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0 && a.dev_err != nullptr)
        atomicOr(a.dev_err, NOMAS_DEVERR_BAD_FRAME_INDEX);
      return;
    }
  } else {
    f = hl.idx[j];
  }
  const bool is_k = blockIdx.z == 0;
  const uint2 *codes = reinterpret_cast<const uint2 *>(is_k ? a.src_k : a.src_v);
  const float *scales = is_k ? a.src_ks : a.src_vs;
  uint4 *dst = reinterpret_cast<uint4 *>(is_k ? a.dst_k : a.dst_v);
  const int64_t src_row0 = (int64_t)f * a.tokens_per_frame;
  const int64_t dst_row0 = (int64_t)(a.first_frame + j) * a.tokens_per_frame;
  const int64_t n_chunks = a.tokens_per_frame * (kRowElems / 8);  // per frame

  const int64_t c0 = (int64_t)blockIdx.x * kDqTile + threadIdx.x;
  uint2 cv[kDqUnroll];
  float sv[kDqUnroll];
#pragma unroll
  for (int u = 0; u < kDqUnroll; ++u) {
    const int64_t c = c0 + (int64_t)u * kThreads;
    if (c < n_chunks) {
      cv[u] = codes[src_row0 * (kRowElems / 8) + c];
      sv[u] = scales[(src_row0 + c / (kRowElems / 8)) * kHeads + (c % (kRowElems / 8)) / 16];
    }
  }
#pragma unroll
  for (int u = 0; u < kDqUnroll; ++u) {
    const int64_t c = c0 + (int64_t)u * kThreads;
    if (c < n_chunks) {
      const uint32_t w[2] = {cv[u].x, cv[u].y};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = (float)(int8_t)((w[i / 2] >> (16 * (i & 1))) & 0xff);
        const float hi = (float)(int8_t)((w[i / 2] >> (16 * (i & 1) + 8)) & 0xff);
        __nv_bfloat162 b = __floats2bfloat162_rn(product_round_to_odd(lo, sv[u]),
                                                 product_round_to_odd(hi, sv[u]));
        o[i] = *reinterpret_cast<uint32_t *>(&b);
      }
      dst[dst_row0 * kRowVecs + c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, const SelectHostList *host_list,
                          cudaStream_t stream) {
  if (a.n_frames <= 0) return cudaSuccess;
  const int64_t tiles = (a.frame_vecs + kTileVecs - 1) / kTileVecs;
  if (tiles > 0x7fffffff || a.n_frames > 65535) return cudaErrorInvalidValue;
  dim3 grid((unsigned)tiles, (unsigned)a.n_frames, 2);
  static const SelectHostList kEmpty = {};
  select_kernel<<<grid, kThreads, 0, stream>>>(a, host_list ? *host_list : kEmpty);
  return cudaGetLastError();
}

}  // namespace nomas

namespace nomas {

cudaError_t launch_select_i8(const SelectI8Args &a, const SelectHostList *host_list,
                             cudaStream_t stream) {
  if (a.n_frames <= 0) return cudaSuccess;
  const int64_t n_chunks = a.tokens_per_frame * (kRowElems / 8);
  const int64_t tiles = (n_chunks + kDqTile - 1) / kDqTile;
  if (tiles > 0x7fffffff || a.n_frames > 65535) return cudaErrorInvalidValue;
  dim3 grid((unsigned)tiles, (unsigned)a.n_frames, 2);
  static const SelectHostList kEmpty = {};
  select_i8_kernel<<<grid, kThreads, 0, stream>>>(a, host_list ? *host_list : kEmpty);
  return cudaGetLastError();
}

}  // namespace nomas
