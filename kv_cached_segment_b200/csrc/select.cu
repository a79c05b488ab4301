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
// thread issues its 8 independent 16-byte loads before its 8 stores.
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
