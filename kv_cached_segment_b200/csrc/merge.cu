// Merge of attention results computed over disjoint key shards (memory-bound).
//
// "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
// (ai.thesatyajit.com), section "What 'world memory' stores": the standard
// preset spreads the cache over eight GPUs (sp_size 8).  Each GPU attends over
// its shard of the keys and returns (O_r, LSE_r); the whole is
// LSE = ln sum_r e^{LSE_r}, O = sum_r e^{LSE_r - LSE} O_r.
//
// A thread owns one 16-byte chunk (8 dims) of one (row, head): it reads the
// R shard LSEs of its (row, head) (shared by the 16 threads of the head and
// served by L1), then R chunks of O, accumulating in fp32.  Traffic per row:
// R x 4 KiB read + 4 KiB written (+ LSEs).
#include <cuda_bf16.h>

#include "nomas_internal.h"

namespace nomas {
namespace {

constexpr int kThreads = 256;  // one row (16 heads x 16 chunks) per block

__global__ void __launch_bounds__(kThreads)
merge_kernel(const uint16_t *__restrict__ o_parts, const float *__restrict__ lse_parts,
             int32_t n_parts, int64_t n_q, uint16_t *__restrict__ o, float *__restrict__ lse) {
  const int64_t row = blockIdx.x;
  const int head = threadIdx.x >> 4;
  const int chunk = threadIdx.x & 15;
  if (row >= n_q) return;
  float m = -INFINITY;
  for (int r = 0; r < n_parts; ++r)
    m = fmaxf(m, lse_parts[((int64_t)r * kHeads + head) * n_q + row]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float total = 0.f;
  if (m != -INFINITY) {
    for (int r = 0; r < n_parts; ++r) {
      const float w = expf(lse_parts[((int64_t)r * kHeads + head) * n_q + row] - m);
      total += w;
      const uint4 v = reinterpret_cast<const uint4 *>(
          o_parts + ((int64_t)r * n_q + row) * kRowElems + head * kHeadDim)[chunk];
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(wd[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(wd[i] & 0xffff0000u), acc[2 * i + 1]);
      }
    }
  }
  const float inv = total > 0.f ? 1.f / total : 0.f;
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    out[i] = *reinterpret_cast<uint32_t *>(&b);
  }
  reinterpret_cast<uint4 *>(o + row * kRowElems + head * kHeadDim)[chunk] =
      make_uint4(out[0], out[1], out[2], out[3]);
  if (lse != nullptr && chunk == 0)
    lse[(int64_t)head * n_q + row] = total > 0.f ? m + logf(total) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge(const uint16_t *o_parts, const float *lse_parts, int32_t n_parts,
                         int64_t n_q, uint16_t *o, float *lse, cudaStream_t stream) {
  if (n_q <= 0) return cudaSuccess;
  if (n_q > 0x7fffffff) return cudaErrorInvalidValue;
  merge_kernel<<<(unsigned)n_q, kThreads, 0, stream>>>(o_parts, lse_parts, n_parts, n_q, o, lse);
  return cudaGetLastError();
}

}  // namespace nomas
