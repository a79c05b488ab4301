// Merge of attention results computed over disjoint key shards (memory-bound).
//
// "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
// (ai.thesatyajit.com), section "What 'world memory' stores": the standard
// preset spreads the cache over eight GPUs (sp_size 8).  Each GPU attends over
// its shard of the keys and returns (O_r, LSE_r); the whole is
// LSE = ln sum_r e^{LSE_r}, O = sum_r e^{LSE_r - LSE} O_r.
//
// A block merges 16 query rows in two phases.  Phase 1: thread (head, row)
// reads the R shard LSEs of its (row, head) -- consecutive threads read
// consecutive rows, so the reads coalesce -- and leaves the normalised
// weights e^{LSE_r - LSE} in shared memory, and the merged LSE in global
// memory.  Phase 2: the block walks its rows; for each, thread (head, chunk)
// owns one 16-byte chunk (8 dims), reads the R partial chunks (the 256
// threads cover one 4 KiB row, so every part's row is one coalesced read),
// four parts in flight at a time, and accumulates in fp32.
// Traffic per row: R x (4 KiB + 64 B) read + 4 KiB + 64 B written.
#include <cuda_bf16.h>

#include "nomas_internal.h"

namespace nomas {
namespace {

constexpr int kRows = 16;                  // query rows per block
constexpr int kThreads = kRows * kHeads;   // phase 1: one (row, head) per thread
constexpr int kWRow = kHeads + 1;          // padded [row][head] plane of one part
constexpr int kWPlane = kRows * kWRow;

__global__ void __launch_bounds__(kThreads)
merge_kernel(const uint16_t *__restrict__ o_parts, const float *__restrict__ lse_parts,
             int32_t n_parts, int64_t n_q, uint16_t *__restrict__ o, float *__restrict__ lse) {
  extern __shared__ float w_s[];  // [n_parts][kRows][kWRow]
  const int64_t row0 = (int64_t)blockIdx.x * kRows;
  {
    const int h = threadIdx.x >> 4, rr = threadIdx.x & 15;
    const int64_t row = row0 + rr;
    float *w = w_s + rr * kWRow + h;
    float m = -INFINITY;
    if (row < n_q)
      for (int r = 0; r < n_parts; ++r)
        m = fmaxf(m, lse_parts[((int64_t)r * kHeads + h) * n_q + row]);
    float total = 0.f;
    for (int r = 0; r < n_parts; ++r) {
      const float e =
          m == -INFINITY ? 0.f : expf(lse_parts[((int64_t)r * kHeads + h) * n_q + row] - m);
      w[r * kWPlane] = e;
      total += e;
    }
    const float inv = total > 0.f ? 1.f / total : 0.f;
    for (int r = 0; r < n_parts; ++r) w[r * kWPlane] *= inv;
    if (lse != nullptr && row < n_q)
      lse[(int64_t)h * n_q + row] = total > 0.f ? m + logf(total) : -INFINITY;
  }
  __syncthreads();
  const int h = threadIdx.x >> 4, c = threadIdx.x & 15;
  const int64_t part_vecs = n_q * kRowVecs;  // one part, in 16-byte chunks
  for (int i = 0; i < kRows; ++i) {
    const int64_t row = row0 + i;
    if (row >= n_q) break;
    const float *w = w_s + i * kWRow + h;
    const uint4 *src = reinterpret_cast<const uint4 *>(o_parts) + row * kRowVecs + h * 16 + c;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    auto add = [&](uint4 v, float wr) {
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] = fmaf(wr, __uint_as_float(wd[k] << 16), acc[2 * k]);
        acc[2 * k + 1] = fmaf(wr, __uint_as_float(wd[k] & 0xffff0000u), acc[2 * k + 1]);
      }
    };
    int r = 0;
    for (; r + 4 <= n_parts; r += 4) {
      uint4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = src[(int64_t)(r + k) * part_vecs];
#pragma unroll
      for (int k = 0; k < 4; ++k) add(v[k], w[(r + k) * kWPlane]);
    }
    for (; r < n_parts; ++r) add(src[(int64_t)r * part_vecs], w[r * kWPlane]);
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
      out[k] = *reinterpret_cast<uint32_t *>(&b);
    }
    reinterpret_cast<uint4 *>(o + row * kRowElems + h * kHeadDim)[c] =
        make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace

cudaError_t launch_merge(const uint16_t *o_parts, const float *lse_parts, int32_t n_parts,
                         int64_t n_q, uint16_t *o, float *lse, cudaStream_t stream) {
  if (n_q <= 0) return cudaSuccess;
  const int64_t blocks = (n_q + kRows - 1) / kRows;
  if (blocks > 0x7fffffff || n_parts > NOMAS_MAX_MERGE_PARTS) return cudaErrorInvalidValue;
  const size_t smem = (size_t)n_parts * kWPlane * sizeof(float);
  merge_kernel<<<(unsigned)blocks, kThreads, smem, stream>>>(o_parts, lse_parts, n_parts, n_q, o,
                                                              lse);
  return cudaGetLastError();
}

}  // namespace nomas
