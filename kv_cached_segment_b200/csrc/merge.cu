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
// memory.  Phase 2: the block walks its rows; thread (head, chunk) owns one
// 16-byte chunk (8 dims) of a row, reads the R partial chunks (256 threads
// cover 4 KiB of rows, so every part's rows are one coalesced read), four
// parts in flight at a time, and accumulates in fp32.  Rows hold H heads
// (16, or fewer for head-sharded attention): 16 / H rows per pass.
// Traffic per row: R x (H x 256 B + 4 H B) read + H x 256 B + 4 H B written.
//
// The same kernel serves two layouts of the partials: stacked in one buffer
// (nomas_attention_merge, all rows, one output), or found through a table of
// R pointers with a row range and up to 32 outputs (nomas_attention_merge_peers).
// With pointers into other GPUs' memory, the table form is the exchange and
// the merge in one kernel: each GPU reads the partial rows it owns from every
// GPU and stores the merged rows into every GPU's output, with plain loads
// and stores over NVLink.
#include <type_traits>

#include <cuda_bf16.h>

#include "nomas_internal.h"

namespace nomas {
namespace {

constexpr int kRows = 16;                  // query rows per block
constexpr int kThreads = kRows * kHeads;   // phase 1: one (row, head) per thread
constexpr int kWRow = kHeads + 1;          // padded [row][head] plane of one part
constexpr int kWPlane = kRows * kWRow;
constexpr int kChunks = kHeadDim * 2 / 16;  // 16-byte chunks per head

// Where the R partial results live.  Stacked: one buffer, part r at a fixed
// stride ([R][n_q][H][128] and [R][H][n_q]).  Table (16 heads): R base
// pointers, any of which may address another GPU's memory mapped into this
// process.
template <int H>
struct StackedParts {
  const uint16_t *o;
  const float *lse;
  int64_t n_q;
  __device__ __forceinline__ const uint4 *o_row(int r, int64_t row) const {
    return reinterpret_cast<const uint4 *>(o) + ((int64_t)r * n_q + row) * (H * kChunks);
  }
  __device__ __forceinline__ float lse_at(int r, int h, int64_t row) const {
    return lse[((int64_t)r * H + h) * n_q + row];
  }
};
struct TableParts {
  const uint16_t *o[NOMAS_MAX_MERGE_PARTS];
  const float *lse[NOMAS_MAX_MERGE_PARTS];
  int64_t n_q;
  __device__ __forceinline__ const uint4 *o_row(int r, int64_t row) const {
    return reinterpret_cast<const uint4 *>(o[r]) + row * (kHeads * kChunks);
  }
  __device__ __forceinline__ float lse_at(int r, int h, int64_t row) const {
    return lse[r][(int64_t)h * n_q + row];
  }
};
// Where the merged rows go: every listed output gets the same rows ([n_q]
// rows each; a null LSE pointer skips that output's LSE).
struct Outputs {
  uint16_t *o[NOMAS_MAX_MERGE_OUTPUTS];
  float *lse[NOMAS_MAX_MERGE_OUTPUTS];
  int32_t n;
};

template <class Parts, int H>
__global__ void __launch_bounds__(kThreads)
merge_kernel(const Parts parts, int32_t n_parts, int64_t n_q, int64_t row_begin,
             int64_t row_end, const Outputs outs) {
  extern __shared__ float w_s[];  // [n_parts][kRows][kWRow]
  const int64_t row0 = row_begin + (int64_t)blockIdx.x * kRows;
  if (threadIdx.x < kRows * H) {
    const int h = threadIdx.x >> 4, rr = threadIdx.x & 15;
    const int64_t row = row0 + rr;
    float *w = w_s + rr * kWRow + h;
    // A NaN LSE marks a partial whose attention block aborted: the merged
    // row becomes NaN (weights and LSE), never a merge of the other parts.
    float m = -INFINITY;
    bool bad = false;
    if (row < row_end)
      for (int r = 0; r < n_parts; ++r) {
        const float x = parts.lse_at(r, h, row);
        bad |= isnan(x);
        m = fmaxf(m, x);
      }
    float total = 0.f;
    for (int r = 0; r < n_parts; ++r) {
      const float e = m == -INFINITY ? 0.f : expf(parts.lse_at(r, h, row) - m);
      w[r * kWPlane] = e;
      total += e;
    }
    const float inv = bad ? NAN : (total > 0.f ? 1.f / total : 0.f);
    for (int r = 0; r < n_parts; ++r) w[r * kWPlane] *= inv;
    if (row < row_end) {
      const float l = bad ? NAN : (total > 0.f ? m + logf(total) : -INFINITY);
      for (int k = 0; k < outs.n; ++k)
        if (outs.lse[k] != nullptr) outs.lse[k][(int64_t)h * n_q + row] = l;
    }
  }
  __syncthreads();
  // Phase 2: H x 16 chunks per row, 16 / H rows per pass, H passes.
  const int chunk = threadIdx.x % (H * kChunks);
  const int h = chunk / kChunks;
  for (int pass = 0; pass < H; ++pass) {
    const int i = pass * (kThreads / (H * kChunks)) + (int)threadIdx.x / (H * kChunks);
    const int64_t row = row0 + i;
    if (row >= row_end) break;
    const float *w = w_s + i * kWRow + h;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    auto add = [&](uint4 v, float wr) {
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] = fmaf(wr, __uint_as_float(wd[k] << 16), acc[2 * k]);
        acc[2 * k + 1] = fmaf(wr, __uint_as_float(wd[k] & 0xffff0000u), acc[2 * k + 1]);
      }
    };
    const int off = chunk;  // this thread's 16-byte chunk of the row
    int r = 0;
    for (; r + 4 <= n_parts; r += 4) {
      uint4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = parts.o_row(r + k, row)[off];
#pragma unroll
      for (int k = 0; k < 4; ++k) add(v[k], w[(r + k) * kWPlane]);
    }
    for (; r < n_parts; ++r) add(parts.o_row(r, row)[off], w[r * kWPlane]);
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
      out[k] = *reinterpret_cast<uint32_t *>(&b);
    }
    const uint4 packed = make_uint4(out[0], out[1], out[2], out[3]);
    for (int k = 0; k < outs.n; ++k)
      reinterpret_cast<uint4 *>(outs.o[k] + row * (H * kHeadDim))[off] = packed;
  }
}

}  // namespace

cudaError_t launch_merge(const uint16_t *o_parts, const float *lse_parts, int32_t n_parts,
                         int64_t n_q, int32_t heads, uint16_t *o, float *lse, cudaStream_t stream) {
  if (n_q <= 0) return cudaSuccess;
  const int64_t blocks = (n_q + kRows - 1) / kRows;
  if (blocks > 0x7fffffff || n_parts > NOMAS_MAX_MERGE_PARTS) return cudaErrorInvalidValue;
  const size_t smem = (size_t)n_parts * kWPlane * sizeof(float);
  Outputs outs{};
  outs.o[0] = o;
  outs.lse[0] = lse;
  outs.n = 1;
  auto go = [&](auto hc) {
    constexpr int H = decltype(hc)::value;
    merge_kernel<StackedParts<H>, H><<<(unsigned)blocks, kThreads, smem, stream>>>(
        StackedParts<H>{o_parts, lse_parts, n_q}, n_parts, n_q, 0, n_q, outs);
  };
  switch (heads) {
    case 1: go(std::integral_constant<int, 1>{}); break;
    case 2: go(std::integral_constant<int, 2>{}); break;
    case 4: go(std::integral_constant<int, 4>{}); break;
    case 8: go(std::integral_constant<int, 8>{}); break;
    case kHeads: go(std::integral_constant<int, kHeads>{}); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_merge_peers(const uint16_t *const *o_parts, const float *const *lse_parts,
                               int32_t n_parts, int64_t n_q, int64_t row0, int64_t n_rows,
                               uint16_t *const *o_outs, float *const *lse_outs, int32_t n_outs,
                               cudaStream_t stream) {
  if (n_rows <= 0) return cudaSuccess;
  const int64_t blocks = (n_rows + kRows - 1) / kRows;
  if (blocks > 0x7fffffff || n_parts < 1 || n_parts > NOMAS_MAX_MERGE_PARTS || n_outs < 1 ||
      n_outs > NOMAS_MAX_MERGE_OUTPUTS)
    return cudaErrorInvalidValue;
  TableParts parts{};
  for (int r = 0; r < n_parts; ++r) {
    parts.o[r] = o_parts[r];
    parts.lse[r] = lse_parts[r];
  }
  parts.n_q = n_q;
  Outputs outs{};
  for (int k = 0; k < n_outs; ++k) {
    outs.o[k] = o_outs[k];
    outs.lse[k] = lse_outs != nullptr ? lse_outs[k] : nullptr;
  }
  outs.n = n_outs;
  const size_t smem = (size_t)n_parts * kWPlane * sizeof(float);
  merge_kernel<TableParts, kHeads><<<(unsigned)blocks, kThreads, smem, stream>>>(
      parts, n_parts, n_q, row0, row0 + n_rows, outs);
  return cudaGetLastError();
}

}  // namespace nomas
