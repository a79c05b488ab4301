// Internal interfaces between the C-ABI layer (abi.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nomas.h"

namespace nomas {

constexpr int kHeads = 16;
constexpr int kHeadDim = 128;
constexpr int kRowElems = kHeads * kHeadDim;       // 2048 bf16
constexpr int64_t kRowBytes = kRowElems * 2;       // 4096 B
constexpr int kRowVecs = kRowBytes / 16;           // 256 x 16 B

// ---------------------------------------------------------------- RoPE ----
struct RopeArgs {
  const uint16_t *q_in;   // may be null
  uint16_t *q_out;
  const uint16_t *k_in;   // may be null
  uint16_t *k_out;
  const uint16_t *v_in;   // may be null (no V stream)
  uint16_t *v_out;
  int64_t n_q_rows;       // rows of Q processed (video + text)
  int64_t n_kv_rows;      // rows of K (and V) processed
  int64_t n_video;        // rows [0, n_video) are rotated (0: plain copy)
  int32_t grid_h, grid_w, t0;
  // Per-pair angular frequency (radians per position unit) and the axis
  // (0 = t, 1 = h, 2 = w) of the 64 rotation pairs of a head.
  double omega[kHeadDim / 2];
  int8_t axis[kHeadDim / 2];
  // INT8 cache output (used by launch_rope_append_i8 instead of k_out/v_out):
  // codes [rows][16][128] int8 and scales [rows][16] fp32, per token and head.
  int8_t *k_codes, *v_codes;
  float *k_scales, *v_scales;
};
cudaError_t launch_rope_append(const RopeArgs &a, cudaStream_t stream);
cudaError_t launch_rope_append_i8(const RopeArgs &a, cudaStream_t stream);

// -------------------------------------------------------------- select ----
constexpr int kSelectHostFramesPerLaunch = 2048;
struct SelectArgs {
  const uint16_t *src_k, *src_v;
  uint16_t *dst_k, *dst_v;
  const int32_t *idx_dev;      // device list, or null for the host list below
  int32_t *dev_err;
  int64_t frame_vecs;          // 16-B vectors per frame per tensor
  int64_t n_src_frames;
  int32_t n_frames;            // frames handled by this launch
  int32_t first_frame;         // window frame of entry 0 of this launch
};
struct SelectHostList {
  int32_t idx[kSelectHostFramesPerLaunch];
};
cudaError_t launch_select(const SelectArgs &a, const SelectHostList *host_list,
                          cudaStream_t stream);
// Gather + dequantize from an INT8 cache into a bf16 window.
struct SelectI8Args {
  const int8_t *src_k, *src_v;        // codes [rows][16][128]
  const float *src_ks, *src_vs;       // scales [rows][16]
  uint16_t *dst_k, *dst_v;            // bf16 [rows][16][128]
  const int32_t *idx_dev;
  int32_t *dev_err;
  int64_t tokens_per_frame;
  int64_t n_src_frames;
  int32_t n_frames;
  int32_t first_frame;
};
cudaError_t launch_select_i8(const SelectI8Args &a, const SelectHostList *host_list,
                             cudaStream_t stream);

// ----------------------------------------------------------- attention ----
constexpr int kMaxSpans = 4;
struct AttnArgs {
  CUtensorMap tmap_q;
  CUtensorMap tmap_k[kMaxSpans];
  CUtensorMap tmap_v[kMaxSpans];
  int64_t span_len[kMaxSpans];
  int32_t n_spans;             // non-empty spans, packed to the front
  int32_t heads;               // heads per row of Q, K, V, O (16; fewer for head-sharded
                               // dense calls): rows are heads x 128 elements
  int32_t n_q;
  uint16_t *o;
  float *lse;                  // may be null
  float scale_log2;            // softmax scale * log2(e)
  int32_t *dev_err;            // may be null
  unsigned long long wait_limit_ns;
  int32_t testing_skip_load;   // -1, or the K/V load index the producer leaves out
  // Block-sparse selection (null tile_list: every tile of every span, in order).
  const int32_t *tile_list;    // [q_blocks][heads][max_tiles] global key-tile ids
  const int32_t *tile_count;   // [q_blocks][heads] entries used in each row
  int32_t max_tiles;
  int32_t tile_base[kMaxSpans + 1];  // first global tile id of each span; [n_spans] = total
  // Split of the key tiles (dense mode): block z of the grid's third
  // dimension streams global tiles [T z / S, T (z + 1) / S) of the T tiles and
  // writes its partial O and LSE to part z of o ([S][n_q][16][128]) and lse
  // ([S][16][n_q]).  1: no split.
  int32_t kv_splits;
  // Owner-routed partial outputs (key-sharded attention over peer memory):
  // when n_owners > 0, query row i belongs to the owner s with
  // owner_row0[s] <= i < owner_row0[s + 1], and its O and LSE go to part
  // owner_slot of that owner's stacked buffers owner_o[s] ([R][n_q][16][128])
  // and owner_lse[s] ([R][16][n_q]) instead of o and lse.
  int32_t n_owners;
  int32_t owner_slot;
  int64_t owner_row0[NOMAS_MAX_MERGE_PARTS + 1];
  uint16_t *owner_o[NOMAS_MAX_MERGE_PARTS];
  float *owner_lse[NOMAS_MAX_MERGE_PARTS];
  // INT8 history: when i8 != 0, span 0 is INT8 codes (tmap_k[0] / tmap_v[0]
  // map [len][16][128] int8) with fp32 scales i8_scale[0] (K) and
  // i8_scale[1] (V), [len][16]; value = code * scale.
  int32_t i8;
  const float *i8_scale[2];
};
cudaError_t launch_attention(const AttnArgs &a, cudaStream_t stream);
// The one-tile (pair = false) and CTA-pair schedules: dense bf16 keys only,
// K/V tensor maps with 128-row (one-tile) or 64-row (pair) boxes.
bool attention_pair_supported(const AttnArgs &a);
cudaError_t launch_attention_pair(const AttnArgs &a, bool pair, cudaStream_t stream);
cudaError_t launch_attention_empty(uint16_t *o, float *lse, int64_t n_q, int32_t heads,
                                   cudaStream_t stream);

// ---------------------------------------------------------------- merge ----
// Rows of `heads` heads (1, 2, 4, 8 or 16).
cudaError_t launch_merge(const uint16_t *o_parts, const float *lse_parts, int32_t n_parts,
                         int64_t n_q, int32_t heads, uint16_t *o, float *lse, cudaStream_t stream);
// Rows [row0, row0 + n_rows) of n_parts partials found through pointer
// tables (host arrays), written to n_outs outputs.
cudaError_t launch_merge_peers(const uint16_t *const *o_parts, const float *const *lse_parts,
                               int32_t n_parts, int64_t n_q, int64_t row0, int64_t n_rows,
                               uint16_t *const *o_outs, float *const *lse_outs, int32_t n_outs,
                               cudaStream_t stream);

// ----------------------------------------------------------------- errors --
// Sets the message nomas_last_error() returns on this thread; returns st.
nomas_status report_error(nomas_status st, const char *message);

}  // namespace nomas
