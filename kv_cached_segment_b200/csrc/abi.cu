// C-ABI entry points of libnomas (declared in include/nomas.h).
//
// Host side only: argument validation, tensor-map (TMA descriptor) encoding
// and kernel launches.  Every check happens before anything is launched, so a
// rejected call leaves device memory untouched.  Nothing here allocates
// device memory, synchronises or keeps a caller pointer past the call.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "nomas.h"
#include "nomas_internal.h"

using namespace nomas;

namespace {

thread_local std::string g_last_error;

nomas_status fail(nomas_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

nomas_status cuda_fail(cudaError_t e, const char *what) {
  return fail(NOMAS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

nomas_status ok() {
  g_last_error.clear();
  return NOMAS_OK;
}

// NVTX range over one C-ABI call (header-only NVTX v3: inert unless a
// profiler is attached), so that traces show which call enqueued which work.
struct ApiRange {
  explicit ApiRange(const char *name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange &) = delete;
  ApiRange &operator=(const ApiRange &) = delete;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [a, a + an) and [b, b + bn) overlap (bytes).
bool overlap(const void *a, int64_t an, const void *b, int64_t bn) {
  if (a == nullptr || b == nullptr || an <= 0 || bn <= 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + (uintptr_t)bn && y < x + (uintptr_t)an;
}

nomas_status check_shape(int32_t heads, int32_t head_dim) {
  if (heads != kHeads || head_dim != kHeadDim)
    return fail(NOMAS_ERR_UNSUPPORTED, "only heads=16, head_dim=128 are implemented (got %d, %d)",
                heads, head_dim);
  return NOMAS_OK;
}

nomas_status check_layout(const nomas_seg_layout *l, int64_t *n_video) {
  if (l == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "layout is NULL");
  if (l->frames < 0 || l->grid_h < 0 || l->grid_w < 0 || l->n_text < 0 || l->t0 < 0)
    return fail(NOMAS_ERR_INVALID_ARG, "layout fields must be >= 0");
  *n_video = (int64_t)l->frames * l->grid_h * l->grid_w;
  if (*n_video > ((int64_t)1 << 31) || l->t0 > (1 << 30))
    return fail(NOMAS_ERR_INVALID_ARG, "layout too large");
  return NOMAS_OK;
}

// Fills the per-pair frequency and axis tables of a rotary configuration.
nomas_status fill_rope(const nomas_rope3d_cfg *cfg, RopeArgs *a) {
  if (cfg == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "rope cfg is NULL");
  const int d[3] = {cfg->d_t, cfg->d_h, cfg->d_w};
  for (int i = 0; i < 3; ++i)
    if (d[i] <= 0 || (d[i] & 1))
      return fail(NOMAS_ERR_INVALID_ARG, "rope split entries must be even and > 0 (%d, %d, %d)",
                  d[0], d[1], d[2]);
  if (d[0] + d[1] + d[2] != kHeadDim)
    return fail(NOMAS_ERR_INVALID_ARG, "rope split must sum to head_dim=128 (%d+%d+%d)", d[0],
                d[1], d[2]);
  if (!(cfg->theta > 0.f) || !std::isfinite(cfg->theta))
    return fail(NOMAS_ERR_INVALID_ARG, "rope theta must be finite and > 0");
  const double theta = (double)cfg->theta;
  for (int p = 0; p < kHeadDim / 2; ++p) {
    int ax, j;
    if (2 * p < d[0]) {
      ax = 0;
      j = p;
    } else if (2 * p < d[0] + d[1]) {
      ax = 1;
      j = p - d[0] / 2;
    } else {
      ax = 2;
      j = p - (d[0] + d[1]) / 2;
    }
    a->axis[p] = (int8_t)ax;
    a->omega[p] = std::pow(theta, -2.0 * (double)j / (double)d[ax]);
  }
  return NOMAS_OK;
}

// cuTensorMapEncodeTiled, reached through the runtime so the library does not
// link libcuda directly.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D view of a [rows][heads][128] bf16 tensor (heads 16 unless a
// head-sharded call has fewer): inner extent heads x 128 elements, row pitch
// heads x 256 B; box = 64 elements (128 B, one swizzle span) x box_rows rows.
nomas_status rows_map(CUtensorMap *m, const void *ptr, int64_t rows, uint32_t box_rows = 128,
                      int32_t heads = kHeads) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(NOMAS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {(cuuint64_t)heads * kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)heads * kHeadDim * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NOMAS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return NOMAS_OK;
}

// 2-D view of a [rows][16][128] int8 code tensor: inner extent 2048 bytes,
// row pitch 2048 B; box = 128 codes (one head, one swizzle span) x 128 rows.
nomas_status codes_map(CUtensorMap *m, const void *ptr, int64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(NOMAS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {(cuuint64_t)kRowElems, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kRowElems};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NOMAS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return NOMAS_OK;
}

// A bf16 or INT8 layer cache seen by the append path.
struct CacheView {
  void *k, *v;
  float *k_scale, *v_scale;  // INT8 only
  int64_t capacity, len;
  int32_t heads, head_dim;
  bool int8;
};

nomas_status append_common(const CacheView &c, const void *k_seg, const void *v_seg,
                           int64_t n_tokens, const void *q_in, void *q_out,
                           const nomas_seg_layout *layout, const nomas_rope3d_cfg *cfg,
                           void *stream) {
  nomas_status st = check_shape(c.heads, c.head_dim);
  if (st != NOMAS_OK) return st;
  if (c.k == nullptr || c.v == nullptr || !aligned16(c.k) || !aligned16(c.v))
    return fail(NOMAS_ERR_INVALID_ARG, "cache k/v must be non-NULL and 16-byte aligned");
  if (c.int8 && (c.k_scale == nullptr || c.v_scale == nullptr || !aligned16(c.k_scale) ||
                 !aligned16(c.v_scale)))
    return fail(NOMAS_ERR_INVALID_ARG, "cache scales must be non-NULL and 16-byte aligned");
  if (c.capacity < 0 || c.len < 0 || c.len > c.capacity)
    return fail(NOMAS_ERR_INVALID_ARG, "cache len/capacity inconsistent (%lld/%lld)",
                (long long)c.len, (long long)c.capacity);
  if (n_tokens < 0) return fail(NOMAS_ERR_INVALID_ARG, "n_tokens < 0");
  if (n_tokens > 0 && (k_seg == nullptr || v_seg == nullptr))
    return fail(NOMAS_ERR_INVALID_ARG, "k_seg and v_seg are required");
  if ((q_in == nullptr) != (q_out == nullptr))
    return fail(NOMAS_ERR_INVALID_ARG, "q_in and q_out must both be set or both be NULL");
  if (!aligned16(k_seg) || !aligned16(v_seg) || !aligned16(q_in) || !aligned16(q_out))
    return fail(NOMAS_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  RopeArgs a{};
  int64_t n_video = 0, n_text = 0;
  if (layout != nullptr) {
    if ((st = check_layout(layout, &n_video)) != NOMAS_OK) return st;
    n_text = layout->n_text;
  }
  if (cfg != nullptr) {
    if (layout == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "rope cfg given without a layout");
    if ((st = fill_rope(cfg, &a)) != NOMAS_OK) return st;
    if (n_video != n_tokens)
      return fail(NOMAS_ERR_INVALID_ARG, "n_tokens (%lld) != frames*grid_h*grid_w (%lld)",
                  (long long)n_tokens, (long long)n_video);
  }
  if (c.len + n_tokens > c.capacity)
    return fail(NOMAS_ERR_CAPACITY, "append of %lld rows at len %lld exceeds capacity %lld",
                (long long)n_tokens, (long long)c.len, (long long)c.capacity);
  const int64_t q_rows = q_in != nullptr ? n_tokens + n_text : 0;
  const int64_t elem = c.int8 ? 1 : 2;  // bytes per cached value
  uint8_t *k_dst = static_cast<uint8_t *>(c.k) + c.len * kRowElems * elem;
  uint8_t *v_dst = static_cast<uint8_t *>(c.v) + c.len * kRowElems * elem;
  const int64_t seg_bytes = n_tokens * kRowBytes, q_bytes = q_rows * kRowBytes;
  const int64_t dst_bytes = n_tokens * kRowElems * elem;
  if (overlap(k_seg, seg_bytes, k_dst, dst_bytes) || overlap(v_seg, seg_bytes, v_dst, dst_bytes) ||
      overlap(k_seg, seg_bytes, v_dst, dst_bytes) || overlap(v_seg, seg_bytes, k_dst, dst_bytes))
    return fail(NOMAS_ERR_INVALID_ARG, "segment K/V overlap the cache rows being written");
  if (q_in != nullptr && q_out != q_in && overlap(q_in, q_bytes, q_out, q_bytes))
    return fail(NOMAS_ERR_INVALID_ARG, "q_out partially overlaps q_in");
  if (q_out != nullptr && (overlap(q_out, q_bytes, k_dst, dst_bytes) ||
                           overlap(q_out, q_bytes, v_dst, dst_bytes)))
    return fail(NOMAS_ERR_INVALID_ARG, "q_out overlaps the cache rows being written");
  a.q_in = static_cast<const uint16_t *>(q_in);
  a.q_out = static_cast<uint16_t *>(q_out);
  a.k_in = static_cast<const uint16_t *>(k_seg);
  a.v_in = static_cast<const uint16_t *>(v_seg);
  if (c.int8) {
    a.k_codes = reinterpret_cast<int8_t *>(k_dst);
    a.v_codes = reinterpret_cast<int8_t *>(v_dst);
    a.k_scales = c.k_scale + c.len * kHeads;
    a.v_scales = c.v_scale + c.len * kHeads;
  } else {
    a.k_out = reinterpret_cast<uint16_t *>(k_dst);
    a.v_out = reinterpret_cast<uint16_t *>(v_dst);
  }
  a.n_q_rows = q_rows;
  a.n_kv_rows = n_tokens;
  a.n_video = cfg != nullptr ? n_tokens : 0;
  if (layout != nullptr) {
    a.grid_h = layout->grid_h;
    a.grid_w = layout->grid_w;
    a.t0 = layout->t0;
  }
  if (q_rows > 0 || n_tokens > 0) {
    const cudaError_t e = c.int8 ? launch_rope_append_i8(a, static_cast<cudaStream_t>(stream))
                                 : launch_rope_append(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
  }
  return NOMAS_OK;
}

nomas_status select_common(const CacheView &src, int32_t tokens_per_frame,
                           const int32_t *frame_idx, int32_t n_frames, int32_t idx_on_device,
                           nomas_kvcache *window, int32_t *dev_err, void *stream) {
  nomas_status st = check_shape(src.heads, src.head_dim);
  if (st != NOMAS_OK) return st;
  if ((st = check_shape(window->heads, window->head_dim)) != NOMAS_OK) return st;
  if (tokens_per_frame <= 0) return fail(NOMAS_ERR_INVALID_ARG, "src tokens_per_frame <= 0");
  if (n_frames < 0) return fail(NOMAS_ERR_INVALID_ARG, "n_frames < 0");
  if (src.len < 0 || src.len > src.capacity || window->capacity < 0)
    return fail(NOMAS_ERR_INVALID_ARG, "src len/capacity inconsistent");
  const int64_t P = tokens_per_frame;
  const int64_t rows = (int64_t)n_frames * P;
  if (rows > window->capacity)
    return fail(NOMAS_ERR_CAPACITY, "window capacity %lld < %d frames x %lld rows",
                (long long)window->capacity, n_frames, (long long)P);
  if (n_frames > 0) {
    if (frame_idx == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "frame_idx is NULL");
    if (src.k == nullptr || src.v == nullptr || window->k == nullptr || window->v == nullptr ||
        !aligned16(src.k) || !aligned16(src.v) || !aligned16(window->k) || !aligned16(window->v))
      return fail(NOMAS_ERR_INVALID_ARG, "cache k/v must be non-NULL and 16-byte aligned");
    if (src.int8 && (src.k_scale == nullptr || src.v_scale == nullptr ||
                     !aligned16(src.k_scale) || !aligned16(src.v_scale)))
      return fail(NOMAS_ERR_INVALID_ARG, "cache scales must be non-NULL and 16-byte aligned");
    const int64_t sb = src.len * kRowElems * (src.int8 ? 1 : 2), wb = rows * kRowBytes;
    if (overlap(src.k, sb, window->k, wb) || overlap(src.v, sb, window->v, wb) ||
        overlap(src.k, sb, window->v, wb) || overlap(src.v, sb, window->k, wb) ||
        overlap(window->k, wb, window->v, wb))
      return fail(NOMAS_ERR_INVALID_ARG, "window overlaps the source cache");
    if (src.int8) {
      const int64_t scb = src.len * kHeads * 4;
      if (overlap(src.k_scale, scb, window->k, wb) || overlap(src.k_scale, scb, window->v, wb) ||
          overlap(src.v_scale, scb, window->k, wb) || overlap(src.v_scale, scb, window->v, wb))
        return fail(NOMAS_ERR_INVALID_ARG, "window overlaps the source scales");
    }
  }
  const int64_t n_src_frames = src.len / P;
  if (idx_on_device && n_frames > 0 && dev_err == nullptr)
    return fail(NOMAS_ERR_INVALID_ARG, "dev_err is required for a device-resident frame list");
  if (!idx_on_device) {
    for (int32_t j = 0; j < n_frames; ++j)
      if (frame_idx[j] < 0 || frame_idx[j] >= n_src_frames)
        return fail(NOMAS_ERR_INDEX, "frame_idx[%d] = %d outside [0, %lld)", j, frame_idx[j],
                    (long long)n_src_frames);
  }
  const int chunk = idx_on_device ? 65535 : kSelectHostFramesPerLaunch;
  SelectHostList hl;
  for (int32_t f0 = 0; f0 < n_frames; f0 += chunk) {
    const int32_t nf = (n_frames - f0) < chunk ? (n_frames - f0) : chunk;
    if (!idx_on_device) std::memcpy(hl.idx, frame_idx + f0, sizeof(int32_t) * nf);
    cudaError_t e;
    if (src.int8) {
      SelectI8Args a{};
      a.src_k = static_cast<const int8_t *>(src.k);
      a.src_v = static_cast<const int8_t *>(src.v);
      a.src_ks = src.k_scale;
      a.src_vs = src.v_scale;
      a.dst_k = static_cast<uint16_t *>(window->k);
      a.dst_v = static_cast<uint16_t *>(window->v);
      a.idx_dev = idx_on_device ? frame_idx : nullptr;
      a.dev_err = dev_err;
      a.tokens_per_frame = P;
      a.n_src_frames = n_src_frames;
      a.first_frame = f0;
      a.n_frames = nf;
      e = launch_select_i8(a, idx_on_device ? nullptr : &hl, static_cast<cudaStream_t>(stream));
    } else {
      SelectArgs a{};
      a.src_k = static_cast<const uint16_t *>(src.k);
      a.src_v = static_cast<const uint16_t *>(src.v);
      a.dst_k = static_cast<uint16_t *>(window->k);
      a.dst_v = static_cast<uint16_t *>(window->v);
      a.idx_dev = idx_on_device ? frame_idx : nullptr;
      a.dev_err = dev_err;
      a.frame_vecs = P * kRowVecs;
      a.n_src_frames = n_src_frames;
      a.first_frame = f0;
      a.n_frames = nf;
      e = launch_select(a, idx_on_device ? nullptr : &hl, static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) return cuda_fail(e, "select launch");
  }
  window->tokens_per_frame = tokens_per_frame;
  window->len = rows;
  return ok();
}

unsigned long long g_wait_limit_ns = 2000000000ull;  // 2 s per pipeline wait
std::atomic<int32_t> g_pipeline{0};  // process default schedule, 0: built-in

nomas_status attention_common(const void *q, int64_t n_q, const nomas_kv_span *spans,
                              int32_t n_spans, const int32_t *tile_list,
                              const int32_t *tile_count, int32_t max_tiles, void *o, float *lse,
                              float softmax_scale, int32_t heads, int32_t head_dim,
                              int32_t *dev_err, const nomas_attention_opts *opts,
                              int32_t kv_splits, void *scratch, int64_t scratch_bytes,
                              const struct OwnerRouting *routing, void *stream,
                              const nomas_kv_span_i8 *i8_span = nullptr);

// Destination of owner-routed partial outputs (see AttnArgs::n_owners).
struct OwnerRouting {
  int32_t n_owners, slot;
  const int64_t *row0;   // n_owners + 1 entries
  void *const *o;        // n_owners stacked [R][n_q][16][128] buffers
  float *const *lse;     // n_owners stacked [R][16][n_q] buffers
};

// Scratch of a key-split attention: S partial outputs [S][n_q][16][128] bf16,
// then their LSEs [S][16][n_q] fp32.
int64_t split_scratch_bytes(int64_t n_q, int32_t kv_splits) {
  return (int64_t)kv_splits * n_q * (kRowBytes + kHeads * 4);
}

}  // namespace

extern "C" {

const char *nomas_last_error(void) { return g_last_error.c_str(); }

const char *nomas_version(void) { return "nomas 0.1.0 (sm_100a)"; }

nomas_status nomas_rope3d_qk(const void *q, const void *k, void *q_out, void *k_out,
                             const nomas_seg_layout *layout, const nomas_rope3d_cfg *cfg,
                             int32_t heads, int32_t head_dim, void *stream) {
  const ApiRange nvtx_range("nomas_rope3d_qk");
  nomas_status st = check_shape(heads, head_dim);
  if (st != NOMAS_OK) return st;
  int64_t n_video = 0;
  if ((st = check_layout(layout, &n_video)) != NOMAS_OK) return st;
  RopeArgs a{};
  if ((st = fill_rope(cfg, &a)) != NOMAS_OK) return st;
  const int64_t n = n_video + layout->n_text;
  if (q == nullptr || q_out == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "q and q_out are required");
  if ((k == nullptr) != (k_out == nullptr))
    return fail(NOMAS_ERR_INVALID_ARG, "k and k_out must both be set or both be NULL");
  if (!aligned16(q) || !aligned16(q_out) || !aligned16(k) || !aligned16(k_out))
    return fail(NOMAS_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const int64_t bytes = n * kRowBytes;
  if (q_out != q && overlap(q, bytes, q_out, bytes))
    return fail(NOMAS_ERR_INVALID_ARG, "q_out partially overlaps q");
  if (k != nullptr && k_out != k && overlap(k, bytes, k_out, bytes))
    return fail(NOMAS_ERR_INVALID_ARG, "k_out partially overlaps k");
  if (k != nullptr && (overlap(q_out, bytes, k_out, bytes) || overlap(q_out, bytes, k, bytes) ||
                       overlap(k_out, bytes, q, bytes)))
    return fail(NOMAS_ERR_INVALID_ARG, "Q and K buffers overlap");
  a.q_in = static_cast<const uint16_t *>(q);
  a.q_out = static_cast<uint16_t *>(q_out);
  a.k_in = static_cast<const uint16_t *>(k);
  a.k_out = static_cast<uint16_t *>(k_out);
  a.n_q_rows = n;
  a.n_kv_rows = k != nullptr ? n : 0;
  a.n_video = n_video;
  a.grid_h = layout->grid_h;
  a.grid_w = layout->grid_w;
  a.t0 = layout->t0;
  if (n == 0) return ok();
  const cudaError_t e = launch_rope_append(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rope3d launch");
  return ok();
}

nomas_status nomas_kvcache_append(nomas_kvcache *cache, const void *k_seg, const void *v_seg,
                                  int64_t n_tokens, const void *q_in, void *q_out,
                                  const nomas_seg_layout *layout, const nomas_rope3d_cfg *cfg,
                                  void *stream) {
  const ApiRange nvtx_range("nomas_kvcache_append");
  if (cache == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "cache is NULL");
  CacheView view{cache->k, cache->v, nullptr, nullptr, cache->capacity, cache->len,
                 cache->heads, cache->head_dim, false};
  const nomas_status st =
      append_common(view, k_seg, v_seg, n_tokens, q_in, q_out, layout, cfg, stream);
  if (st != NOMAS_OK) return st;
  cache->len += n_tokens;
  return ok();
}

nomas_status nomas_kvcache_append_i8(nomas_kvcache_i8 *cache, const void *k_seg,
                                     const void *v_seg, int64_t n_tokens, const void *q_in,
                                     void *q_out, const nomas_seg_layout *layout,
                                     const nomas_rope3d_cfg *cfg, void *stream) {
  const ApiRange nvtx_range("nomas_kvcache_append_i8");
  if (cache == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "cache is NULL");
  CacheView view{cache->k, cache->v, cache->k_scale, cache->v_scale, cache->capacity,
                 cache->len, cache->heads, cache->head_dim, true};
  const nomas_status st =
      append_common(view, k_seg, v_seg, n_tokens, q_in, q_out, layout, cfg, stream);
  if (st != NOMAS_OK) return st;
  cache->len += n_tokens;
  return ok();
}

nomas_status nomas_kvcache_select(const nomas_kvcache *src, const int32_t *frame_idx,
                                  int32_t n_frames, int32_t idx_on_device, nomas_kvcache *window,
                                  int32_t *dev_err, void *stream) {
  const ApiRange nvtx_range("nomas_kvcache_select");
  if (src == nullptr || window == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "src/window is NULL");
  CacheView view{src->k, src->v, nullptr, nullptr, src->capacity, src->len,
                 src->heads, src->head_dim, false};
  return select_common(view, src->tokens_per_frame, frame_idx, n_frames, idx_on_device, window,
                       dev_err, stream);
}

nomas_status nomas_kvcache_select_i8(const nomas_kvcache_i8 *src, const int32_t *frame_idx,
                                     int32_t n_frames, int32_t idx_on_device,
                                     nomas_kvcache *window, int32_t *dev_err, void *stream) {
  const ApiRange nvtx_range("nomas_kvcache_select_i8");
  if (src == nullptr || window == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "src/window is NULL");
  CacheView view{src->k, src->v, src->k_scale, src->v_scale, src->capacity, src->len,
                 src->heads, src->head_dim, true};
  return select_common(view, src->tokens_per_frame, frame_idx, n_frames, idx_on_device, window,
                       dev_err, stream);
}

nomas_status nomas_kvcache_select_i8_codes(const nomas_kvcache_i8 *src, const int32_t *frame_idx,
                                           int32_t n_frames, int32_t idx_on_device,
                                           nomas_kvcache_i8 *window, int32_t *dev_err,
                                           void *stream) {
  const ApiRange nvtx_range("nomas_kvcache_select_i8_codes");
  if (src == nullptr || window == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "src/window is NULL");
  nomas_status st = check_shape(src->heads, src->head_dim);
  if (st != NOMAS_OK) return st;
  if ((st = check_shape(window->heads, window->head_dim)) != NOMAS_OK) return st;
  const int64_t P = src->tokens_per_frame;
  if (P <= 0) return fail(NOMAS_ERR_INVALID_ARG, "src tokens_per_frame <= 0");
  if (n_frames < 0) return fail(NOMAS_ERR_INVALID_ARG, "n_frames < 0");
  if (src->len < 0 || src->len > src->capacity || window->capacity < 0)
    return fail(NOMAS_ERR_INVALID_ARG, "src len/capacity inconsistent");
  const int64_t rows = (int64_t)n_frames * P;
  if (rows > window->capacity)
    return fail(NOMAS_ERR_CAPACITY, "window capacity %lld < %d frames x %lld rows",
                (long long)window->capacity, n_frames, (long long)P);
  if (n_frames > 0) {
    if (frame_idx == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "frame_idx is NULL");
    const void *ptrs[8] = {src->k, src->v, src->k_scale, src->v_scale,
                           window->k, window->v, window->k_scale, window->v_scale};
    for (const void *q : ptrs)
      if (q == nullptr || !aligned16(q))
        return fail(NOMAS_ERR_INVALID_ARG,
                    "INT8 caches' codes and scales must be non-NULL and 16-byte aligned");
    const int64_t scb = src->len * kRowElems, sscb = src->len * kHeads * 4;
    const int64_t wcb = rows * kRowElems, wscb = rows * kHeads * 4;
    const int64_t ssz[4] = {scb, scb, sscb, sscb}, wsz[4] = {wcb, wcb, wscb, wscb};
    for (int i = 0; i < 4; ++i)
      for (int j = 0; j < 4; ++j)
        if (overlap(ptrs[i], ssz[i], ptrs[4 + j], wsz[j]) ||
            (j > i && overlap(ptrs[4 + i], wsz[i], ptrs[4 + j], wsz[j])))
          return fail(NOMAS_ERR_INVALID_ARG, "window overlaps the source cache or itself");
  }
  const int64_t n_src_frames = src->len / P;
  if (idx_on_device && n_frames > 0 && dev_err == nullptr)
    return fail(NOMAS_ERR_INVALID_ARG, "dev_err is required for a device-resident frame list");
  if (!idx_on_device) {
    for (int32_t j = 0; j < n_frames; ++j)
      if (frame_idx[j] < 0 || frame_idx[j] >= n_src_frames)
        return fail(NOMAS_ERR_INDEX, "frame_idx[%d] = %d outside [0, %lld)", j, frame_idx[j],
                    (long long)n_src_frames);
  }
  // Codes and scales are plain byte runs per frame: the bit-copy gather of
  // the bf16 path moves them, once for the codes and once for the scales.
  const int chunk = idx_on_device ? 65535 : kSelectHostFramesPerLaunch;
  SelectHostList hl;
  for (int32_t f0 = 0; f0 < n_frames; f0 += chunk) {
    const int32_t nf = (n_frames - f0) < chunk ? (n_frames - f0) : chunk;
    if (!idx_on_device) std::memcpy(hl.idx, frame_idx + f0, sizeof(int32_t) * nf);
    for (int part = 0; part < 2; ++part) {
      SelectArgs a{};
      a.src_k = static_cast<const uint16_t *>(part == 0 ? src->k : (const void *)src->k_scale);
      a.src_v = static_cast<const uint16_t *>(part == 0 ? src->v : (const void *)src->v_scale);
      a.dst_k = static_cast<uint16_t *>(part == 0 ? window->k : (void *)window->k_scale);
      a.dst_v = static_cast<uint16_t *>(part == 0 ? window->v : (void *)window->v_scale);
      a.idx_dev = idx_on_device ? frame_idx : nullptr;
      // report a bad device index once, from the codes' launch
      a.dev_err = part == 0 ? dev_err : nullptr;
      a.frame_vecs = P * (part == 0 ? kRowElems : kHeads * 4) / 16;
      a.n_src_frames = n_src_frames;
      a.first_frame = f0;
      a.n_frames = nf;
      const cudaError_t e =
          launch_select(a, idx_on_device ? nullptr : &hl, static_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return cuda_fail(e, "select launch");
    }
  }
  window->tokens_per_frame = (int32_t)P;
  window->len = rows;
  return ok();
}

nomas_status nomas_set_attention_pipeline(int32_t pipeline) {
  if (pipeline < 0 || pipeline > NOMAS_ATTN_PIPELINE_PAIR)
    return fail(NOMAS_ERR_INVALID_ARG, "unknown attention pipeline %d", pipeline);
  g_pipeline.store(pipeline, std::memory_order_relaxed);
  return ok();
}

nomas_status nomas_segment_attention_i8(const void *q, int64_t n_q,
                                        const nomas_kv_span_i8 *history,
                                        const nomas_kv_span *spans, int32_t n_spans, void *o,
                                        float *lse, float softmax_scale, int32_t heads,
                                        int32_t head_dim, int32_t *dev_err,
                                        const nomas_attention_opts *opts, void *stream) {
  const ApiRange nvtx_range("nomas_segment_attention_i8");
  if (history == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "history is NULL");
  return attention_common(q, n_q, spans, n_spans, nullptr, nullptr, 0, o, lse, softmax_scale,
                          heads, head_dim, dev_err, opts, 1, nullptr, 0, nullptr, stream,
                          history);
}

nomas_status nomas_attention_merge(const void *o_parts, const float *lse_parts, int32_t n_parts,
                                   int64_t n_q, void *o, float *lse, int32_t heads,
                                   int32_t head_dim, void *stream) {
  const ApiRange nvtx_range("nomas_attention_merge");
  if (head_dim != kHeadDim || !(heads == 1 || heads == 2 || heads == 4 || heads == 8 ||
                                heads == kHeads))
    return fail(NOMAS_ERR_UNSUPPORTED, "heads=%d, head_dim=%d not implemented (1, 2, 4, 8 or 16 "
                "heads of 128)", heads, head_dim);
  if (n_parts <= 0 || n_q < 0 || n_q > 0x7fff0000LL)
    return fail(NOMAS_ERR_INVALID_ARG, "need n_parts >= 1 and 0 <= n_q < 2^31");
  if (n_parts > NOMAS_MAX_MERGE_PARTS)
    return fail(NOMAS_ERR_UNSUPPORTED, "n_parts %d exceeds %d", n_parts, NOMAS_MAX_MERGE_PARTS);
  if (n_q == 0) return ok();
  if (o_parts == nullptr || lse_parts == nullptr || o == nullptr || !aligned16(o_parts) ||
      !aligned16(o) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(NOMAS_ERR_INVALID_ARG, "merge pointers missing or misaligned");
  const int64_t rb = (int64_t)heads * kHeadDim * 2, lr = (int64_t)heads * 4;
  const int64_t pb = (int64_t)n_parts * n_q * rb, lb = (int64_t)n_parts * n_q * lr;
  const int64_t ob = n_q * rb, olb = n_q * lr;
  if (overlap(o, ob, o_parts, pb) || overlap(o, ob, lse_parts, lb) ||
      (lse != nullptr && (overlap(lse, olb, o_parts, pb) || overlap(lse, olb, lse_parts, lb) ||
                          overlap(lse, olb, o, ob))))
    return fail(NOMAS_ERR_INVALID_ARG, "merge outputs overlap the inputs");
  const cudaError_t e = launch_merge(static_cast<const uint16_t *>(o_parts), lse_parts, n_parts,
                                     n_q, heads, static_cast<uint16_t *>(o), lse,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

nomas_status nomas_attention_merge_peers(const void *const *o_parts, const float *const *lse_parts,
                                         int32_t n_parts, int64_t n_q, int64_t row0,
                                         int64_t n_rows, void *const *o_outs,
                                         float *const *lse_outs, int32_t n_outs, int32_t heads,
                                         int32_t head_dim, void *stream) {
  const ApiRange nvtx_range("nomas_attention_merge_peers");
  nomas_status st = check_shape(heads, head_dim);
  if (st != NOMAS_OK) return st;
  if (n_parts < 1 || n_outs < 1)
    return fail(NOMAS_ERR_INVALID_ARG, "need n_parts >= 1 and n_outs >= 1");
  if (n_parts > NOMAS_MAX_MERGE_PARTS || n_outs > NOMAS_MAX_MERGE_OUTPUTS)
    return fail(NOMAS_ERR_UNSUPPORTED, "at most %d parts and %d outputs (got %d, %d)",
                NOMAS_MAX_MERGE_PARTS, NOMAS_MAX_MERGE_OUTPUTS, n_parts, n_outs);
  if (n_q < 0 || n_q > 0x7fff0000LL || row0 < 0 || n_rows < 0 || row0 + n_rows > n_q)
    return fail(NOMAS_ERR_INVALID_ARG, "rows [%lld, %lld) outside [0, n_q = %lld)",
                (long long)row0, (long long)(row0 + n_rows), (long long)n_q);
  if (n_rows == 0) return ok();
  if (o_parts == nullptr || lse_parts == nullptr || o_outs == nullptr)
    return fail(NOMAS_ERR_INVALID_ARG, "pointer tables missing");
  const int64_t pb = n_q * kRowBytes, lb = n_q * kHeads * 4;
  for (int r = 0; r < n_parts; ++r)
    if (o_parts[r] == nullptr || lse_parts[r] == nullptr || !aligned16(o_parts[r]) ||
        (reinterpret_cast<uintptr_t>(lse_parts[r]) & 3u))
      return fail(NOMAS_ERR_INVALID_ARG, "part %d pointers missing or misaligned", r);
  for (int k = 0; k < n_outs; ++k) {
    float *lk = lse_outs != nullptr ? lse_outs[k] : nullptr;
    if (o_outs[k] == nullptr || !aligned16(o_outs[k]) || (reinterpret_cast<uintptr_t>(lk) & 3u))
      return fail(NOMAS_ERR_INVALID_ARG, "output %d pointers missing or misaligned", k);
    for (int r = 0; r < n_parts; ++r)
      if (overlap(o_outs[k], pb, o_parts[r], pb) || overlap(o_outs[k], pb, lse_parts[r], lb) ||
          overlap(lk, lb, o_parts[r], pb) || overlap(lk, lb, lse_parts[r], lb))
        return fail(NOMAS_ERR_INVALID_ARG, "output %d overlaps part %d", k, r);
  }
  const cudaError_t e = launch_merge_peers(
      reinterpret_cast<const uint16_t *const *>(o_parts), lse_parts, n_parts, n_q, row0, n_rows,
      reinterpret_cast<uint16_t *const *>(o_outs), lse_outs, n_outs,
      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "peer merge launch");
  return ok();
}

nomas_status nomas_segment_attention(const void *q, int64_t n_q, const nomas_kv_span *spans,
                                     int32_t n_spans, void *o, float *lse, float softmax_scale,
                                     int32_t heads, int32_t head_dim, int32_t *dev_err,
                                     void *stream) {
  return nomas_segment_attention_ex(q, n_q, spans, n_spans, o, lse, softmax_scale, heads, head_dim,
                                    dev_err, nullptr, stream);
}

nomas_status nomas_segment_attention_ex(const void *q, int64_t n_q, const nomas_kv_span *spans,
                                        int32_t n_spans, void *o, float *lse, float softmax_scale,
                                        int32_t heads, int32_t head_dim, int32_t *dev_err,
                                        const nomas_attention_opts *opts, void *stream) {
  const ApiRange nvtx_range("nomas_segment_attention_ex");
  return attention_common(q, n_q, spans, n_spans, nullptr, nullptr, 0, o, lse, softmax_scale,
                          heads, head_dim, dev_err, opts, 1, nullptr, 0, nullptr, stream);
}

nomas_status nomas_segment_attention_to_owners(const void *q, int64_t n_q,
                                               const nomas_kv_span *spans, int32_t n_spans,
                                               int32_t n_owners, const int64_t *owner_row0,
                                               void *const *owner_o, float *const *owner_lse,
                                               int32_t slot, float softmax_scale, int32_t heads,
                                               int32_t head_dim, int32_t *dev_err,
                                               void *stream) {
  const ApiRange nvtx_range("nomas_segment_attention_to_owners");
  if (n_owners < 1 || n_owners > NOMAS_MAX_MERGE_PARTS)
    return fail(NOMAS_ERR_INVALID_ARG, "n_owners must be in [1, %d] (got %d)",
                NOMAS_MAX_MERGE_PARTS, n_owners);
  if (slot < 0 || slot >= NOMAS_MAX_MERGE_PARTS)
    return fail(NOMAS_ERR_INVALID_ARG, "slot must be in [0, %d) (got %d)", NOMAS_MAX_MERGE_PARTS,
                slot);
  if (owner_row0 == nullptr || owner_o == nullptr || owner_lse == nullptr)
    return fail(NOMAS_ERR_INVALID_ARG, "owner tables are required");
  if (owner_row0[0] != 0 || owner_row0[n_owners] != n_q)
    return fail(NOMAS_ERR_INVALID_ARG, "owner rows must start at 0 and end at n_q");
  const int64_t part_bytes = n_q * kRowBytes, part_lse = n_q * kHeads * 4;
  for (int s = 0; s < n_owners; ++s) {
    if (owner_row0[s + 1] < owner_row0[s])
      return fail(NOMAS_ERR_INVALID_ARG, "owner rows must not decrease");
    if (owner_o[s] == nullptr || owner_lse[s] == nullptr || !aligned16(owner_o[s]) ||
        (reinterpret_cast<uintptr_t>(owner_lse[s]) & 3u))
      return fail(NOMAS_ERR_INVALID_ARG, "owner %d buffers missing or misaligned", s);
    // this rank's part of owner s's buffers must not overlap the inputs
    const void *po = static_cast<const uint8_t *>(owner_o[s]) + (int64_t)slot * part_bytes;
    const void *pl = reinterpret_cast<const uint8_t *>(owner_lse[s]) + (int64_t)slot * part_lse;
    if (overlap(po, part_bytes, q, part_bytes) || overlap(pl, part_lse, q, part_bytes))
      return fail(NOMAS_ERR_INVALID_ARG, "owner %d buffers overlap q", s);
    for (int k = 0; k < n_spans && spans != nullptr; ++k) {
      const int64_t sb = spans[k].len * kRowBytes;
      if (overlap(po, part_bytes, spans[k].k, sb) || overlap(po, part_bytes, spans[k].v, sb) ||
          overlap(pl, part_lse, spans[k].k, sb) || overlap(pl, part_lse, spans[k].v, sb))
        return fail(NOMAS_ERR_INVALID_ARG, "owner %d buffers overlap span %d", s, k);
    }
  }
  const OwnerRouting routing{n_owners, slot, owner_row0, owner_o, owner_lse};
  // o and lse name this rank's part of the first owner's buffers: only their
  // presence and alignment are checked; the kernel writes through the table.
  void *o0 = static_cast<uint8_t *>(owner_o[0]) + (int64_t)slot * part_bytes;
  float *l0 = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(owner_lse[0]) +
                                        (int64_t)slot * part_lse);
  return attention_common(q, n_q, spans, n_spans, nullptr, nullptr, 0, o0, l0, softmax_scale,
                          heads, head_dim, dev_err, nullptr, 1, nullptr, 0, &routing, stream);
}

int64_t nomas_segment_attention_scratch_bytes(int64_t n_q, int32_t kv_splits) {
  if (n_q < 0 || kv_splits < 1) return 0;
  return kv_splits > 1 ? split_scratch_bytes(n_q, kv_splits) : 0;
}

nomas_status nomas_segment_attention_split(const void *q, int64_t n_q, const nomas_kv_span *spans,
                                           int32_t n_spans, void *o, float *lse,
                                           float softmax_scale, int32_t heads, int32_t head_dim,
                                           int32_t kv_splits, void *scratch,
                                           int64_t scratch_bytes, int32_t *dev_err,
                                           void *stream) {
  const ApiRange nvtx_range("nomas_segment_attention_split");
  return attention_common(q, n_q, spans, n_spans, nullptr, nullptr, 0, o, lse, softmax_scale,
                          heads, head_dim, dev_err, nullptr, kv_splits, scratch, scratch_bytes,
                          nullptr, stream);
}

nomas_status nomas_segment_attention_sparse(const void *q, int64_t n_q,
                                            const nomas_kv_span *spans, int32_t n_spans,
                                            const int32_t *tile_list, const int32_t *tile_count,
                                            int32_t max_tiles, void *o, float *lse,
                                            float softmax_scale, int32_t heads, int32_t head_dim,
                                            int32_t *dev_err, void *stream) {
  const ApiRange nvtx_range("nomas_segment_attention_sparse");
  if (tile_list == nullptr || tile_count == nullptr)
    return fail(NOMAS_ERR_INVALID_ARG, "tile_list and tile_count are required");
  if (max_tiles < 0) return fail(NOMAS_ERR_INVALID_ARG, "max_tiles < 0");
  if (dev_err == nullptr)
    return fail(NOMAS_ERR_INVALID_ARG, "dev_err is required with a device-resident tile list");
  if ((reinterpret_cast<uintptr_t>(tile_list) & 3u) || (reinterpret_cast<uintptr_t>(tile_count) & 3u))
    return fail(NOMAS_ERR_INVALID_ARG, "tile_list and tile_count must be 4-byte aligned");
  return attention_common(q, n_q, spans, n_spans, tile_list, tile_count, max_tiles, o, lse,
                          softmax_scale, heads, head_dim, dev_err, nullptr, 1, nullptr, 0,
                          nullptr, stream);
}

}  // extern "C"

namespace {

nomas_status attention_common(const void *q, int64_t n_q, const nomas_kv_span *spans,
                              int32_t n_spans, const int32_t *tile_list,
                              const int32_t *tile_count, int32_t max_tiles, void *o, float *lse,
                              float softmax_scale, int32_t heads, int32_t head_dim,
                              int32_t *dev_err, const nomas_attention_opts *opts,
                              int32_t kv_splits, void *scratch, int64_t scratch_bytes,
                              const OwnerRouting *routing, void *stream,
                              const nomas_kv_span_i8 *i8_span) {
  // Heads per row: 16, or for a dense bf16 call without routed outputs 1, 2,
  // 4 or 8 (the local heads of a head-sharded layout).
  const bool few_heads_ok = (i8_span == nullptr || i8_span->len == 0) && tile_list == nullptr &&
                            routing == nullptr;
  if (head_dim != kHeadDim ||
      !(heads == kHeads || (few_heads_ok && (heads == 1 || heads == 2 || heads == 4 || heads == 8))))
    return fail(NOMAS_ERR_UNSUPPORTED,
                "heads=%d, head_dim=%d not implemented (16 heads of 128; 1, 2, 4 or 8 heads for "
                "dense bf16 calls)", heads, head_dim);
  nomas_status st = NOMAS_OK;
  // Bytes of one row of Q, K, V or O, and of one query's LSE values.
  const int64_t row_bytes = (int64_t)heads * kHeadDim * 2, lse_row = (int64_t)heads * 4;
  const bool i8 = i8_span != nullptr && i8_span->len != 0;
  // Kernel schedule: the call's, else the process default, else the built-in
  // choice; the one-tile and pair schedules take dense bf16 keys only.
  // The process default applies to dense bf16 calls; a schedule named in the
  // call's options must fit the call.
  const bool dense_bf16 = !i8 && tile_list == nullptr;
  int32_t pipeline = dense_bf16 ? g_pipeline.load(std::memory_order_relaxed) : 0;
  if (opts != nullptr && opts->pipeline != 0) pipeline = opts->pipeline;
  if (pipeline < 0 || pipeline > NOMAS_ATTN_PIPELINE_PAIR)
    return fail(NOMAS_ERR_INVALID_ARG, "unknown attention pipeline %d", pipeline);
  if (pipeline == 0) pipeline = dense_bf16 ? NOMAS_ATTN_PIPELINE_DEFAULT_DENSE : NOMAS_ATTN_PIPELINE_TWO_TILE;
  if (pipeline != NOMAS_ATTN_PIPELINE_TWO_TILE && !dense_bf16)
    return fail(NOMAS_ERR_UNSUPPORTED,
                "the one-tile and pair attention schedules take dense bf16 keys only");
  const uint32_t kv_box_rows = pipeline == NOMAS_ATTN_PIPELINE_PAIR ? 64u : 128u;
  if (i8_span != nullptr && (i8_span->len < 0 || i8_span->len > 0x7fff0000LL))
    return fail(NOMAS_ERR_INVALID_ARG, "INT8 history length out of range");
  if (i8 && (n_spans + 1 > kMaxSpans))
    return fail(NOMAS_ERR_UNSUPPORTED, "at most %d key/value spans with the INT8 history (got %d)",
                kMaxSpans - 1, n_spans);
  if (kv_splits < 1 || kv_splits > NOMAS_MAX_MERGE_PARTS)
    return fail(NOMAS_ERR_INVALID_ARG, "kv_splits must be in [1, %d] (got %d)",
                NOMAS_MAX_MERGE_PARTS, kv_splits);
  if (n_spans < 0) return fail(NOMAS_ERR_INVALID_ARG, "n_spans < 0");
  if (n_spans > kMaxSpans)
    return fail(NOMAS_ERR_UNSUPPORTED, "at most %d key/value spans (got %d)", kMaxSpans, n_spans);
  if (n_spans > 0 && spans == nullptr) return fail(NOMAS_ERR_INVALID_ARG, "spans is NULL");
  if (n_q < 0 || n_q > 0x7fff0000LL) return fail(NOMAS_ERR_INVALID_ARG, "n_q out of range");
  if (n_q == 0) return ok();
  if (q == nullptr || o == nullptr || !aligned16(q) || !aligned16(o))
    return fail(NOMAS_ERR_INVALID_ARG, "q and o must be non-NULL and 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return fail(NOMAS_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(NOMAS_ERR_INVALID_ARG, "softmax_scale not finite");
  const int64_t qb = n_q * row_bytes;
  if (overlap(q, qb, o, qb)) return fail(NOMAS_ERR_INVALID_ARG, "o overlaps q");
  if (lse != nullptr && (overlap(lse, n_q * lse_row, o, qb) || overlap(lse, n_q * lse_row, q, qb)))
    return fail(NOMAS_ERR_INVALID_ARG, "lse overlaps q or o");
  const int64_t sb = kv_splits > 1 ? split_scratch_bytes(n_q, kv_splits) : 0;
  if (kv_splits > 1) {
    if (scratch == nullptr || !aligned16(scratch))
      return fail(NOMAS_ERR_INVALID_ARG, "scratch must be non-NULL and 16-byte aligned");
    if (scratch_bytes < sb)
      return fail(NOMAS_ERR_CAPACITY, "scratch of %lld bytes, %lld needed", (long long)scratch_bytes,
                  (long long)sb);
    if (overlap(scratch, sb, q, qb) || overlap(scratch, sb, o, qb) ||
        (lse != nullptr && overlap(scratch, sb, lse, n_q * lse_row)))
      return fail(NOMAS_ERR_INVALID_ARG, "scratch overlaps q, o or lse");
  }
  AttnArgs a{};
  int n_used = 0;
  if (i8) {
    // span 0: the INT8 history (codes through TMA, scales read by the kernel)
    const nomas_kv_span_i8 &h = *i8_span;
    if (h.k == nullptr || h.v == nullptr || h.k_scale == nullptr || h.v_scale == nullptr ||
        !aligned16(h.k) || !aligned16(h.v) || !aligned16(h.k_scale) || !aligned16(h.v_scale))
      return fail(NOMAS_ERR_INVALID_ARG,
                  "INT8 history codes and scales must be non-NULL and 16-byte aligned");
    const int64_t cb = h.len * kRowElems, scb = h.len * kHeads * 4;
    const void *parts[4] = {h.k, h.v, h.k_scale, h.v_scale};
    const int64_t sizes[4] = {cb, cb, scb, scb};
    for (int i = 0; i < 4; ++i)
      if (overlap(parts[i], sizes[i], o, qb) ||
          (lse != nullptr && overlap(parts[i], sizes[i], lse, n_q * lse_row)) ||
          overlap(parts[i], sizes[i], scratch, sb))
        return fail(NOMAS_ERR_INVALID_ARG, "INT8 history overlaps an output or the scratch");
    if ((st = codes_map(&a.tmap_k[0], h.k, h.len)) != NOMAS_OK) return st;
    if ((st = codes_map(&a.tmap_v[0], h.v, h.len)) != NOMAS_OK) return st;
    a.span_len[0] = h.len;
    a.tile_base[1] = (int32_t)((h.len + 127) / 128);
    a.i8 = 1;
    a.i8_scale[0] = h.k_scale;
    a.i8_scale[1] = h.v_scale;
    n_used = 1;
  }
  for (int s = 0; s < n_spans; ++s) {
    const nomas_kv_span &sp = spans[s];
    if (sp.len < 0 || sp.len > 0x7fff0000LL)
      return fail(NOMAS_ERR_INVALID_ARG, "span %d length out of range", s);
    if (sp.len == 0) continue;
    if (sp.k == nullptr || sp.v == nullptr || !aligned16(sp.k) || !aligned16(sp.v))
      return fail(NOMAS_ERR_INVALID_ARG, "span %d k/v must be non-NULL and 16-byte aligned", s);
    const int64_t sbytes = sp.len * row_bytes;
    if (overlap(sp.k, sbytes, o, qb) || overlap(sp.v, sbytes, o, qb) ||
        (lse != nullptr && (overlap(sp.k, sbytes, lse, n_q * lse_row) ||
                            overlap(sp.v, sbytes, lse, n_q * lse_row))) ||
        overlap(sp.k, sbytes, scratch, sb) || overlap(sp.v, sbytes, scratch, sb))
      return fail(NOMAS_ERR_INVALID_ARG, "span %d overlaps an output or the scratch", s);
    if ((st = rows_map(&a.tmap_k[n_used], sp.k, sp.len, kv_box_rows, heads)) != NOMAS_OK) return st;
    if ((st = rows_map(&a.tmap_v[n_used], sp.v, sp.len, kv_box_rows, heads)) != NOMAS_OK) return st;
    a.span_len[n_used] = sp.len;
    a.tile_base[n_used + 1] = a.tile_base[n_used] + (int32_t)((sp.len + 127) / 128);
    ++n_used;
  }
  a.tile_list = tile_list;
  a.tile_count = tile_count;
  a.max_tiles = max_tiles;
  if (n_used == 0) {
    if (routing != nullptr) {
      // no keys: O = 0, LSE = -inf in this rank's part of every owner's buffers
      for (int s = 0; s < routing->n_owners; ++s) {
        const cudaError_t e = launch_attention_empty(
            static_cast<uint16_t *>(routing->o[s]) + (int64_t)routing->slot * n_q * kRowElems,
            routing->lse[s] + (int64_t)routing->slot * kHeads * n_q, n_q, kHeads,
            static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "attention (no keys) launch");
      }
      return ok();
    }
    const cudaError_t e = launch_attention_empty(static_cast<uint16_t *>(o), lse, n_q, heads,
                                                 static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "attention (no keys) launch");
    return ok();
  }
  if ((st = rows_map(&a.tmap_q, q, n_q, 128, heads)) != NOMAS_OK) return st;
  a.heads = heads;
  const double scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)kHeadDim);
  a.scale_log2 = (float)(scale * 1.4426950408889634);
  a.n_spans = n_used;
  a.n_q = (int32_t)n_q;
  a.o = static_cast<uint16_t *>(o);
  a.lse = lse;
  a.kv_splits = 1;
  a.n_owners = 0;
  if (routing != nullptr) {
    a.n_owners = routing->n_owners;
    a.owner_slot = routing->slot;
    for (int s = 0; s <= routing->n_owners; ++s) a.owner_row0[s] = routing->row0[s];
    for (int s = 0; s < routing->n_owners; ++s) {
      a.owner_o[s] = static_cast<uint16_t *>(routing->o[s]);
      a.owner_lse[s] = routing->lse[s];
    }
  }
  uint16_t *part_o = nullptr;
  float *part_lse = nullptr;
  if (kv_splits > 1) {
    // Partial results of the S key ranges go to the scratch, then one merge
    // writes o and lse.
    part_o = static_cast<uint16_t *>(scratch);
    part_lse = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) +
                                         (int64_t)kv_splits * n_q * kRowBytes);
    a.o = part_o;
    a.lse = part_lse;
    a.kv_splits = kv_splits;
  }
  a.dev_err = dev_err;
  a.wait_limit_ns = g_wait_limit_ns;
  a.testing_skip_load = -1;
  if (opts != nullptr) {
    if (opts->wait_limit_ns > 0) a.wait_limit_ns = opts->wait_limit_ns;
    if (opts->testing_skip_kv_load < -1)
      return fail(NOMAS_ERR_INVALID_ARG, "testing_skip_kv_load must be >= -1");
    a.testing_skip_load = opts->testing_skip_kv_load;
  }
  cudaError_t e =
      pipeline == NOMAS_ATTN_PIPELINE_TWO_TILE
          ? launch_attention(a, static_cast<cudaStream_t>(stream))
          : launch_attention_pair(a, pipeline == NOMAS_ATTN_PIPELINE_PAIR,
                                  static_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidKernelImage && a.i8)
    return fail(NOMAS_ERR_CUDA, "INT8 attention kernel not compiled to %d registers per thread at "
                "launch; refusing to run its register split", 128);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  if (kv_splits > 1) {
    e = launch_merge(part_o, part_lse, kv_splits, n_q, heads, static_cast<uint16_t *>(o), lse,
                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "merge of key splits launch");
  }
  return ok();
}

}  // namespace

// Records a failure from another source file of the library in the same
// per-thread message that nomas_last_error() returns.
nomas_status nomas::report_error(nomas_status st, const char *message) {
  return fail(st, "%s", message);
}
