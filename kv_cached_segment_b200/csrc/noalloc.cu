// Key-split attention whose scratch is a fixed array inside the library, for
// callers that cannot allocate device memory.
//
// Who needs it: a caller whose device memory is fully reserved up front (a
// serving process that claims its whole budget at start and hands out only
// its own pools), or a host framework that owns the device allocator and
// forbids allocations made behind its back, or a latency-critical loop where
// cudaMalloc / cudaFree, which can synchronise the device, are not allowed.
// nomas_segment_attention_split needs caller-provided scratch; this entry
// point takes none and uses the array below instead.
//
// The array lives in device memory of every GPU on which this entry point
// is used (with lazy module loading, from its first call on that device; with
// eager loading, from library load) until the process exits.  Every call
// shares it: calls that overlap on the GPU (two streams, or two host threads)
// race on it and must be serialised by the caller.  Each call overwrites
// every byte it reads (each partial output row and LSE is written by its CTA
// before the merge reads it; a CTA whose pipeline wait ran out writes NaN
// rows, which the merge turns into NaN output rows), so nothing has to start
// at zero and no earlier call's contents can reach an output.
//
// The array's device address is asked of the runtime (cudaGetSymbolAddress,
// with the device current) on every call made outside stream capture, and
// kept per device.  A call made while its stream is capturing uses the kept
// address instead, since the lookup may load the module, which capture does
// not allow: make one call on the device before capturing, and another after
// the device's primary context has been reset (cudaDeviceReset), which moves
// the array.
#include <cstdio>
#include <mutex>

#include "nomas.h"
#include "nomas_internal.h"

namespace {

// The scratch: partial O rows and LSEs of the key ranges.
static __device__ __align__(256) uint8_t g_split_scratch[NOMAS_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_split_scratch on each device.  In host code the name
// g_split_scratch is only a host-side stand-in for the symbol, never a
// device pointer, so the address is asked of the runtime once per device,
// with that device current.
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// True unless `stream` is known not to be capturing.  Asking about the legacy
// stream while another stream captures in global mode is itself an error;
// that counts as capturing.
bool maybe_capturing(cudaStream_t stream) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &st) != cudaSuccess) {
    (void)cudaGetLastError();
    return true;
  }
  return st != cudaStreamCaptureStatusNone;
}

cudaError_t scratch_address(cudaStream_t stream, void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!maybe_capturing(stream)) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_split_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  if (g_scratch_ptr[dev] == nullptr) return cudaErrorStreamCaptureUnsupported;
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" nomas_status nomas_segment_attention_split_noalloc(
    const void *q, int64_t n_q, const nomas_kv_span *spans, int32_t n_spans, void *o, float *lse,
    float softmax_scale, int32_t heads, int32_t head_dim, int32_t kv_splits, int32_t *dev_err,
    void *stream) {
  const int64_t need = nomas_segment_attention_scratch_bytes(n_q, kv_splits);
  if (need > (int64_t)NOMAS_NOALLOC_SCRATCH_BYTES) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "%d key splits of %lld query rows need %lld bytes of scratch; the built-in "
             "array holds %lld (use fewer splits or nomas_segment_attention_split)",
             kv_splits, (long long)n_q, (long long)need, (long long)NOMAS_NOALLOC_SCRATCH_BYTES);
    return nomas::report_error(NOMAS_ERR_CAPACITY, msg);
  }
  void *scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (e != cudaSuccess) {
      char msg[240];
      snprintf(msg, sizeof(msg),
               e == cudaErrorStreamCaptureUnsupported
                   ? "device address of the built-in scratch array: not known yet on this "
                     "device and the stream is capturing (make one call before capture)"
                   : "device address of the built-in scratch array: %s",
               cudaGetErrorString(e));
      return nomas::report_error(NOMAS_ERR_CUDA, msg);
    }
  }
  return nomas_segment_attention_split(q, n_q, spans, n_spans, o, lse, softmax_scale, heads,
                                       head_dim, kv_splits, scratch,
                                       (int64_t)NOMAS_NOALLOC_SCRATCH_BYTES, dev_err, stream);
}
