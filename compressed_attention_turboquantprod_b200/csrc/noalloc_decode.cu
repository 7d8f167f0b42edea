// tq_decode_attention_noalloc: decode attention whose scratch lives in a
// statically allocated device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory or hand the library
// a scratch buffer, e.g. a plugin inside an inference engine whose host
// framework owns every device allocation and offers plugins no workspace, or a
// process whose device memory is fully reserved up front by another allocator.
//
// The scratch array is a file-scope __device__ object: every GPU on which this
// library is loaded holds TQ_NOALLOC_SCRATCH_BYTES for it until the process
// exits.  Host code cannot use the array's name as a device address (it names a
// host-side shadow), so the device address is looked up once per device with
// cudaGetSymbolAddress while that device is current, and cached.
#include <mutex>

#include "tq_internal.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

namespace tq {
// Device address of the scratch array on the current device (set up on first use).
int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::set_error(TQ_ERR_CUDA, "tq_decode_attention_noalloc: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return tq::set_error(TQ_ERR_UNSUPPORTED, "tq_decode_attention_noalloc: device index out of range");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return tq::set_error(TQ_ERR_CUDA, "tq_decode_attention_noalloc: cudaGetSymbolAddress failed");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TQ_OK;
}
}  // namespace tq

extern "C" int tq_decode_attention_noalloc(const tq_cache* c, const void* Q, int Hq,
                                           float softmax_scale, const float* Pi, const float* S,
                                           const float* centroids, void* out, float* logits,
                                           int num_splits, void* stream) {
  // Scratch the decode needs with these arguments and the cache's current length,
  // from the split count the decode itself takes (0 when the arguments are
  // invalid: tq_decode_attention below then reports why).
  const size_t need = tq::decode_ws_bytes_now(c, Hq, num_splits);
  if (need > (size_t)TQ_NOALLOC_SCRATCH_BYTES)
    return tq::set_error(TQ_ERR_UNSUPPORTED,
                         "tq_decode_attention_noalloc: needs %zu bytes of scratch, more than the "
                         "static maximum of %zu bytes (use tq_decode_attention with a workspace)",
                         need, (size_t)TQ_NOALLOC_SCRATCH_BYTES);
  void* ws = nullptr;
  int st = tq::noalloc_scratch(&ws);
  if (st != TQ_OK) return st;
  return tq_decode_attention(c, Q, Hq, softmax_scale, Pi, S, centroids, out, logits, num_splits,
                             ws, (size_t)TQ_NOALLOC_SCRATCH_BYTES, stream);
}
