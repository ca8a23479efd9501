// kv4_decode_attention_noalloc: the decode attention of kv4_decode_attention for callers
// that cannot allocate device memory -- code that runs where cudaMalloc is unavailable
// or forbidden (inside a memory pool that must not grow, a real-time loop that may not
// call the allocator, an embedding runtime that owns all device memory) and therefore
// cannot supply a workspace. The scratch space lives in a fixed-size array in this
// library's device image instead; the caller still passes every input and output.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/kv4.h"
#include "kv4_device.cuh"
#include "kv4_internal.h"

namespace {

// Scratch for the work list and the partial softmax states of one call. Every GPU that
// loads the library holds these bytes until the process exits.
constexpr size_t kStaticScratchBytes = KV4_NOALLOC_SCRATCH_BYTES;  // 32 MiB, see kv4.h
__device__ __align__(256) unsigned char kv4_static_scratch[kStaticScratchBytes];

// Device address of the array, looked up once per device. In host code the array's
// name is only a stand-in, never a device address, so kernels get the looked-up pointer.
// The address belongs to the device's primary context as it was at the first call: after
// cudaDeviceReset (a new primary context) it is stale, which kv4.h states as a limit.
constexpr int kMaxDevices = 64;
void *g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mutex;

cudaError_t scratch_for_current_device(void **ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, kv4_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch[dev] = p;
  }
  *ptr = g_scratch[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t kv4_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

kv4_status kv4_decode_attention_noalloc(const kv4_config *cfg, const kv4_int4_pool *pool,
                                        const kv4_int8_side *side, const kv4_batch *batch,
                                        const void *q, void *out, float *out_f32, float *lse,
                                        int32_t *err_flag, kv4_stream_t stream) {
  // The argument checks, the size of the work and the refusal of a batch too large for
  // the array (after the fall-back to 64-page chunks) are kv4_decode_attention's own,
  // given the array as a workspace of kStaticScratchBytes.
  if (cfg == nullptr || batch == nullptr) return KV4_ERR_INVALID_ARG;
  void *scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return KV4_ERR_CUDA;
  return kv4_decode_attention(cfg, pool, side, batch, q, out, out_f32, lse, scratch,
                              kStaticScratchBytes, err_flag, stream);
}

}  // extern "C"
