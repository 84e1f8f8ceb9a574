// decode_noalloc.cu - sparse decode attention for callers that cannot allocate device memory.
//
// mustafar_decode_attn needs a caller-provided workspace when it splits the context across
// CTAs (per-split partial softmax states plus one ticket counter per (batch row, kv head)).
// Some callers have no way to provide one: serving engines that reserve all device memory
// up front and hand kernels only their input and output buffers, plugin interfaces of a host
// framework that owns the allocator, or code paths where a cudaMalloc would synchronise the
// device.  This entry point keeps that workspace in a fixed-size array in the library's own
// device memory instead, so a call allocates nothing.
#include <cstdio>
#include <cstring>

#include "internal.h"

namespace mustafar {
namespace {

// Split-K scratch for mustafar_decode_attn_noalloc.  Every GPU that loads the library holds
// these bytes until the process exits.  Host code must not pass this symbol to a kernel: on the
// host it is only a stand-in, so its device address is looked up below.
static __device__ __align__(256) uint8_t g_decode_scratch[MUSTAFAR_NOALLOC_SCRATCH_BYTES];

// Device address of g_decode_scratch in the current device's context.  Looked up on every call
// (a cheap host query once the module is loaded) rather than cached, so that a context created
// again after cudaDeviceReset is never handed an address from the one before it.
cudaError_t scratch_address(void **out) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace mustafar

extern "C" mustafar_status mustafar_decode_attn_noalloc(const void *q, int32_t num_q_heads, const mustafar_cache_t *k,
                                                        const mustafar_cache_t *v, const int32_t *d_seq_len,
                                                        int32_t max_len, float scale, void *out, float *lse,
                                                        int32_t num_splits, uint32_t *d_err,
                                                        mustafar_stream_t stream) {
  void *scratch = nullptr;
  cudaError_t e = mustafar::scratch_address(&scratch);
  if (e != cudaSuccess) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "decode_attn_noalloc: device address of the scratch array: %s",
                  cudaGetErrorString(e));
    mustafar::set_last_error(msg);
    return MUSTAFAR_ERR_CUDA;
  }
  if (k != nullptr && k->batch > 0 && k->num_kv_heads > 0) {
    // the ticket counters at the start of the scratch must read zero when the kernel starts;
    // earlier calls leave them at zero, but a call that failed part-way may not have
    const size_t counters = ((static_cast<size_t>(k->batch) * k->num_kv_heads * 4 + 255) / 256) * 256;
    if (counters <= MUSTAFAR_NOALLOC_SCRATCH_BYTES) {
      e = cudaMemsetAsync(scratch, 0, counters, reinterpret_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) {
        mustafar::set_last_error("decode_attn_noalloc: clearing the scratch ticket counters failed");
        return MUSTAFAR_ERR_CUDA;
      }
    }
  }
  const mustafar_status s = mustafar_decode_attn(q, num_q_heads, k, v, d_seq_len, max_len, scale, out, lse, scratch,
                                                 MUSTAFAR_NOALLOC_SCRATCH_BYTES, num_splits, d_err, stream);
  if (s == MUSTAFAR_ERR_WORKSPACE) {
    char msg[512];
    std::snprintf(msg, sizeof(msg),
                  "decode_attn_noalloc: this shape and split count need more split-K scratch than the library's "
                  "fixed %u bytes (%s); use fewer splits, or mustafar_decode_attn with a caller workspace",
                  static_cast<unsigned>(MUSTAFAR_NOALLOC_SCRATCH_BYTES), mustafar_last_error());
    mustafar::set_last_error(msg);
  }
  return s;
}
