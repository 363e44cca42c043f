// kvq_decode_attn_noalloc: paged decode attention for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the time
// they run decode: a plugin running inside another framework's step, where
// that framework owns every device byte and forbids allocation mid-step; or a
// latency-critical decode loop that must never hit the implicit device
// synchronisation cudaMalloc/cudaFree can cause. kvq_decode_attn needs a
// caller-provided workspace for its split-K partials; this entry point takes
// that scratch from a fixed array compiled into the library instead, so the
// caller passes only inputs and outputs.
//
// The scratch is a file-scope static __device__ array of
// KVQ_NOALLOC_SCRATCH_BYTES (64 MiB). Every GPU on which the library's code is
// loaded holds those bytes until the process exits. Host code cannot use the
// array's name as a device address, so on the first call on each device (with
// that device current) the address is fetched once with cudaGetSymbolAddress
// and cached; make that first call before any stream capture. All calls share
// the one array and it keeps the previous call's contents: nothing in it must
// start at zero (every chunk partial the merge reads is written by the same
// call first), but two calls whose kernels overlap on the GPU (different
// streams, or different host threads) race on it and must be serialised by the
// caller.

#include <cuda_runtime.h>

#include <mutex>

#include "kvq_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attn_noalloc(const void* q, int32_t batch, const void* k_cache,
                                       const void* v_cache, const void* const* scales,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       int32_t max_context_len, float sm_scale, void* out,
                                       kvq_out_dtype out_dtype, int32_t partition_tokens,
                                       kvq_fmt fmt, const kvq_dims* dims, kvq_stream_t stream) {
  // the size check runs before anything touches a device
  const size_t need = kvq_decode_workspace_bytes(batch, max_context_len, partition_tokens, fmt, dims);
  if (need == 0 && batch != 0) return kvq::check_dims(dims) == KVQ_OK ? KVQ_ERR_ARG : kvq::check_dims(dims);
  if (need > size_t(KVQ_NOALLOC_SCRATCH_BYTES)) return KVQ_ERR_WORKSPACE;
  if (batch == 0) return KVQ_OK;
  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != KVQ_OK) return rc;
  return kvq_decode_attn(q, batch, k_cache, v_cache, scales, block_tables, context_lens,
                         max_context_len, sm_scale, out, out_dtype, scratch,
                         size_t(KVQ_NOALLOC_SCRATCH_BYTES), partition_tokens, fmt, dims, stream);
}
