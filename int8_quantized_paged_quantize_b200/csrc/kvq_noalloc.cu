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
// array's name as a device address, so the address is fetched with
// cudaGetSymbolAddress, with the device current, the first time a call runs on
// a device, and cached. The cache is keyed by the device's context as well: if
// the context was destroyed and made again (cudaDeviceReset), the module is
// loaded again, the array may move, and the next call looks the address up
// anew instead of writing through a stale pointer. Make the first call on a
// device before any stream capture. All calls share the one array and it keeps
// the previous call's contents: nothing in it must start at zero (every chunk
// partial the merge reads is written by the same call first), but two calls
// whose kernels overlap on the GPU (different streams, or different host
// threads) race on it and must be serialised by the caller.

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kvq_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct ScratchEntry {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;
};

std::mutex g_mu;
ScratchEntry g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current context (0 if none is current or the driver
// cannot tell): two contexts made one after the other on a device never share
// an id, so a change of id means the module, and the array, were loaded anew.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) !=
            cudaSuccess || q != cudaDriverEntryPointSuccess)
      fn = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(fn);
  }();
  static CtxGetIdFn get_id = [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) !=
            cudaSuccess || q != cudaDriverEntryPointSuccess)
      fn = nullptr;
    return reinterpret_cast<CtxGetIdFn>(fn);
  }();
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device: looked up once
// per device and context; without a context id (an old driver) on every call.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchEntry& e = g_scratch[dev];
  unsigned long long id = current_context_id();
  if (e.ptr == nullptr || id == 0 || id != e.ctx_id) {
    void* p = nullptr;
    // also makes the device's primary context current if none was
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return KVQ_ERR_CUDA;
    if (id == 0) id = current_context_id();
    e.ptr = p;
    e.ctx_id = id;
  }
  *out = e.ptr;
  return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attn_noalloc(const void* q, int32_t batch, const void* k_cache,
                                       const void* v_cache, const void* const* scales,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       int32_t max_context_len, float sm_scale, void* out,
                                       kvq_out_dtype out_dtype, int32_t partition_tokens,
                                       kvq_fmt fmt, const kvq_dims* dims, kvq_stream_t stream) {
  // every check, the size against the array included, runs before anything
  // touches a device, with the results kvq_decode_attn gives
  kvq::DecodePlan plan;
  int rc = kvq::check_decode_common(batch, max_context_len, partition_tokens, fmt, dims, &plan);
  if (rc != KVQ_OK) return rc;
  if (out_dtype != KVQ_OUT_BF16 && out_dtype != KVQ_OUT_F32) return KVQ_ERR_ARG;
  if (plan.total > size_t(KVQ_NOALLOC_SCRATCH_BYTES)) return KVQ_ERR_WORKSPACE;
  if (batch == 0) return KVQ_OK;
  const void *ks, *vs;
  rc = kvq::check_decode_inputs(q, k_cache, v_cache, scales, block_tables, context_lens, sm_scale,
                                fmt, &ks, &vs);
  if (rc != KVQ_OK) return rc;
  if (out == nullptr || (reinterpret_cast<uintptr_t>(out) & 15u) != 0) return KVQ_ERR_ARG;
  void* scratch = nullptr;
  rc = scratch_for_current_device(&scratch);
  if (rc != KVQ_OK) return rc;
  return kvq_decode_attn(q, batch, k_cache, v_cache, scales, block_tables, context_lens,
                         max_context_len, sm_scale, out, out_dtype, scratch,
                         size_t(KVQ_NOALLOC_SCRATCH_BYTES), partition_tokens, fmt, dims, stream);
}
