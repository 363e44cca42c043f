// C ABI of libkvq: host-side argument checks, the split-K plan, and dispatch to
// the CUDA kernels in kvq_kernels.cu. See include/kvq.h for the contract.

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "kvq_internal.h"

namespace kvq {

namespace {
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dev_ok(const void* p) { return p != nullptr && aligned16(p); }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }
int cuda_rc(int e) { return e == 0 ? KVQ_OK : KVQ_ERR_CUDA; }
}  // namespace

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // clear a sticky "no device" error from the query
    return 148;
  }
  return n;
}

// Split-K chunking. A chunk is a whole number of 128-token tiles; it is the
// smallest run of one sequence's tiles a decode CTA takes, so a (sequence, KV
// head) yields at most ceil(max_ctx / chunk) + 1 partials (the workspace
// slots). Automatic choice: the smallest chunk that cuts the longest sequence
// into at most 15 runs. The persistent decode kernel then spreads any batch
// over every resident CTA while the workspace stays at 16 partials per row.
int make_plan(int32_t batch, int32_t max_ctx, int32_t partition_tokens, const kvq_dims* d,
              DecodePlan* plan, int32_t n_query) {
  if (batch < 0 || max_ctx < 0 || partition_tokens < 0) return KVQ_ERR_ARG;
  if (partition_tokens % kTileTokens != 0) return KVQ_ERR_ARG;
  int64_t part = partition_tokens;
  if (part == 0) {
    const int64_t tiles = std::max<int64_t>(1, (int64_t(max_ctx) + kTileTokens - 1) / kTileTokens);
    part = int64_t(kTileTokens) * ((tiles + 14) / 15);
  }
  const int64_t splits = std::max<int64_t>(1, (int64_t(max_ctx) + part - 1) / part);
  plan->partition = int32_t(part);
  plan->max_splits = int32_t(splits);
  plan->slots = int32_t(splits + 1);
  int gp = 1;
  const int groups = row_groups(d->n_q_heads / d->n_kv_heads * n_query, &gp);
  const size_t rows = size_t(batch) * d->n_q_heads * size_t(n_query) * size_t(plan->slots);
  plan->o_bytes = round256(rows * d->head_dim * sizeof(float));
  plan->ml_bytes = round256(rows * 2 * sizeof(float));
  // partial counts: one per (sequence, row group) for the decode kernel, one
  // per query row for the prefill kernel
  const size_t counts = std::max(size_t(batch) * d->n_kv_heads * size_t(groups),
                                 size_t(batch) * d->n_q_heads * size_t(n_query));
  plan->cnt_bytes = round256(counts * sizeof(int32_t));
  plan->total = plan->o_bytes + plan->ml_bytes + plan->cnt_bytes;
  return KVQ_OK;
}

namespace {
constexpr long long kDefaultWaitLimit = 2000000000LL;   // about one second of SM clock
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};
}  // namespace

long long decode_wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

int check_decode_common(int32_t batch, int32_t max_ctx, int32_t partition_tokens, kvq_fmt fmt,
                        const kvq_dims* dims, DecodePlan* plan, int32_t n_query) {
  if (!fmt_valid(fmt)) return KVQ_ERR_ARG;
  int rc = check_dims(dims);
  if (rc != KVQ_OK) return rc;
  if (batch < 0 || max_ctx < 0 || n_query < 1) return KVQ_ERR_ARG;
  if (int64_t(max_ctx) > int64_t(dims->max_blocks_per_seq) * dims->block_size) return KVQ_ERR_ARG;
  return make_plan(batch, max_ctx, partition_tokens, dims, plan, n_query);
}

int check_decode_inputs(const void* q, const void* kc, const void* vc, const void* const* scales,
                        const int32_t* tables, const int32_t* ctx, float sm_scale, kvq_fmt fmt,
                        const void** ks, const void** vs) {
  if (!dev_ok(q) || !dev_ok(kc) || !dev_ok(vc) || !dev_ok(tables) || !dev_ok(ctx))
    return KVQ_ERR_ARG;
  if (!std::isfinite(sm_scale)) return KVQ_ERR_ARG;
  *ks = *vs = nullptr;
  if (fmt != KVQ_BF16) {
    if (!scales || !dev_ok(scales[0]) || !dev_ok(scales[1])) return KVQ_ERR_ARG;
    *ks = scales[0];
    *vs = scales[1];
  }
  return KVQ_OK;
}

}  // namespace kvq

using namespace kvq;

extern "C" {

int kvq_version(void) { return 100; }

const char* kvq_status_string(int status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_ARG: return "invalid argument (null or misaligned pointer, bad size or enum)";
    case KVQ_ERR_UNSUPPORTED: return "unsupported shape (block_size 16, head_dim 64/128, GQA group 1/2/4/8)";
    case KVQ_ERR_WORKSPACE: return "decode workspace too small";
    case KVQ_ERR_CUDA: return "CUDA launch or call failed";
    case KVQ_ERR_POOL_EXHAUSTED: return "block pool exhausted";
    case KVQ_ERR_DEVICE: return "a kernel flagged a data fault (see kvq_device_error)";
    default: return "unknown status";
  }
}

int kvq_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
               void* k_cache, void* v_cache, void* k_scale, void* v_scale, kvq_fmt fmt,
               const kvq_dims* dims, kvq_stream_t stream) {
  if (!fmt_valid(fmt) || num_tokens < 0) return KVQ_ERR_ARG;
  int rc = check_dims(dims);
  if (rc != KVQ_OK) return rc;
  if (num_tokens == 0) return KVQ_OK;
  if (!dev_ok(k) || !dev_ok(v) || !dev_ok(slot_mapping) || !dev_ok(k_cache) || !dev_ok(v_cache))
    return KVQ_ERR_ARG;
  if (fmt != KVQ_BF16 && (!dev_ok(k_scale) || !dev_ok(v_scale))) return KVQ_ERR_ARG;
  return cuda_rc(launch_append(k, v, slot_mapping, num_tokens, k_cache, v_cache, k_scale, v_scale,
                               fmt, *dims, stream));
}

size_t kvq_decode_workspace_bytes(int32_t batch, int32_t max_context_len, int32_t partition_tokens,
                                  kvq_fmt fmt, const kvq_dims* dims) {
  DecodePlan plan;
  if (check_decode_common(batch, max_context_len, partition_tokens, fmt, dims, &plan) != KVQ_OK)
    return 0;
  return plan.total;
}

int kvq_decode_partial(const void* q, int32_t batch, const void* k_cache, const void* v_cache,
                       const void* const* scales, const int32_t* block_tables,
                       const int32_t* context_lens, int32_t max_context_len, float sm_scale,
                       void* workspace, size_t workspace_bytes, int32_t partition_tokens,
                       kvq_fmt fmt, const kvq_dims* dims, kvq_stream_t stream) {
  DecodePlan plan;
  int rc = check_decode_common(batch, max_context_len, partition_tokens, fmt, dims, &plan);
  if (rc != KVQ_OK) return rc;
  if (batch == 0) return KVQ_OK;
  const void *ks, *vs;
  rc = check_decode_inputs(q, k_cache, v_cache, scales, block_tables, context_lens, sm_scale, fmt,
                           &ks, &vs);
  if (rc != KVQ_OK) return rc;
  if (!dev_ok(workspace)) return KVQ_ERR_ARG;
  if (workspace_bytes < plan.total) return KVQ_ERR_WORKSPACE;
  return cuda_rc(launch_decode_partial(q, batch, k_cache, v_cache, ks, vs, block_tables,
                                       context_lens, max_context_len, sm_scale, plan, workspace,
                                       fmt, *dims, stream));
}

int kvq_decode_merge(int32_t batch, const int32_t* context_lens, int32_t max_context_len,
                     void* out, kvq_out_dtype out_dtype, const void* workspace,
                     size_t workspace_bytes,
                     int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                     kvq_stream_t stream) {
  DecodePlan plan;
  int rc = check_decode_common(batch, max_context_len, partition_tokens, fmt, dims, &plan);
  if (rc != KVQ_OK) return rc;
  if (out_dtype != KVQ_OUT_BF16 && out_dtype != KVQ_OUT_F32) return KVQ_ERR_ARG;
  if (batch == 0) return KVQ_OK;
  if (!dev_ok(context_lens) || !dev_ok(out) || !dev_ok(workspace)) return KVQ_ERR_ARG;
  if (workspace_bytes < plan.total) return KVQ_ERR_WORKSPACE;
  return cuda_rc(launch_decode_merge(batch, context_lens, max_context_len, out,
                                     out_dtype == KVQ_OUT_F32, workspace, plan, *dims, stream));
}

int kvq_decode_attn(const void* q, int32_t batch, const void* k_cache, const void* v_cache,
                    const void* const* scales, const int32_t* block_tables,
                    const int32_t* context_lens, int32_t max_context_len, float sm_scale,
                    void* out, kvq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                    int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                    kvq_stream_t stream) {
  DecodePlan plan;
  int rc = check_decode_common(batch, max_context_len, partition_tokens, fmt, dims, &plan);
  if (rc != KVQ_OK) return rc;
  if (out_dtype != KVQ_OUT_BF16 && out_dtype != KVQ_OUT_F32) return KVQ_ERR_ARG;
  if (batch == 0) return KVQ_OK;
  if (!dev_ok(out)) return KVQ_ERR_ARG;
  rc = kvq_decode_partial(q, batch, k_cache, v_cache, scales, block_tables, context_lens,
                          max_context_len, sm_scale, workspace, workspace_bytes, partition_tokens,
                          fmt, dims, stream);
  if (rc != KVQ_OK) return rc;
  return kvq_decode_merge(batch, context_lens, max_context_len, out, out_dtype, workspace,
                          workspace_bytes, partition_tokens, fmt, dims, stream);
}

int kvq_set_wait_limit(int64_t cycles) {
  if (cycles < 0) return KVQ_ERR_ARG;
  g_wait_limit.store(cycles == 0 ? kDefaultWaitLimit : (long long)cycles, std::memory_order_relaxed);
  return KVQ_OK;
}

int64_t kvq_get_wait_limit(void) { return decode_wait_limit(); }

int kvq_device_error(uint32_t* flags, int clear) {
  if (!flags) return KVQ_ERR_ARG;
  const int e = read_device_error(flags, clear);
  if (e != 0) return KVQ_ERR_CUDA;
  return *flags ? KVQ_ERR_DEVICE : KVQ_OK;
}

// Multi-query decode: the n_query positions of a query head are the rows
// n_query * h .. n_query * h + n_query - 1 of its KV head's G * n_query rows.
// The decode kernel takes those rows in groups of up to 8 (row_groups), each
// a virtual head of the work list with the KV head's pages, and adds the
// causal limit of each position; the plan, the launch and the merge see
// n_q_heads * n_query query rows per sequence.
namespace {
constexpr int32_t kMaxQueryPositions = 1024;

int verify_launch(const void* q, int32_t batch, int32_t n_query, const void* k_cache,
                  const void* v_cache, const void* const* scales, const int32_t* block_tables,
                  const int32_t* context_lens, int32_t max_context_len, float sm_scale, void* out,
                  kvq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                  int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                  kvq_stream_t stream, bool prefill) {
  if (n_query < 1 || n_query > kMaxQueryPositions) return KVQ_ERR_ARG;
  DecodePlan plan;
  int rc = check_decode_common(batch, max_context_len, partition_tokens, fmt, dims, &plan, n_query);
  if (rc != KVQ_OK) return rc;
  if (out_dtype != KVQ_OUT_BF16 && out_dtype != KVQ_OUT_F32) return KVQ_ERR_ARG;
  if (batch == 0) return KVQ_OK;
  if (!dev_ok(out)) return KVQ_ERR_ARG;
  const void *ks, *vs;
  rc = check_decode_inputs(q, k_cache, v_cache, scales, block_tables, context_lens, sm_scale, fmt,
                           &ks, &vs);
  if (rc != KVQ_OK) return rc;
  if (!dev_ok(workspace)) return KVQ_ERR_ARG;
  if (workspace_bytes < plan.total) return KVQ_ERR_WORKSPACE;
  kvq_dims eff = *dims;
  eff.n_q_heads = dims->n_q_heads * n_query;
  if (prefill) {
    // query rows as the MMA's M dimension (128-row blocks), one count per row
    rc = cuda_rc(launch_prefill_partial(q, batch, k_cache, v_cache, ks, vs, block_tables,
                                        context_lens, max_context_len, sm_scale, plan, workspace,
                                        fmt, *dims, stream, n_query));
    if (rc != KVQ_OK) return rc;
    return cuda_rc(launch_decode_merge(batch, context_lens, max_context_len, out,
                                       out_dtype == KVQ_OUT_F32, workspace, plan, eff, stream, 1));
  }
  rc = cuda_rc(launch_decode_partial(q, batch, k_cache, v_cache, ks, vs, block_tables, context_lens,
                                     max_context_len, sm_scale, plan, workspace, fmt, eff, stream,
                                     n_query));
  if (rc != KVQ_OK) return rc;
  return cuda_rc(launch_decode_merge(batch, context_lens, max_context_len, out,
                                     out_dtype == KVQ_OUT_F32, workspace, plan, eff, stream));
}

size_t verify_ws(int32_t batch, int32_t n_query, int32_t max_context_len,
                 int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims) {
  if (n_query < 1 || n_query > kMaxQueryPositions) return 0;
  DecodePlan plan;
  if (check_decode_common(batch, max_context_len, partition_tokens, fmt, dims, &plan, n_query) !=
      KVQ_OK)
    return 0;
  return plan.total;
}
}  // namespace

size_t kvq_decode_verify_workspace_bytes(int32_t batch, int32_t n_query, int32_t max_context_len,
                                         int32_t partition_tokens, kvq_fmt fmt,
                                         const kvq_dims* dims) {
  return verify_ws(batch, n_query, max_context_len, partition_tokens, fmt, dims);
}

int kvq_decode_verify(const void* q, int32_t batch, int32_t n_query, const void* k_cache,
                      const void* v_cache, const void* const* scales,
                      const int32_t* block_tables, const int32_t* context_lens,
                      int32_t max_context_len, float sm_scale, void* out,
                      kvq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                      int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                      kvq_stream_t stream) {
  return verify_launch(q, batch, n_query, k_cache, v_cache, scales, block_tables, context_lens,
                       max_context_len, sm_scale, out, out_dtype, workspace, workspace_bytes,
                       partition_tokens, fmt, dims, stream, false);
}

size_t kvq_prefill_attn_workspace_bytes(int32_t batch, int32_t chunk_len, int32_t max_context_len,
                                        int32_t partition_tokens, kvq_fmt fmt,
                                        const kvq_dims* dims) {
  return verify_ws(batch, chunk_len, max_context_len, partition_tokens, fmt, dims);
}

int kvq_prefill_attn(const void* q, int32_t batch, int32_t chunk_len, const void* k_cache,
                     const void* v_cache, const void* const* scales, const int32_t* block_tables,
                     const int32_t* context_lens, int32_t max_context_len, float sm_scale,
                     void* out, kvq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                     int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                     kvq_stream_t stream) {
  return verify_launch(q, batch, chunk_len, k_cache, v_cache, scales, block_tables, context_lens,
                       max_context_len, sm_scale, out, out_dtype, workspace, workspace_bytes,
                       partition_tokens, fmt, dims, stream, true);
}

// ---------------------------------------------------------------- KIVI-style low-bit cache
int kvq_kivi_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                    void* k_codes, void* v_codes, void* k_meta, void* v_meta, kvq_fmt fmt,
                    const kvq_dims* dims, kvq_stream_t stream) {
  if (!fmt_kivi(fmt) || num_tokens < 0 || num_tokens % 128 != 0) return KVQ_ERR_ARG;
  int rc = check_dims(dims);
  if (rc != KVQ_OK) return rc;
  if (num_tokens == 0) return KVQ_OK;
  if (!dev_ok(k) || !dev_ok(v) || !dev_ok(slot_mapping) || !dev_ok(k_codes) || !dev_ok(v_codes) ||
      !dev_ok(k_meta) || !dev_ok(v_meta))
    return KVQ_ERR_ARG;
  return cuda_rc(launch_kivi_append(k, v, slot_mapping, num_tokens, k_codes, v_codes, k_meta, v_meta,
                                    kivi_bits(fmt), *dims, stream));
}

namespace {
int kivi_plans(int32_t batch, int32_t max_quant_len, int32_t max_res_len, kvq_fmt fmt,
               const kvq_dims* dims, const kvq_dims* res_dims, DecodePlan* pa, DecodePlan* pb) {
  if (!fmt_kivi(fmt) || batch < 0 || max_quant_len < 0 || max_res_len < 0) return KVQ_ERR_ARG;
  int rc = check_dims(dims);
  if (rc != KVQ_OK) return rc;
  rc = check_dims(res_dims);
  if (rc != KVQ_OK) return rc;
  if (res_dims->n_kv_heads != dims->n_kv_heads || res_dims->n_q_heads != dims->n_q_heads ||
      res_dims->head_dim != dims->head_dim)
    return KVQ_ERR_ARG;
  if (max_quant_len % 128 != 0) return KVQ_ERR_ARG;
  if (int64_t(max_quant_len) > int64_t(dims->max_blocks_per_seq) * dims->block_size ||
      int64_t(max_res_len) > int64_t(res_dims->max_blocks_per_seq) * res_dims->block_size)
    return KVQ_ERR_ARG;
  rc = make_plan(batch, max_quant_len, 0, dims, pa);
  if (rc != KVQ_OK) return rc;
  return make_plan(batch, max_res_len, 0, res_dims, pb);
}
}  // namespace

size_t kvq_kivi_decode_workspace_bytes(int32_t batch, int32_t max_quant_len, int32_t max_res_len,
                                       kvq_fmt fmt, const kvq_dims* dims,
                                       const kvq_dims* res_dims) {
  DecodePlan pa, pb;
  if (kivi_plans(batch, max_quant_len, max_res_len, fmt, dims, res_dims, &pa, &pb) != KVQ_OK)
    return 0;
  return pa.total + pb.total;
}

int kvq_kivi_decode_attn(const void* q, int32_t batch, const void* k_codes, const void* v_codes,
                         const void* const* meta, const int32_t* block_tables,
                         const int32_t* quant_lens, int32_t max_quant_len, const void* res_k,
                         const void* res_v, const int32_t* res_tables, const int32_t* res_lens,
                         int32_t max_res_len, float sm_scale, void* out, kvq_out_dtype out_dtype,
                         void* workspace, size_t workspace_bytes, kvq_fmt fmt,
                         const kvq_dims* dims, const kvq_dims* res_dims, kvq_stream_t stream) {
  DecodePlan pa, pb;
  int rc = kivi_plans(batch, max_quant_len, max_res_len, fmt, dims, res_dims, &pa, &pb);
  if (rc != KVQ_OK) return rc;
  if (out_dtype != KVQ_OUT_BF16 && out_dtype != KVQ_OUT_F32) return KVQ_ERR_ARG;
  if (batch == 0) return KVQ_OK;
  if (!dev_ok(q) || !dev_ok(k_codes) || !dev_ok(v_codes) || !meta || !dev_ok(meta[0]) ||
      !dev_ok(meta[1]) || !dev_ok(block_tables) || !dev_ok(quant_lens) || !dev_ok(res_k) ||
      !dev_ok(res_v) || !dev_ok(res_tables) || !dev_ok(res_lens) || !dev_ok(out) ||
      !dev_ok(workspace))
    return KVQ_ERR_ARG;
  if (!std::isfinite(sm_scale)) return KVQ_ERR_ARG;
  if (workspace_bytes < pa.total + pb.total) return KVQ_ERR_WORKSPACE;
  return cuda_rc(launch_kivi_decode(q, batch, k_codes, v_codes, meta[0], meta[1], block_tables,
                                    quant_lens, max_quant_len, res_k, res_v, res_tables, res_lens,
                                    max_res_len, sm_scale, out, out_dtype == KVQ_OUT_F32, workspace,
                                    pa, pb, kivi_bits(fmt), *dims, *res_dims, stream));
}

}  // extern "C"
