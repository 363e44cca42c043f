// Internal declarations shared by the host translation units of libkvq.
// Device code lives in kvq_kernels.cu; the C ABI in kvq_api.cpp; the block
// allocator in kvq_pool.cpp.
#pragma once

#include <cstddef>
#include <cstdint>

#include "kvq.h"

namespace kvq {

constexpr int kBlockSize = 16;     // tokens per page
constexpr int kTileTokens = 128;   // partition_tokens granularity

// Element bytes of the cache arrays and BF16 metadata values per (token, head).
inline int elem_bytes(kvq_fmt f) { return f == KVQ_BF16 ? 2 : 1; }
inline bool fmt_fp8(kvq_fmt f) { return f == KVQ_FP8_E4M3 || f == KVQ_FP8_E5M2; }
// Per-token metadata values (0 for BF16 and the static-scale formats).
inline int meta_values(kvq_fmt f) { return fmt_fp8(f) ? 1 : (f == KVQ_INT8_ASYM ? 2 : 0); }
// Static-scale INT8: one scale per (KV head, channel) or one per cache.
inline bool fmt_static(kvq_fmt f) { return f == KVQ_INT8_CHANNEL || f == KVQ_INT8_TENSOR; }
// The 8-bit / BF16 formats of kvq_append and kvq_decode_attn.
inline bool fmt_valid(int f) { return f >= KVQ_BF16 && f <= KVQ_INT8_TENSOR; }
// The KIVI-style low-bit formats (kvq_kivi_* calls) and their code bits.
inline bool fmt_kivi(int f) { return f == KVQ_KIVI2 || f == KVQ_KIVI4; }
inline int kivi_bits(int f) { return f == KVQ_KIVI2 ? 2 : 4; }

// Checks the shape rules of kvq.h. Returns KVQ_OK, KVQ_ERR_ARG or KVQ_ERR_UNSUPPORTED.
int check_dims(const kvq_dims* d);

// The query rows of one KV head (G query heads x n_query positions) are taken
// by the decode kernel in row groups of gp rows, gp the largest of 8, 4, 2, 1
// that divides the row count: each group is one "virtual head" of the work
// list that reads the KV head's pages. Returns the number of groups per KV
// head and writes gp.
inline int row_groups(int rows, int* gp) {
  int g = 8;
  while (g > 1 && rows % g != 0) g /= 2;
  *gp = g;
  return rows / g;
}

// Split-K plan of one decode call.
struct DecodePlan {
  int32_t partition;   // tokens per split (multiple of kTileTokens); the smallest
                       // run of one sequence's tokens a decode CTA takes
  int32_t max_splits;  // splits of the longest sequence
  int32_t slots;       // partial slots per (sequence, query head): max_splits + 1
  size_t o_bytes;      // partial outputs  [B][Hq][slots][D] f32
  size_t ml_bytes;     // partial (max, sum) [B][Hq][slots][2] f32
  size_t cnt_bytes;    // partials written per (sequence, row group) [B][Hk * groups] int32
                       // (decode kernel) or per query row [B][Hq * n_query] (prefill kernel)
  size_t total;        // workspace bytes (256-aligned pieces)
};
// Fills `plan` for query rows n_q_heads * n_query per sequence; returns KVQ_OK
// or KVQ_ERR_ARG.
int make_plan(int32_t batch, int32_t max_ctx, int32_t partition_tokens, const kvq_dims* d,
              DecodePlan* plan, int32_t n_query = 1);

// Number of SMs of the current device (148 if no device can be queried).
int device_sm_count();

// Bound, in SM clock cycles, on each pipeline wait of the decode kernels
// launched from now on (kvq_set_wait_limit; default about one second).
long long decode_wait_limit();

// Argument checks shared by every decode entry point (format, dims, sizes,
// max_context_len against the block-table width) and the split plan.
// Returns KVQ_OK, KVQ_ERR_ARG or KVQ_ERR_UNSUPPORTED.
int check_decode_common(int32_t batch, int32_t max_ctx, int32_t partition_tokens, kvq_fmt fmt,
                        const kvq_dims* dims, DecodePlan* plan, int32_t n_query = 1);
// Device-pointer checks of a decode call; *ks, *vs receive the scale arrays.
int check_decode_inputs(const void* q, const void* kc, const void* vc, const void* const* scales,
                        const int32_t* tables, const int32_t* ctx, float sm_scale, kvq_fmt fmt,
                        const void** ks, const void** vs);

// Kernel launchers (kvq_kernels.cu). They assume validated arguments and return
// a cudaError_t value as int.
int launch_append(const void* k, const void* v, const int64_t* slots, int32_t T, void* kc,
                  void* vc, void* ks, void* vs, kvq_fmt fmt, const kvq_dims& d, void* stream);
int launch_decode_partial(const void* q, int32_t B, const void* kc, const void* vc,
                          const void* ks, const void* vs, const int32_t* tables,
                          const int32_t* ctx, int32_t max_ctx, float sm_scale,
                          const DecodePlan& plan, void* ws, kvq_fmt fmt, const kvq_dims& d,
                          void* stream, int n_query = 1);
// Chunked-prefill partials: the n_query positions of the G query heads of a KV
// head as 128-row blocks of the query-row-major kernel; one count per row.
int launch_prefill_partial(const void* q, int32_t B, const void* kc, const void* vc,
                           const void* ks, const void* vs, const int32_t* tables,
                           const int32_t* ctx, int32_t max_ctx, float sm_scale,
                           const DecodePlan& plan, void* ws, kvq_fmt fmt, const kvq_dims& d,
                           void* stream, int n_query);
int launch_decode_merge(int32_t B, const int32_t* ctx, int32_t max_ctx, void* out, bool out_f32,
                        const void* ws, const DecodePlan& plan, const kvq_dims& d, void* stream,
                        int rows_per_count = 0);
int read_device_error(uint32_t* flags, int clear);
int launch_kivi_decode(const void* q, int32_t B, const void* kc, const void* vc, const void* km,
                       const void* vm, const int32_t* tables, const int32_t* qlens,
                       int32_t max_qlen, const void* rk, const void* rv,
                       const int32_t* rtables, const int32_t* rlens, int32_t max_rlen,
                       float sm_scale, void* out, bool out_f32, void* ws, const DecodePlan& pa,
                       const DecodePlan& pb, int bits, const kvq_dims& d, const kvq_dims& rd,
                       void* stream);
int launch_kivi_append(const void* k, const void* v, const int64_t* slots, int32_t T, void* kc,
                       void* vc, void* km, void* vm, int bits, const kvq_dims& d, void* stream);

}  // namespace kvq
