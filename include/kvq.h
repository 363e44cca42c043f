/*
 * kvq.h - C ABI of libkvq: a quantized paged KV cache (FP8 E4M3 / INT8
 * asymmetric) for autoregressive decode on NVIDIA B200 (sm_100a).
 *
 * The library has two hot operations, both CUDA kernels launched on the
 * caller's stream:
 *   kvq_append       quantize-on-append of new tokens' K and V into the paged pool
 *   kvq_decode_attn  paged GQA decode attention over the quantized cache
 * plus a host-side block allocator and size queries.
 *
 * Sources (web pages, cited by title and section):
 *   [LIMITS]   "KV cache quantization: what FP8/INT8 K and V really give, and
 *              their limits" (molayo1419.me)
 *   [76X]      "Fitting 76x concurrent requests with an FP8 KV cache"
 *              (storycompiler.tistory.com/431)
 *   [COMPRESS] "KV Cache compression" (ryotta.opik.net)
 *   [GUIDE]    "From FP8 KV cache to INT4 weight-only: GPU LLM serving
 *              optimisation guide (May 2026)" (daewooki.github.io)
 *
 * Conventions for every call
 * --------------------------
 * - Pointers marked "device" are CUDA device pointers on the current device;
 *   "host" pointers are ordinary host memory. Every device pointer must be
 *   16-byte aligned.
 * - The caller owns every buffer and the stream. The hot calls (kvq_append,
 *   kvq_decode_attn and its two phases) allocate no memory; the split-K
 *   scratch of decode comes from the caller (kvq_decode_workspace_bytes).
 * - Return value: KVQ_OK (0) or a negative kvq_status. Argument checks run on
 *   the host before any launch; a failed check launches nothing. Launches are
 *   asynchronous: KVQ_ERR_CUDA reports a launch failure only.
 * - The decode kernels (kvq_decode_attn, _partial, _verify, kvq_prefill_attn)
 *   and the merge are launched as programmatic dependents of the kernel ahead
 *   of them on the stream: when that kernel signals early completion (the
 *   append kernel of kvq_append does), their set-up (barriers, tensor
 *   memory) overlaps its tail, and they read every argument in device memory
 *   (context lengths, query, block tables, scales, pages, workspace) only
 *   after it has finished. Ordinary kernels never signal, so with them the
 *   order is the usual one.
 * - Data-dependent faults (a slot or block id outside the pool, a context
 *   length beyond the block table or beyond max_context_len) cannot be seen on
 *   the host. Kernels skip the offending token, page or sequence and set a bit
 *   in a per-device error word that kvq_device_error() reads.
 * - Supported shapes: block_size 16; head_dim 64 or 128; GQA group
 *   G = n_q_heads / n_kv_heads in {1, 2, 4, 8}. Other shapes return
 *   KVQ_ERR_UNSUPPORTED.
 *
 * Device layouts (one layer; K and V are separate arrays)
 * -------------------------------------------------------
 *   element  E = 1 byte (FP8 E4M3 code or int8 code) or 2 bytes (BF16)
 *   page     one (block, KV head): 16 tokens x head_dim elements = 16*D*E bytes,
 *            made of 16-byte chunks
 *   K cache  [num_blocks][n_kv_heads][2][D*E/16][8][16/E]: chunk (c, t) holds
 *            elements d in [c*16/E, (c+1)*16/E) of token t, at page offset
 *            (t/8)*8*D*E + c*128 + (t%8)*16 (each 8-token group stores its
 *            16-byte chunks as 8 x 16-byte core matrices)
 *   V cache  [num_blocks][n_kv_heads][E][D][16/E]: chunk (u, d) holds tokens
 *            t in [u*16/E, (u+1)*16/E) of channel d, at page offset (u*D + d)*16
 *            (the page is stored transposed)
 *   scales   FP8 (E4M3, E5M2): [num_blocks][n_kv_heads][block_size] BF16 scale
 *            INT8: [num_blocks][n_kv_heads][block_size][2] BF16 {scale, zero_point}
 *            BF16: none (pass NULL)
 * Both pages are tensor-core operands as stored: K is the K-major operand of
 * S = K.q (rows = tokens), V the K-major operand of O^T = V^T.P (rows =
 * channels); a page is one contiguous 1-D copy.
 * A token at sequence position p lives in slot
 *   block_tables[b][p / block_size] * block_size + p % block_size.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t). NULL is the legacy default stream. */
typedef struct CUstream_st* kvq_stream_t;

typedef enum {
  KVQ_BF16 = 0,      /* unquantized BF16 cache: the comparison baseline */
  KVQ_FP8_E4M3 = 1,  /* OCP E4M3 codes (max 448, RNE, saturating) + BF16 scale */
  KVQ_INT8_ASYM = 2, /* signed int8 codes + BF16 {scale, zero_point} */
  KVQ_FP8_E5M2 = 3,  /* OCP E5M2 codes (max 57344, RNE, saturating) + BF16 scale */
  KVQ_INT8_CHANNEL = 4, /* signed int8 codes, symmetric, one static BF16 scale per
                           (KV head, channel), given by the caller */
  KVQ_INT8_TENSOR = 5,  /* signed int8 codes, symmetric, one static BF16 scale for
                           the whole K (and one for V) cache, given by the caller */
  KVQ_KIVI2 = 6,        /* KIVI-style 2-bit codes: K per channel over 128-token
                           groups, V per token; kvq_kivi_* calls only */
  KVQ_KIVI4 = 7         /* the same with 4-bit codes */
} kvq_fmt;

typedef enum {
  KVQ_OUT_BF16 = 0,  /* decode output rounded to BF16 (round to nearest even) */
  KVQ_OUT_F32 = 1    /* decode output as the kernel's FP32 result */
} kvq_out_dtype;

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_ARG = -1,            /* null/misaligned pointer, bad size or enum */
  KVQ_ERR_UNSUPPORTED = -2,    /* shape outside the supported set */
  KVQ_ERR_WORKSPACE = -3,      /* decode workspace smaller than required */
  KVQ_ERR_CUDA = -4,           /* a CUDA call or launch failed */
  KVQ_ERR_POOL_EXHAUSTED = -5, /* the block allocator has too few free blocks */
  KVQ_ERR_DEVICE = -6          /* kvq_device_error found a flagged fault */
} kvq_status;

/* Bits of the per-device error word (kvq_device_error). */
#define KVQ_DEVERR_SLOT 0x1u     /* append: slot >= num_blocks * block_size */
#define KVQ_DEVERR_BLOCK 0x2u    /* decode: block id outside [0, num_blocks) */
#define KVQ_DEVERR_CONTEXT 0x4u  /* decode: context_len < 0, > max_context_len,
                                    or > max_blocks_per_seq * block_size */
#define KVQ_DEVERR_TIMEOUT 0x8u  /* decode: a pipeline wait ran out (about 1 s by
                                    default, kvq_set_wait_limit); the output rows
                                    of the sequences that CTA worked on come out
                                    as NaN and the call's output is not valid */

typedef struct {
  int32_t num_blocks;         /* blocks in the pool */
  int32_t block_size;         /* tokens per block; must be 16 */
  int32_t n_kv_heads;         /* KV heads (Hk) */
  int32_t n_q_heads;          /* query heads (Hq); Hq / Hk in {1, 2, 4, 8} */
  int32_t head_dim;           /* D: 64 or 128 */
  int32_t max_blocks_per_seq; /* W: the row length of block_tables */
} kvq_dims;

/* Library version (major * 10000 + minor * 100 + patch). */
int kvq_version(void);

/* Static text for a kvq_status value. */
const char* kvq_status_string(int status);

/*
 * Bytes of ONE cache array (K or V) and of its scale array for `dims`.
 * [COMPRESS] "1. The KV cache memory problem" gives the element count
 * 2 x layers x n_kv_heads x head_dim x tokens x bytes; one cache array is one
 * of the two halves of one layer for num_blocks * block_size tokens.
 * meta_bytes is 0 for KVQ_BF16; for the per-token formats it is the per-token
 * scale array of kvq_append; for KVQ_INT8_CHANNEL it is the static
 * [n_kv_heads][head_dim] BF16 scale array, for KVQ_INT8_TENSOR one BF16 value
 * (padded to 16 bytes). Host only; no CUDA call.
 */
int kvq_cache_bytes(const kvq_dims* dims, kvq_fmt fmt, size_t* cache_bytes,
                    size_t* meta_bytes);

/* ------------------------------------------------------------------------ */
/* Host block allocator.                                                      */
/* [GUIDE] "Core concepts 2) PagedAttention": the cache is a pool of fixed-    */
/* size blocks and each request is mapped to just the blocks it needs.        */
/* [COMPRESS] "6.2": low-bit K/V fit more tokens into each block's bytes.     */
/* The allocator hands out block ids; device memory is the caller's. Not     */
/* thread-safe: one pool per thread, or external locking.                     */
/* ------------------------------------------------------------------------ */
typedef struct kvq_pool kvq_pool;

/* Create a pool of dims->num_blocks free blocks for `n_layers` layers of the
 * given format. *out receives the handle (host memory owned by the library;
 * release with kvq_pool_destroy). */
int kvq_pool_create(const kvq_dims* dims, kvq_fmt fmt, int32_t n_layers, kvq_pool** out);
void kvq_pool_destroy(kvq_pool* pool);

/* Device bytes the pool stands for: element bytes of K and V over all layers
 * (the closed form of [COMPRESS] section 1 for num_blocks * block_size tokens)
 * and the bytes of their per-token scale arrays. */
int kvq_pool_bytes(const kvq_pool* pool, size_t* element_bytes, size_t* meta_bytes);

/* Number of free blocks. */
int kvq_pool_num_free(const kvq_pool* pool, int32_t* n_free);

/* Take n blocks (all or none) and write their ids to block_ids[0..n) (host).
 * KVQ_ERR_POOL_EXHAUSTED if fewer than n are free. */
int kvq_pool_alloc(kvq_pool* pool, int32_t n, int32_t* block_ids);

/* Return n blocks. KVQ_ERR_ARG (and nothing freed) if an id is out of range,
 * repeated, or not currently allocated. */
int kvq_pool_free(kvq_pool* pool, int32_t n, const int32_t* block_ids);

/* Grow one sequence from cur_len to cur_len + n_new tokens: allocate the new
 * blocks it needs into block_table_row[ceil(cur_len/bs) .. ) (host, length
 * dims->max_blocks_per_seq) and write the slot of each new token to
 * slots[0..n_new) (host). All or nothing: KVQ_ERR_POOL_EXHAUSTED or
 * KVQ_ERR_ARG (row too short) leave the row and the pool unchanged. */
int kvq_pool_extend_seq(kvq_pool* pool, int32_t* block_table_row, int32_t cur_len,
                        int32_t n_new, int64_t* slots);

/* ------------------------------------------------------------------------ */
/* Quantize-on-append.                                                        */
/* [LIMITS] "What KV cache quantization actually is": K/V are quantized only */
/* when stored, the scale comes from the full BF16 values, and the per-token */
/* scales are kept in BF16. [LIMITS] "Formats you will actually meet": E4M3  */
/* for K/V; INT8 per-token asymmetric with a (scale, zero_point) pair.       */
/* [COMPRESS] "5.1" and "6.3": quantize right after K,V are computed.        */
/* ------------------------------------------------------------------------ */
/*
 * k, v          device, [num_tokens][n_kv_heads][head_dim] BF16, contiguous:
 *               the new tokens' keys and values.
 * slot_mapping  device, [num_tokens] int64: destination slot of each token
 *               (block = slot / block_size, offset = slot % block_size).
 *               A negative slot skips the token; a slot >= num_blocks *
 *               block_size skips it and sets KVQ_DEVERR_SLOT. Slots must be
 *               distinct within one call.
 * k_cache, v_cache  device, the layouts in the file header.
 * k_scale, v_scale  device scale arrays (NULL for KVQ_BF16). Written per token
 *               for FP8 / E5M2 / INT8_ASYM; read-only inputs for the static
 *               formats: KVQ_INT8_CHANNEL [n_kv_heads][head_dim] BF16,
 *               KVQ_INT8_TENSOR [1] BF16.
 * Per (token, KV head) row of D values:
 *   FP8:  s = bf16_rne(max|x| / 448); code = e4m3_rne_satfinite(x / s)
 *   INT8: xmin = min(0, min x), xmax = max(0, max x);
 *         s = bf16_rne((xmax - xmin) / 255); zp = clamp(-128 - rint(xmin / s), -128, 127);
 *         code = clamp(rint(x / s) + zp, -128, 127)
 *   INT8_CHANNEL / INT8_TENSOR ([LIMITS] "Formats you will actually meet": a
 *         per-channel scale per head_dim slice, or one per-tensor scale, fixed
 *         ahead of the tokens): s = the given scale of the element's (head,
 *         channel) or of the cache; code = clamp(rint(x / s), -127, 127);
 *         s <= 0 (or NaN) stores code 0. Dequantized value: code * s.
 *   (all divisions IEEE f32, rint ties to even; s == 0 stores zero codes and zp 0)
 *   BF16: the values are copied.
 */
int kvq_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
               void* k_cache, void* v_cache, void* k_scale, void* v_scale, kvq_fmt fmt,
               const kvq_dims* dims, kvq_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Paged GQA decode attention.                                                */
/* [GUIDE] "Core concepts 1)": decode attends one query position against the */
/* whole cached K/V and is bound by reading it. [LIMITS] "What KV cache      */
/* quantization actually is": dequantization is fused into the attention    */
/* kernel right before the matmuls. [76X] "4. Precision loss?": 8-bit        */
/* storage, FP32 accumulation. [COMPRESS] "5.1": a separate dequantization   */
/* kernel would give back the bandwidth gain.                                */
/* ------------------------------------------------------------------------ */
/*
 * Scratch bytes kvq_decode_attn needs for these sizes. partition_tokens is the
 * split-K chunk (a positive multiple of 128): the smallest run of one
 * sequence's tokens a decode CTA takes, so one (sequence, KV head) produces at
 * most ceil(max_context_len / partition_tokens) + 1 partials. 0 lets the
 * library choose the smallest chunk that gives at most 16 partials.
 * Returns 0 for invalid arguments.
 */
size_t kvq_decode_workspace_bytes(int32_t batch, int32_t max_context_len, int32_t partition_tokens,
                                  kvq_fmt fmt, const kvq_dims* dims);

/*
 * out[b][h] = softmax_t(sm_scale * q[b][h] . K_b[t][h/G]) weighted sum of V_b[t][h/G],
 * t = 0 .. context_lens[b]-1, where K_b/V_b are the dequantized cache rows read
 * through block_tables[b]; G = n_q_heads / n_kv_heads (query head h uses KV head h / G).
 *
 * q             device, [batch][n_q_heads][head_dim] BF16.
 * k_cache, v_cache  device, the layouts in the file header.
 * scales        host array of 2 device pointers {k_scale, v_scale} (both NULL, or
 *               scales itself NULL, for KVQ_BF16): the per-token arrays of
 *               kvq_append, or the static arrays of the INT8_CHANNEL / TENSOR
 *               formats (for those the kernel multiplies the query by the K
 *               scale of each channel and the output by the V scale of each
 *               channel, since code * s_d factors out of both sums).
 * block_tables  device, [batch][max_blocks_per_seq] int32.
 * context_lens  device, [batch] int32: cached tokens per sequence, the token
 *               appended in this step included. 0 gives an all-zero output row.
 * max_context_len  host bound on every context_lens[b]; sizes the split grid.
 * sm_scale      softmax scale (usually 1/sqrt(head_dim)).
 * out           device, [batch][n_q_heads][head_dim], BF16 or FP32 per out_dtype.
 * out_dtype     KVQ_OUT_BF16 or KVQ_OUT_F32. The kernel computes in FP32; BF16
 *               output is that result rounded to nearest even.
 * workspace     device scratch of at least kvq_decode_workspace_bytes(...) bytes;
 *               contents on entry do not matter.
 * partition_tokens  as for kvq_decode_workspace_bytes (0 = automatic).
 * The work (sequence, KV head, 128-token tile) is shared evenly over the
 * GPU's resident CTAs; each CTA's run of one (sequence, head) computes an
 * online-softmax partial (max, sum, unnormalized output) and a merge kernel
 * combines the partials with a log-sum-exp rescale.
 */
int kvq_decode_attn(const void* q, int32_t batch, const void* k_cache, const void* v_cache,
                    const void* const* scales, const int32_t* block_tables,
                    const int32_t* context_lens, int32_t max_context_len, float sm_scale,
                    void* out, kvq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                    int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                    kvq_stream_t stream);

/* The two phases of kvq_decode_attn, for callers that time or overlap them.
 * kvq_decode_partial writes per-chunk partials into the workspace;
 * kvq_decode_merge reads them and writes out. Same arguments and errors as
 * kvq_decode_attn; the two calls must use the same batch, max_context_len,
 * partition_tokens, dims and workspace. */
int kvq_decode_partial(const void* q, int32_t batch, const void* k_cache, const void* v_cache,
                       const void* const* scales, const int32_t* block_tables,
                       const int32_t* context_lens, int32_t max_context_len, float sm_scale,
                       void* workspace, size_t workspace_bytes, int32_t partition_tokens,
                       kvq_fmt fmt, const kvq_dims* dims, kvq_stream_t stream);
int kvq_decode_merge(int32_t batch, const int32_t* context_lens, int32_t max_context_len,
                     void* out, kvq_out_dtype out_dtype, const void* workspace,
                     size_t workspace_bytes,
                     int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                     kvq_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Decode without a caller workspace. The pages have no counterpart to this:   */
/* it is kvq_decode_attn with its scratch taken from the library itself.       */
/* ------------------------------------------------------------------------ */
/* Size of the scratch array compiled into the library (64 MiB per device). */
#define KVQ_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * Same arguments, result and errors as kvq_decode_attn, minus the workspace.
 * For callers that cannot allocate device memory while decoding (a plugin
 * inside another framework's step, where the framework owns all device memory;
 * a latency-critical loop that must not hit the device synchronisation of
 * cudaMalloc/cudaFree). The split-K scratch comes from one static device array
 * of KVQ_NOALLOC_SCRATCH_BYTES, held by every GPU that loads the library until
 * the process exits; the call allocates nothing.
 * - Every argument check of kvq_decode_attn runs first, with the same result
 *   (batch 0 included). Then KVQ_ERR_WORKSPACE, before touching the device,
 *   when the split plan (kvq_decode_workspace_bytes for the same arguments)
 *   needs more than KVQ_NOALLOC_SCRATCH_BYTES; use a larger partition_tokens
 *   or kvq_decode_attn.
 * - The first call on each device looks up the array's device address (with
 *   that device current) and caches it together with the id of the device's
 *   context; after a cudaDeviceReset the next call sees a new context and
 *   looks the address up again. Make the first call on a device (and the first
 *   after a reset) before any stream capture.
 * - All calls share the array and it keeps the last call's contents (nothing in
 *   it needs to start at zero). Calls whose kernels overlap on the GPU (other
 *   streams, other host threads) race on it: serialise them.
 */
int kvq_decode_attn_noalloc(const void* q, int32_t batch, const void* k_cache,
                            const void* v_cache, const void* const* scales,
                            const int32_t* block_tables, const int32_t* context_lens,
                            int32_t max_context_len, float sm_scale, void* out,
                            kvq_out_dtype out_dtype, int32_t partition_tokens, kvq_fmt fmt,
                            const kvq_dims* dims, kvq_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Multi-query decode (speculative verification).                              */
/* [LIMITS] "How it interacts with speculative decoding": the target model     */
/* scores all K+1 proposed positions in one pass that reads the quantized     */
/* cache and dequantizes it on the fly.                                        */
/* ------------------------------------------------------------------------ */
/*
 * Each sequence b has n_query new positions: the last n_query tokens of its
 * context, already appended (context_lens[b] counts them). Position j
 * (0 <= j < n_query) attends causally to tokens 0 .. context_lens[b] -
 * n_query + j, i.e. to everything before it and to itself:
 *   out[b][h][j] = softmax_t(sm_scale * q[b][h][j] . K_b[t][h/G]) weighted sum
 *                  of V_b[t][h/G] over t < context_lens[b] - n_query + 1 + j.
 * A position with no visible token gives an all-zero row.
 *
 * q    device, [batch][n_q_heads][n_query][head_dim] BF16.
 * out  device, [batch][n_q_heads][n_query][head_dim], BF16 or FP32 per out_dtype.
 * The cache, scales, block tables and the other arguments are those of
 * kvq_decode_attn. n_query in 1 .. 1024 (KVQ_ERR_ARG otherwise). The G *
 * n_query query rows of a KV head are taken in groups of up to 8 rows (the
 * largest of 8, 4, 2, 1 that divides G * n_query); each group streams the KV
 * head's pages once, and the groups of one KV head run side by side on the
 * GPU, so their repeated reads of a page mostly come from L2.
 * workspace  at least kvq_decode_verify_workspace_bytes(...) bytes; contents on
 *            entry do not matter.
 */
size_t kvq_decode_verify_workspace_bytes(int32_t batch, int32_t n_query, int32_t max_context_len,
                                         int32_t partition_tokens, kvq_fmt fmt,
                                         const kvq_dims* dims);
int kvq_decode_verify(const void* q, int32_t batch, int32_t n_query, const void* k_cache,
                      const void* v_cache, const void* const* scales,
                      const int32_t* block_tables, const int32_t* context_lens,
                      int32_t max_context_len, float sm_scale, void* out,
                      kvq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                      int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                      kvq_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Chunked-prefill attention over the quantized cache.                         */
/* [GUIDE] "Core concepts 1)": prefill processes a prompt's tokens together,   */
/* decode one token at a time against the cache. A long prompt prefilled in    */
/* chunks appends each chunk's K/V (kvq_append, the bulk path) and then lets   */
/* the chunk's queries attend, causally, to everything cached so far: the     */
/* earlier chunks through the quantized pages and the chunk itself.           */
/* ------------------------------------------------------------------------ */
/*
 * The chunk's chunk_len tokens are the last chunk_len tokens of each
 * sequence's context, already appended (context_lens[b] counts them). Chunk
 * position j attends to tokens 0 .. context_lens[b] - chunk_len + j (the same
 * rule as kvq_decode_verify with n_query = chunk_len):
 *   out[b][h][j] = softmax_t(sm_scale * q[b][h][j] . K_b[t][h/G]) weighted sum
 *                  of V_b[t][h/G] over t < context_lens[b] - chunk_len + 1 + j.
 * q    device, [batch][n_q_heads][chunk_len][head_dim] BF16 (head-major).
 * out  device, the same shape, BF16 or FP32 per out_dtype.
 * chunk_len in 1 .. 1024; the other arguments and errors are those of
 * kvq_decode_verify. workspace: kvq_prefill_attn_workspace_bytes(...) bytes
 * (the same size as kvq_decode_verify's for the same arguments).
 * Unlike kvq_decode_verify (the cache tokens as the rows of the tensor-core
 * products, at most 8 query rows per product), this call runs a kernel whose
 * products take 128 query rows of a KV head at a time (the chunk's positions
 * of its G query heads) against 64-token halves of the cache's 128-token
 * tiles, with the 8-bit codes expanded to f16 in shared memory: the scores
 * are exact products accumulated in FP32 and the softmax weights keep 22 bits
 * (two f16 parts; 16 bits as two bf16 parts for a BF16 cache), so the outputs
 * agree with kvq_decode_verify's to rounding.
 */
size_t kvq_prefill_attn_workspace_bytes(int32_t batch, int32_t chunk_len, int32_t max_context_len,
                                        int32_t partition_tokens, kvq_fmt fmt,
                                        const kvq_dims* dims);
int kvq_prefill_attn(const void* q, int32_t batch, int32_t chunk_len, const void* k_cache,
                     const void* v_cache, const void* const* scales, const int32_t* block_tables,
                     const int32_t* context_lens, int32_t max_context_len, float sm_scale,
                     void* out, kvq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                     int32_t partition_tokens, kvq_fmt fmt, const kvq_dims* dims,
                     kvq_stream_t stream);

/* ------------------------------------------------------------------------ */
/* KIVI-style low-bit cache (KVQ_KIVI2, KVQ_KIVI4).                            */
/* [COMPRESS] "2.1": K has a few outlier channels and V a per-token spread, so */
/* K is quantized per channel and V per token. [COMPRESS] "3.1", KIVI:         */
/* asymmetric 2-bit codes, K per channel, V per token, the most recent tokens  */
/* kept in full precision as a residual. [LIMITS] "Formats you will actually   */
/* meet": the 4-bit variants do the same; 4-bit storage is a quarter of BF16.  */
/* ------------------------------------------------------------------------ */
/*
 * A sequence's positions come in groups of 128 (eight 16-token blocks of its
 * block table). A complete group is stored as b-bit codes (b = 2 or 4):
 *   K, per (KV head, channel) over the group's 128 positions, and
 *   V, per (position, KV head) over the head_dim channels:
 *   z = bf16_rne(min x), s = bf16_rne(f32(max x - min x) / (2^b - 1)),
 *   code = clamp(rint(f32(x - z) / s), 0, 2^b - 1) (IEEE f32 subtraction and
 *   division, rint ties to even; s == 0 stores code 0; a zero z or s is +0);
 *   the value read back is code * s + z.
 * The positions after a sequence's last complete group (its residual) stay in
 * BF16 in a separate cache of the KVQ_BF16 layout (kvq_append with KVQ_BF16,
 * its own block tables); the caller quantizes a group once it is complete.
 *
 * Device layouts (one layer, K and V separate):
 *   codes    [num_blocks][n_kv_heads][16 * head_dim * b / 8] bytes per page.
 *            A page is made of 16-code units of 2b bytes. K: the unit of (token
 *            t, channels 16c .. 16c+15) is unit ((t/8) * head_dim/16 + c) * 8 +
 *            t%8 (the tensor-core K operand order); V: the unit of channel d
 *            (tokens 0..15 of the page) is unit d. Inside a unit, code e = 4m + j
 *            (m, j in 0..3): for b = 2 the unit is one 32-bit word and the code
 *            is at bit 8j + 2m; for b = 4 it is word m/2, bit 8j + 4(m%2)
 *            (little-endian words), so one shift and mask per m unpacks four
 *            codes into bytes.
 *   k_meta   [num_blocks][n_kv_heads][16][2] BF16 {s, z}: block i of a group
 *            (i = its position in the sequence / 16, mod 8) holds channels
 *            i*D/8 .. i*D/8 + D/8 - 1 of the group's K (entries 0 .. D/8-1).
 *   v_meta   [num_blocks][n_kv_heads][16][2] BF16 {s, z} per token.
 */

/*
 * Quantize whole groups. k, v: device [num_tokens][n_kv_heads][head_dim] BF16,
 * num_tokens a multiple of 128: every run of 128 tokens is one complete group
 * (positions 128g .. 128g+127 of one sequence, in order). slot_mapping: device
 * [num_tokens] int64; the 16 tokens of a block must fill it in order (slot %
 * 16 == token % 16, one block per 16 tokens). A group whose slots are all
 * negative is skipped; one that breaks the rule above or leaves the pool is
 * skipped and sets KVQ_DEVERR_SLOT. fmt: KVQ_KIVI2 or KVQ_KIVI4.
 * Returns KVQ_ERR_ARG for a token count that is not a multiple of 128.
 */
int kvq_kivi_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                    void* k_codes, void* v_codes, void* k_meta, void* v_meta, kvq_fmt fmt,
                    const kvq_dims* dims, kvq_stream_t stream);

/*
 * Decode attention over each sequence's quantized groups and its residual:
 *   out[b][h] = softmax over the union of (quant_lens[b] tokens read through
 *   block_tables[b], dequantized as above) and (res_lens[b] BF16 tokens read
 *   through res_tables[b] from res_k / res_v), as kvq_decode_attn defines it.
 * quant_lens[b] must be a multiple of 128 (a length that is not is cut to its
 * whole groups and sets KVQ_DEVERR_CONTEXT); max_quant_len (a multiple of 128)
 * and max_res_len bound them. dims describes the low-bit pool, res_dims the
 * residual BF16 pool (same heads and head_dim). meta: host array {k_meta,
 * v_meta}. The groups run on the tensor cores from the codes (the query is
 * rebuilt per group with its channel scales) into split-K partials; a second
 * kernel attends the residual tokens in FP32 and merges them with those
 * partials (a residual block id outside [0, res_dims->num_blocks) skips the
 * token and sets KVQ_DEVERR_BLOCK; a residual length outside [0, max_res_len]
 * or beyond the residual table counts as 0 and sets KVQ_DEVERR_CONTEXT).
 * workspace: at least kvq_kivi_decode_workspace_bytes(...) bytes.
 */
size_t kvq_kivi_decode_workspace_bytes(int32_t batch, int32_t max_quant_len, int32_t max_res_len,
                                       kvq_fmt fmt, const kvq_dims* dims,
                                       const kvq_dims* res_dims);
int kvq_kivi_decode_attn(const void* q, int32_t batch, const void* k_codes, const void* v_codes,
                         const void* const* meta, const int32_t* block_tables,
                         const int32_t* quant_lens, int32_t max_quant_len, const void* res_k,
                         const void* res_v, const int32_t* res_tables, const int32_t* res_lens,
                         int32_t max_res_len, float sm_scale, void* out, kvq_out_dtype out_dtype,
                         void* workspace, size_t workspace_bytes, kvq_fmt fmt,
                         const kvq_dims* dims, const kvq_dims* res_dims, kvq_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Device error word and the decode wait bound.                               */
/* ------------------------------------------------------------------------ */
/*
 * Every wait inside the decode kernels (for a page copy, an MMA, the softmax
 * warps) gives up after a bounded number of SM clock cycles instead of hanging
 * the GPU. A CTA whose wait runs out stops issuing work, waits for the copies
 * and MMAs it already issued, writes NaN markers in place of its partials (so
 * the affected output rows are NaN, not plausible values), frees its tensor
 * memory, returns, and sets KVQ_DEVERR_TIMEOUT; the context stays usable.
 * kvq_set_wait_limit sets that bound, in SM clock cycles, for decode launches
 * made after the call on any device (0 restores the default of 2e9 cycles,
 * about one second at 2 GHz). A bound far below a page's load time makes the
 * waits run out on purpose, which is how the failure path is tested. The
 * setting is process-wide and not ordered against launches from other host
 * threads. Returns KVQ_ERR_ARG for a negative value.
 */
int kvq_set_wait_limit(int64_t cycles);
/* The bound decode launches currently use, in SM clock cycles. */
int64_t kvq_get_wait_limit(void);

/* Read (and if `clear` is non-zero, reset) the current device's error word
 * (KVQ_DEVERR_* bits) into *flags (host). Synchronizes the device. Returns
 * KVQ_ERR_DEVICE if any bit was set, KVQ_OK otherwise. */
int kvq_device_error(uint32_t* flags, int clear);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
